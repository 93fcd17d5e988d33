// time_shift.cu -- the time-mix prologue of RWKV_TimeMix ("代码连连看——RWKV",
// section RWKV_TimeMix, jit_func): the input shifted one token along T
// (time_shift pads a zero row before T and drops the last row) blended per
// channel with the token itself, once for each of k, v, r:
//
//     x_m,t = x_t * mix_m + x_{t-1} * (1 - mix_m),   x_{-1} = x_prev (or 0)
//
// and its backward
//
//     gx_t    = sum_m g_m,t mix_m + sum_m g_m,t+1 (1 - mix_m)   (no second sum at t = T-1)
//     gmix_m  = sum_{b,t} g_m,t (x_t - x_{t-1})
//     gx_prev = sum_m g_m,0 (1 - mix_m)
//
// Both are pure streams: one read of x gives all n_mix outputs (the three
// blends of the page read x and its shifted copy three times each), and one
// read of the n_mix gradients and x gives gx and the mix gradients. A thread
// owns a few channels (forward: 16 bytes, 4 float32 or 8 bf16; backward: 4
// channels) over a run of Lt tokens of one sequence and keeps the previous
// token in registers, so only the first token of each run is read twice.
// Loads are issued a batch of tokens at a time and kept packed until used,
// so that enough bytes are in flight per SM for the HBM rate. The mix
// gradients leave as per-run partial sums that a second kernel adds in a
// fixed order (deterministic).
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

namespace {

constexpr int kTsThreads = 128;
constexpr int kTsReduceWarps = 8;

template <class E>
struct Vec16 {
  static constexpr int N = 16 / sizeof(E);  // channels per 16-byte access
};
// Channels per thread of the backward (its registers hold n_mix + 1 rows of
// them per token in flight) and tokens whose loads it issues together.
template <class E>
struct BwdVec {
  static constexpr int N = sizeof(E) == 2 ? TS_BWD_BF16_VEC : 4;
};

// 16 bytes of E <-> N floats
__device__ __forceinline__ void ld_vec(const float* p, float (&f)[4]) {
  const float4 q = *reinterpret_cast<const float4*>(p);
  f[0] = q.x;
  f[1] = q.y;
  f[2] = q.z;
  f[3] = q.w;
}
__device__ __forceinline__ void ld_vec(const __nv_bfloat16* p, float (&f)[8]) {
  const uint4 q = *reinterpret_cast<const uint4*>(p);
  f[0] = bf16lo(q.x);
  f[1] = bf16hi(q.x);
  f[2] = bf16lo(q.y);
  f[3] = bf16hi(q.y);
  f[4] = bf16lo(q.z);
  f[5] = bf16hi(q.z);
  f[6] = bf16lo(q.w);
  f[7] = bf16hi(q.w);
}
__device__ __forceinline__ void ld_vec(const __nv_bfloat16* p, float (&f)[4]) {
  const uint2 q = *reinterpret_cast<const uint2*>(p);
  f[0] = bf16lo(q.x);
  f[1] = bf16hi(q.x);
  f[2] = bf16lo(q.y);
  f[3] = bf16hi(q.y);
}
__device__ __forceinline__ void st_vec(__nv_bfloat16* p, const float (&f)[4]) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
}
__device__ __forceinline__ void st_vec(float* p, const float (&f)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
}
__device__ __forceinline__ void st_vec(__nv_bfloat16* p, const float (&f)[8]) {
  *reinterpret_cast<uint4*>(p) =
      make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
}
// The raw 16- or 8-byte word of N channels: the backward keeps its batch of
// loads packed (bf16 unpacked takes twice the registers) and unpacks at use.
template <class E, int N>
struct Raw;
template <>
struct Raw<float, 4> {
  using T = float4;
  static __device__ __forceinline__ void unpack(const T& q, float (&f)[4]) {
    f[0] = q.x;
    f[1] = q.y;
    f[2] = q.z;
    f[3] = q.w;
  }
};
template <>
struct Raw<__nv_bfloat16, 8> {
  using T = uint4;
  static __device__ __forceinline__ void unpack(const T& q, float (&f)[8]) {
    f[0] = bf16lo(q.x);
    f[1] = bf16hi(q.x);
    f[2] = bf16lo(q.y);
    f[3] = bf16hi(q.y);
    f[4] = bf16lo(q.z);
    f[5] = bf16hi(q.z);
    f[6] = bf16lo(q.w);
    f[7] = bf16hi(q.w);
  }
};
template <>
struct Raw<__nv_bfloat16, 4> {
  using T = uint2;
  static __device__ __forceinline__ void unpack(const T& q, float (&f)[4]) {
    f[0] = bf16lo(q.x);
    f[1] = bf16hi(q.x);
    f[2] = bf16lo(q.y);
    f[3] = bf16hi(q.y);
  }
};
template <class E, int N>
__device__ __forceinline__ typename Raw<E, N>::T ld_raw(const E* p) {
  return *reinterpret_cast<const typename Raw<E, N>::T*>(p);
}

template <int N>
__device__ __forceinline__ void ld_mix(const float* p, float (&f)[N]) {
#pragma unroll
  for (int i = 0; i < N; i += 4) {
    const float4 q = *reinterpret_cast<const float4*>(p + i);
    f[i] = q.x;
    f[i + 1] = q.y;
    f[i + 2] = q.z;
    f[i + 3] = q.w;
  }
}

// Tokens [t0, t1) of sequence b for the thread's 16 bytes of channels at c.
struct TsRun {
  int b, c, t0, t1, run;
  bool valid;
};
__device__ __forceinline__ TsRun ts_run(int T, int C, int ncb, int nrun, int Lt, int N) {
  TsRun r;
  const int cb = (int)(blockIdx.x % ncb);
  const int rest = (int)(blockIdx.x / ncb);
  r.run = rest % nrun;
  r.b = rest / nrun;
  r.c = (cb * kTsThreads + (int)threadIdx.x) * N;
  r.t0 = r.run * Lt;
  r.t1 = min(T, r.t0 + Lt);
  r.valid = r.c < C;
  return r;
}

// Forward. NMIX blends of one x read; `plane` = B*T*C elements between the
// outputs. Loads of U tokens are issued before any of them is used.
template <class E, int NMIX>
__global__ void __launch_bounds__(kTsThreads) time_shift_mix_kernel(const E* __restrict__ x,
                                                                    const float* __restrict__ mix,
                                                                    const E* __restrict__ x_prev,
                                                                    E* __restrict__ out, int T, int C, int ncb,
                                                                    int nrun, int Lt, int64_t plane) {
  constexpr int N = Vec16<E>::N;
  constexpr int U = TS_FWD_U;
  using R = Raw<E, N>;
  const TsRun r = ts_run(T, C, ncb, nrun, Lt, N);
  if (!r.valid) return;
  float m[NMIX][N], om[NMIX][N];
#pragma unroll
  for (int i = 0; i < NMIX; ++i) {
    ld_mix<N>(mix + (int64_t)i * C + r.c, m[i]);
#pragma unroll
    for (int n = 0; n < N; ++n) om[i][n] = 1.f - m[i][n];
  }
  const int64_t row0 = ((int64_t)r.b * T + r.t0) * C + r.c;
  float prev[N];
  if (r.t0 > 0) {
    ld_vec(x + row0 - C, prev);
  } else if (x_prev) {
    ld_vec(x_prev + (int64_t)r.b * C + r.c, prev);
  } else {
#pragma unroll
    for (int n = 0; n < N; ++n) prev[n] = 0.f;
  }
  const E* xp = x + row0;
  E* op = out + row0;
  for (int t = r.t0; t < r.t1; t += U) {
    typename R::T raw[U];
#pragma unroll
    for (int j = 0; j < U; ++j)
      if (t + j < r.t1) raw[j] = ld_raw<E, N>(xp + (int64_t)j * C);
#pragma unroll
    for (int j = 0; j < U; ++j) {
      if (t + j < r.t1) {
        float cur[N];
        R::unpack(raw[j], cur);
#pragma unroll
        for (int i = 0; i < NMIX; ++i) {
          float o[N];
#pragma unroll
          for (int n = 0; n < N; ++n) o[n] = __fmaf_rn(cur[n], m[i][n], __fmul_rn(prev[n], om[i][n]));
          st_vec(op + (int64_t)i * plane + (int64_t)j * C, o);
        }
#pragma unroll
        for (int n = 0; n < N; ++n) prev[n] = cur[n];
      }
    }
    xp += (int64_t)U * C;
    op += (int64_t)U * C;
  }
}

// Backward. Walks the run upward holding x_{t-1} and g_t; per token it
// reads x_t and the NMIX gradients of token t+1, the loads of U tokens
// issued before any of them is used. part: [NMIX][B*nrun][C] partial mix
// gradients of each run.
template <class E, int NMIX>
__global__ void __launch_bounds__(kTsThreads) time_shift_mix_bwd_kernel(
    const E* __restrict__ x, const float* __restrict__ mix, const E* __restrict__ x_prev, const E* __restrict__ g,
    E* __restrict__ gx, E* __restrict__ gx_prev, float* __restrict__ part, int B, int T, int C, int ncb, int nrun,
    int Lt, int64_t plane) {
  constexpr int N = BwdVec<E>::N;
  constexpr int U = TS_BWD_U;
  const TsRun r = ts_run(T, C, ncb, nrun, Lt, N);
  if (!r.valid) return;
  float m[NMIX][N];
#pragma unroll
  for (int i = 0; i < NMIX; ++i) ld_mix<N>(mix + (int64_t)i * C + r.c, m[i]);
  const int64_t row0 = ((int64_t)r.b * T + r.t0) * C + r.c;
  float xprev[N];
  if (r.t0 > 0) {
    ld_vec(x + row0 - C, xprev);
  } else if (x_prev) {
    ld_vec(x_prev + (int64_t)r.b * C + r.c, xprev);
  } else {
#pragma unroll
    for (int n = 0; n < N; ++n) xprev[n] = 0.f;
  }
  float gcur[NMIX][N], acc[NMIX][N];
#pragma unroll
  for (int i = 0; i < NMIX; ++i) {
    ld_vec(g + (int64_t)i * plane + row0, gcur[i]);
#pragma unroll
    for (int n = 0; n < N; ++n) acc[i][n] = 0.f;
  }
  if (r.t0 == 0 && gx_prev) {
    float gp[N];
#pragma unroll
    for (int n = 0; n < N; ++n) {
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < NMIX; ++i) s = __fmaf_rn(gcur[i][n], 1.f - m[i][n], s);
      gp[n] = s;
    }
    st_vec(gx_prev + (int64_t)r.b * C + r.c, gp);
  }
  const E* xp = x + row0;
  const E* gp = g + row0 + C;  // token t+1
  E* gxp = gx + row0;
  using R = Raw<E, N>;
  for (int t = r.t0; t < r.t1; t += U) {
    typename R::T xr[U], gr[U][NMIX];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      if (t + j < r.t1) xr[j] = ld_raw<E, N>(xp + (int64_t)j * C);
      if (t + j + 1 < T && t + j < r.t1) {
#pragma unroll
        for (int i = 0; i < NMIX; ++i) gr[j][i] = ld_raw<E, N>(gp + (int64_t)i * plane + (int64_t)j * C);
      } else {
#pragma unroll
        for (int i = 0; i < NMIX; ++i) gr[j][i] = typename R::T{};
      }
    }
#pragma unroll
    for (int j = 0; j < U; ++j) {
      if (t + j < r.t1) {
        float xt[1][N], gn[1][NMIX][N];
        R::unpack(xr[j], xt[0]);
#pragma unroll
        for (int i = 0; i < NMIX; ++i) R::unpack(gr[j][i], gn[0][i]);
        float o[N];
#pragma unroll
        for (int n = 0; n < N; ++n) {
          float s = 0.f;
#pragma unroll
          for (int i = 0; i < NMIX; ++i) {
            s = __fmaf_rn(gcur[i][n], m[i][n], s);
            s = __fmaf_rn(gn[0][i][n], 1.f - m[i][n], s);
            acc[i][n] = __fmaf_rn(gcur[i][n], xt[0][n] - xprev[n], acc[i][n]);
          }
          o[n] = s;
        }
        st_vec(gxp + (int64_t)j * C, o);
#pragma unroll
        for (int n = 0; n < N; ++n) {
          xprev[n] = xt[0][n];
#pragma unroll
          for (int i = 0; i < NMIX; ++i) gcur[i][n] = gn[0][i][n];
        }
      }
    }
    xp += (int64_t)U * C;
    gp += (int64_t)U * C;
    gxp += (int64_t)U * C;
  }
  const int64_t rows = (int64_t)B * nrun;
  const int64_t prow = (int64_t)r.b * nrun + r.run;
#pragma unroll
  for (int i = 0; i < NMIX; ++i) {
    float* pp = part + ((int64_t)i * rows + prow) * C + r.c;
#pragma unroll
    for (int n = 0; n < N; n += 4) *reinterpret_cast<float4*>(pp + n) = make_float4(acc[i][n], acc[i][n + 1],
                                                                                    acc[i][n + 2], acc[i][n + 3]);
  }
}

// gmix[i][c] = sum over the rows of part[i]: warp q adds rows q, q + 8, ...
// in ascending order, then warp 0 adds the 8 warp sums in order (the
// result does not depend on timing).
__global__ void __launch_bounds__(32 * kTsReduceWarps) time_shift_reduce_kernel(const float* __restrict__ part,
                                                                               int64_t rows, int C,
                                                                               float* __restrict__ gmix) {
  __shared__ float sw[kTsReduceWarps][32];
  const int lane = threadIdx.x % 32, q = threadIdx.x / 32;
  const int c = blockIdx.x * 32 + lane;
  const int i = blockIdx.y;
  const float* p = part + (int64_t)i * rows * C;
  float a = 0.f;
  if (c < C)
    for (int64_t r = q; r < rows; r += kTsReduceWarps) a += p[r * C + c];
  sw[q][lane] = a;
  __syncthreads();
  if (q == 0 && c < C) {
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < kTsReduceWarps; ++k) s += sw[k][lane];
    gmix[(int64_t)i * C + c] = s;
  }
}


template <class E, int NMIX>
wkv_status run_ts_fwd(const TimeShiftArgs& a, cudaStream_t stream, const char** why) {
  const TsShape s = time_shift_shape(a.B, a.T, a.C, Vec16<E>::N);
  const int64_t plane = a.B * a.T * a.C;
  time_shift_mix_kernel<E, NMIX><<<(unsigned)(s.ncb * s.nrun * a.B), kTsThreads, 0, stream>>>(
      static_cast<const E*>(a.x), a.mix, static_cast<const E*>(a.x_prev), static_cast<E*>(a.out), (int)a.T,
      (int)a.C, s.ncb, s.nrun, s.Lt, plane);
  if (cudaGetLastError() != cudaSuccess) {
    *why = "time_shift_mix kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

template <class E, int NMIX>
wkv_status run_ts_bwd(const TimeShiftArgs& a, cudaStream_t stream, const char** why) {
  const TsShape s = time_shift_shape(a.B, a.T, a.C, BwdVec<E>::N);
  const int64_t plane = a.B * a.T * a.C;
  time_shift_mix_bwd_kernel<E, NMIX><<<(unsigned)(s.ncb * s.nrun * a.B), kTsThreads, 0, stream>>>(
      static_cast<const E*>(a.x), a.mix, static_cast<const E*>(a.x_prev), static_cast<const E*>(a.g),
      static_cast<E*>(a.gx), static_cast<E*>(a.gx_prev), a.part, (int)a.B, (int)a.T, (int)a.C, s.ncb, s.nrun,
      s.Lt, plane);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) {
    time_shift_reduce_kernel<<<dim3((unsigned)ceil_div(a.C, 32), NMIX), 32 * kTsReduceWarps, 0, stream>>>(
        a.part, a.B * s.nrun, (int)a.C, a.gmix);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    *why = "time_shift_mix backward kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

template <class E>
wkv_status ts_dispatch(const TimeShiftArgs& a, bool bwd, cudaStream_t stream, const char** why) {
  switch (a.n_mix) {
    case 1: return bwd ? run_ts_bwd<E, 1>(a, stream, why) : run_ts_fwd<E, 1>(a, stream, why);
    case 2: return bwd ? run_ts_bwd<E, 2>(a, stream, why) : run_ts_fwd<E, 2>(a, stream, why);
    default: return bwd ? run_ts_bwd<E, 3>(a, stream, why) : run_ts_fwd<E, 3>(a, stream, why);
  }
}

}  // namespace

TsShape time_shift_shape(int64_t B, int64_t T, int64_t C, int vec) {
  TsShape s;
  s.ncb = (int)ceil_div(C, (int64_t)kTsThreads * vec);
  // runs per sequence: enough CTAs for ~16 per SM, runs of at least 16 tokens
  const int64_t want = ceil_div(148 * 16, std::max<int64_t>(1, B * s.ncb));
  const int64_t most = std::max<int64_t>(1, ceil_div(T, 16));
  const int64_t nrun = std::max<int64_t>(1, std::min(want, most));
  s.Lt = (int)std::max<int64_t>(1, ceil_div(T, nrun));
  s.nrun = (int)std::max<int64_t>(1, ceil_div(T, s.Lt));
  return s;
}

wkv_status launch_time_shift_mix(const TimeShiftArgs& a, cudaStream_t stream, const char** why) {
  return a.dtype == WKV_BF16 ? ts_dispatch<__nv_bfloat16>(a, false, stream, why)
                             : ts_dispatch<float>(a, false, stream, why);
}

wkv_status launch_time_shift_mix_backward(const TimeShiftArgs& a, cudaStream_t stream, const char** why) {
  return a.dtype == WKV_BF16 ? ts_dispatch<__nv_bfloat16>(a, true, stream, why)
                             : ts_dispatch<float>(a, true, stream, why);
}

}  // namespace wkv
