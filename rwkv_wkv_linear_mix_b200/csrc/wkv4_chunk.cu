// wkv4_chunk.cu -- RWKV-4 WKV as a state-carrying step over batched,
// variable-length inference slots (web-rwkv crate page, section "批量推理" /
// batched inference: num_batch slots, at most token_chunk_size tokens per
// run() call, empty slots skipped, state persisting between calls).
//
// A thread serves 4 adjacent channels of one slot: it loads the slot's
// (aa, bb, base, n, ref) rows for them as 16-byte words, runs the same
// float32 step as wkv4_forward (its packed pair form, two pairs) over the
// slot's tokens of this call, writes y and stores the state back. A call moves at
// most a few tens of MB, so the kernel is bound by latency and by the bytes
// it has in flight: each thread issues the loads of a whole group of tokens
// (kept packed until used) before it starts computing, and 8- or 16-byte
// accesses give a warp 128 channels of a token row per load.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

constexpr int kChunkThreads = 128;

template <class E>
struct ChunkRaw;  // 4 channels of one token, packed
template <>
struct ChunkRaw<float> {
  using T = float4;
  static constexpr int kGroup = 16;
  static __device__ __forceinline__ void unpack(const T& q, float (&f)[4]) {
    f[0] = q.x;
    f[1] = q.y;
    f[2] = q.z;
    f[3] = q.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&f)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  }
};
template <>
struct ChunkRaw<__nv_bfloat16> {
  using T = uint2;
  static constexpr int kGroup = 32;
  static __device__ __forceinline__ void unpack(const T& q, float (&f)[4]) {
    f[0] = bf16lo(q.x);
    f[1] = bf16hi(q.x);
    f[2] = bf16lo(q.y);
    f[3] = bf16hi(q.y);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&f)[4]) {
    *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
  }
};

__device__ __forceinline__ float comp4(const float4& x, int j) {
  return j == 0 ? x.x : j == 1 ? x.y : j == 2 ? x.z : x.w;
}

template <class E>
__global__ void __launch_bounds__(kChunkThreads) wkv4_chunk_kernel(int S, int C, const float* __restrict__ w,
                                                                  const float* __restrict__ u,
                                                                  const E* __restrict__ k, const E* __restrict__ v,
                                                                  E* __restrict__ y, int64_t n_tokens,
                                                                  const int32_t* __restrict__ cu,
                                                                  float* __restrict__ state, unsigned* err) {
  using R = ChunkRaw<E>;
  constexpr int G = R::kGroup;
  const int nq = C / 4;
  const int64_t gid = (int64_t)blockIdx.x * kChunkThreads + threadIdx.x;
  if (gid >= (int64_t)S * nq) return;
  const int s = (int)(gid / nq);
  const int c = (int)(gid - (int64_t)s * nq) * 4;
  const int64_t beg = cu[s];
  const int64_t end = cu[s + 1];
  if (end == beg) return;  // empty slot: skipped, state untouched
  if (end < beg || beg < 0 || end > n_tokens) {
    if (c == 0) record_error(err, WKV_DEVERR_BAD_SLOT);
    return;
  }
  const E* kp = k + beg * C + c;
  const E* vp = v + beg * C + c;
  E* yp = y + beg * C + c;
  const int64_t n = end - beg;
  // the first group of tokens is requested before the state, so that both
  // round trips overlap
  typename R::T kr[G], vr[G];
  auto load_group = [&](int64_t t0) {
#pragma unroll
    for (int j = 0; j < G; ++j) {
      if (t0 + j < n) {
        kr[j] = *reinterpret_cast<const typename R::T*>(kp + (t0 + j) * C);
        vr[j] = *reinterpret_cast<const typename R::T*>(vp + (t0 + j) * C);
      }
    }
  };
  load_group(0);

  float* sp = state + (int64_t)s * 5 * C + c;
  const float4 aa = *reinterpret_cast<const float4*>(sp), bb = *reinterpret_cast<const float4*>(sp + C),
               base = *reinterpret_cast<const float4*>(sp + 2 * (int64_t)C),
               nn = *reinterpret_cast<const float4*>(sp + 3 * (int64_t)C),
               rf = *reinterpret_cast<const float4*>(sp + 4 * (int64_t)C);
  const float4 w4 = *reinterpret_cast<const float4*>(w + c), u4 = *reinterpret_cast<const float4*>(u + c);
  // two channel pairs, each on the packed fp32 pair form of the step (its
  // components round exactly as the scalar step)
  Wkv4State2 st[2];
  float2 ref[2], w2[2], u2[2];
  float k0[4];
  R::unpack(kr[0], k0);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int j = 2 * h;
    st[h] = {make_float2(comp4(aa, j), comp4(aa, j + 1)), make_float2(comp4(bb, j), comp4(bb, j + 1)),
             make_float2(comp4(base, j), comp4(base, j + 1)), make_float2(comp4(nn, j), comp4(nn, j + 1))};
    // a slot that has absorbed nothing yet takes its reference from this call's first token
    ref[h] = make_float2(st[h].base.x == kEmptyPP ? wkv4_ref(k0[j]) : comp4(rf, j),
                         st[h].base.y == kEmptyPP ? wkv4_ref(k0[j + 1]) : comp4(rf, j + 1));
    w2[h] = make_float2(__fmul_rn(comp4(w4, j), kLog2e), __fmul_rn(comp4(w4, j + 1), kLog2e));
    u2[h] = make_float2(__fmul_rn(comp4(u4, j), kLog2e), __fmul_rn(comp4(u4, j + 1), kLog2e));
  }
  for (int64_t t0 = 0; t0 < n; t0 += G) {
    if (t0 > 0) load_group(t0);
#pragma unroll
    for (int j = 0; j < G; ++j) {
      if (t0 + j < n) {
        float kk[4], vv[4], yy[4];
        R::unpack(kr[j], kk);
        R::unpack(vr[j], vv);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 yv = wkv4_token2(st[h], wkv4_key2(make_float2(kk[2 * h], kk[2 * h + 1]), ref[h]),
                                        make_float2(vv[2 * h], vv[2 * h + 1]), u2[h], w2[h]);
          yy[2 * h] = yv.x;
          yy[2 * h + 1] = yv.y;
        }
        R::store(yp + (t0 + j) * C, yy);
      }
    }
  }
  *reinterpret_cast<float4*>(sp) = make_float4(st[0].aa.x, st[0].aa.y, st[1].aa.x, st[1].aa.y);
  *reinterpret_cast<float4*>(sp + C) = make_float4(st[0].bb.x, st[0].bb.y, st[1].bb.x, st[1].bb.y);
  *reinterpret_cast<float4*>(sp + 2 * (int64_t)C) =
      make_float4(st[0].base.x, st[0].base.y, st[1].base.x, st[1].base.y);
  *reinterpret_cast<float4*>(sp + 3 * (int64_t)C) = make_float4(st[0].n.x, st[0].n.y, st[1].n.x, st[1].n.y);
  *reinterpret_cast<float4*>(sp + 4 * (int64_t)C) = make_float4(ref[0].x, ref[0].y, ref[1].x, ref[1].y);
}

__global__ void wkv4_state_init_kernel(int64_t total, int C, float* __restrict__ state) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const int64_t comp = (i / C) % 5;  // 0: aa, 1: bb, 2: base, 3: n, 4: ref
  state[i] = comp == 2 ? kEmptyPP : 0.f;
}

wkv_status launch_wkv4_state_init(int64_t S, int64_t C, float* state, cudaStream_t stream, const char** why) {
  const int64_t total = S * 5 * C;
  wkv4_state_init_kernel<<<(unsigned)ceil_div(total, 256), 256, 0, stream>>>(total, (int)C, state);
  if (cudaGetLastError() != cudaSuccess) {
    *why = "wkv4_state_init kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

wkv_status launch_wkv4_chunk_step(const Wkv4ChunkArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  const unsigned grid = (unsigned)ceil_div(a.S * (a.C / 4), kChunkThreads);
  if (a.dtype == WKV_BF16)
    wkv4_chunk_kernel<__nv_bfloat16><<<grid, kChunkThreads, 0, stream>>>(
        (int)a.S, (int)a.C, a.w, a.u, static_cast<const __nv_bfloat16*>(a.k), static_cast<const __nv_bfloat16*>(a.v),
        static_cast<__nv_bfloat16*>(a.y), a.n_tokens, a.cu_tokens, a.state, err);
  else
    wkv4_chunk_kernel<float><<<grid, kChunkThreads, 0, stream>>>((int)a.S, (int)a.C, a.w, a.u,
                                                                 static_cast<const float*>(a.k),
                                                                 static_cast<const float*>(a.v),
                                                                 static_cast<float*>(a.y), a.n_tokens, a.cu_tokens,
                                                                 a.state, err);
  if (cudaGetLastError() != cudaSuccess) {
    *why = "wkv4_chunk_step kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

}  // namespace wkv
