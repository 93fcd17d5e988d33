// wkv4_chunk.cu -- RWKV-4 WKV as a state-carrying step over batched,
// variable-length inference slots (web-rwkv crate page, section "批量推理" /
// batched inference: num_batch slots, at most token_chunk_size tokens per
// run() call, empty slots skipped, state persisting between calls).
//
// A thread serves a channel pair of one slot: it loads the slot's
// (aa, bb, base, n, ref) for them, runs the same float32 step as
// wkv4_forward (its packed pair form) over the slot's tokens of this call,
// writes y and stores the state back. A slot's tokens are a serial chain, so
// the kernel is bound by latency: each thread issues the loads of a whole
// group of tokens (kept packed until used), the first group before the
// state, and a thread per pair gives the SMs as many warps as the batch has.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

// Channels per thread (2: one packed pair, or 4: two pairs) and threads per
// CTA. Two channels per thread give twice the warps, which is what the
// latency-bound token chains want; four give wider accesses.
#ifndef WKV4_CHUNK_CH
#define WKV4_CHUNK_CH 2
#endif
constexpr int kChunkCh = WKV4_CHUNK_CH;
constexpr int kChunkThreads = kChunkCh == 2 ? 64 : 128;
constexpr int kChunkMinBlocks = kChunkCh == 2 ? 8 : 1;  // two channels: <= 128 registers, 16 warps per SM

// NCH channels of one token, packed as loaded.
template <class E, int NCH>
struct ChunkRaw;
template <>
struct ChunkRaw<float, 4> {
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
struct ChunkRaw<__nv_bfloat16, 4> {
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
template <>
struct ChunkRaw<float, 2> {
  using T = float2;
  static constexpr int kGroup = 16;
  static __device__ __forceinline__ void unpack(const T& q, float (&f)[2]) {
    f[0] = q.x;
    f[1] = q.y;
  }
  static __device__ __forceinline__ void store(float* p, const float (&f)[2]) {
    *reinterpret_cast<float2*>(p) = make_float2(f[0], f[1]);
  }
};
template <>
struct ChunkRaw<__nv_bfloat16, 2> {
  using T = uint32_t;
  static constexpr int kGroup = 16;
  static __device__ __forceinline__ void unpack(const T& q, float (&f)[2]) {
    f[0] = bf16lo(q);
    f[1] = bf16hi(q);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&f)[2]) {
    *reinterpret_cast<uint32_t*>(p) = pack_bf16x2(f[0], f[1]);
  }
};

template <class E>
__global__ void __launch_bounds__(kChunkThreads, kChunkMinBlocks) wkv4_chunk_kernel(int S, int C, const float* __restrict__ w,
                                                                  const float* __restrict__ u,
                                                                  const E* __restrict__ k, const E* __restrict__ v,
                                                                  E* __restrict__ y, int64_t n_tokens,
                                                                  const int32_t* __restrict__ cu,
                                                                  float* __restrict__ state, unsigned* err) {
  constexpr int NCH = kChunkCh, NP = NCH / 2;
  using R = ChunkRaw<E, NCH>;
  constexpr int G = R::kGroup;
  const int nq = C / NCH;
  const int64_t gid = (int64_t)blockIdx.x * kChunkThreads + threadIdx.x;
  if (gid >= (int64_t)S * nq) return;
  const int s = (int)(gid / nq);
  const int c = (int)(gid - (int64_t)s * nq) * NCH;
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

  // NP channel pairs, each on the packed fp32 pair form of the step (its
  // components round exactly as the scalar step)
  float* sp = state + (int64_t)s * 5 * C + c;
  Wkv4State2 st[NP];
  float2 ref[NP], w2[NP], u2[NP];
  float k0[NCH];
  R::unpack(kr[0], k0);
#pragma unroll
  for (int h = 0; h < NP; ++h) {
    const int j = 2 * h;
    st[h] = {ld_pair(sp + j), ld_pair(sp + C + j), ld_pair(sp + 2 * (int64_t)C + j), ld_pair(sp + 3 * (int64_t)C + j)};
    const float2 rf = ld_pair(sp + 4 * (int64_t)C + j);
    // a slot that has absorbed nothing yet takes its reference from this call's first token
    ref[h] = make_float2(st[h].base.x == kEmptyPP ? wkv4_ref(k0[j]) : rf.x,
                         st[h].base.y == kEmptyPP ? wkv4_ref(k0[j + 1]) : rf.y);
    const float2 wc = ld_pair(w + c + j), uc = ld_pair(u + c + j);
    w2[h] = make_float2(__fmul_rn(wc.x, kLog2e), __fmul_rn(wc.y, kLog2e));
    u2[h] = make_float2(__fmul_rn(uc.x, kLog2e), __fmul_rn(uc.y, kLog2e));
  }
  // output form of each pair (wkv4_scaled_pair: decided from u and w alone)
  bool scaled = true;
  float2 E2[NP];
#pragma unroll
  for (int h = 0; h < NP; ++h) {
    scaled = scaled && wkv4_scaled_pair2(u2[h], w2[h]);
    E2[h] = wkv4_out_scale2(u2[h], w2[h]);
  }
  auto run = [&](auto scaled_tag) {
    constexpr bool kScaled = decltype(scaled_tag)::value;
    for (int64_t t0 = 0; t0 < n; t0 += G) {
      if (t0 > 0) load_group(t0);
#pragma unroll
      for (int j = 0; j < G; ++j) {
        if (t0 + j < n) {
          float kk[NCH], vv[NCH], yy[NCH];
          R::unpack(kr[j], kk);
          R::unpack(vr[j], vv);
#pragma unroll
          for (int h = 0; h < NP; ++h) {
            const float2 yv = wkv4_token2<kScaled>(st[h], wkv4_key2(make_float2(kk[2 * h], kk[2 * h + 1]), ref[h]),
                                                   make_float2(vv[2 * h], vv[2 * h + 1]), u2[h], w2[h], E2[h]);
            yy[2 * h] = yv.x;
            yy[2 * h + 1] = yv.y;
          }
          R::store(yp + (t0 + j) * C, yy);
        }
      }
    }
  };
  // (with two pairs per thread both must take the scaled form for the fast
  // loop; a thread whose pairs differ runs the exact loop for the one that
  // needs it and the scaled one for the other, pair by pair below)
  if (NP == 1 || scaled) {
    if (scaled)
      run(BoolConst<true>{});
    else
      run(BoolConst<false>{});
  } else {
    for (int64_t t0 = 0; t0 < n; t0 += G) {
      if (t0 > 0) load_group(t0);
      for (int j = 0; j < G && t0 + j < n; ++j) {
        float kk[NCH], vv[NCH], yy[NCH];
        R::unpack(kr[j], kk);
        R::unpack(vr[j], vv);
        for (int h = 0; h < NP; ++h) {
          const float2 yv = wkv4_token2(st[h], wkv4_key2(make_float2(kk[2 * h], kk[2 * h + 1]), ref[h]),
                                        make_float2(vv[2 * h], vv[2 * h + 1]), u2[h], w2[h],
                                        wkv4_scaled_pair2(u2[h], w2[h]), E2[h]);
          yy[2 * h] = yv.x;
          yy[2 * h + 1] = yv.y;
        }
        R::store(yp + (t0 + j) * C, yy);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < NP; ++h) {
    const int j = 2 * h;
    st_pair(sp + j, st[h].aa);
    st_pair(sp + C + j, st[h].bb);
    st_pair(sp + 2 * (int64_t)C + j, st[h].base);
    st_pair(sp + 3 * (int64_t)C + j, st[h].n);
    st_pair(sp + 4 * (int64_t)C + j, ref[h]);
  }
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
  const unsigned grid = (unsigned)ceil_div(a.S * (a.C / kChunkCh), kChunkThreads);
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
