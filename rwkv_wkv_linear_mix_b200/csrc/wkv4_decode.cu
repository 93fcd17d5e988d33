// wkv4_decode.cu -- the T = 1 fast path of the RWKV-4 slot step (batched
// decode: every slot of a web-rwkv style batch takes exactly one token per
// call, web-rwkv crate page, section "批量推理" / batched inference; the RNN
// form that carries the state between calls is the one the RWKV-4 code
// walkthrough page "代码连连看——RWKV" closes with).
//
// wkv4_chunk_step serves any mix of token counts per slot with one warp per
// 32 channels of a slot, walking the slot's tokens; with one token per slot
// that leaves each thread a handful of 4-byte accesses and the call bound by
// latency. Here the slots' state rows, keys and values are one flat stream:
// a thread takes 4 adjacent channels of one slot (16-byte state accesses, 8-
// or 16-byte key/value accesses) and runs the same float32 scalar step as the
// chunk step for each, so outputs and states are bit-identical to
// wkv4_chunk_step fed one token per slot.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

namespace {

constexpr int kDecThreads = 128;

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void st4(float* p, float4 x) { *reinterpret_cast<float4*>(p) = x; }
__device__ __forceinline__ float comp(const float4& x, int j) {
  return j == 0 ? x.x : j == 1 ? x.y : j == 2 ? x.z : x.w;
}

__device__ __forceinline__ void ld_tok4(const float* p, float (&f)[4]) {
  const float4 q = ld4(p);
  f[0] = q.x;
  f[1] = q.y;
  f[2] = q.z;
  f[3] = q.w;
}
__device__ __forceinline__ void ld_tok4(const __nv_bfloat16* p, float (&f)[4]) {
  const uint2 q = *reinterpret_cast<const uint2*>(p);
  f[0] = bf16lo(q.x);
  f[1] = bf16hi(q.x);
  f[2] = bf16lo(q.y);
  f[3] = bf16hi(q.y);
}
__device__ __forceinline__ void st_tok4(float* p, const float (&f)[4]) { st4(p, make_float4(f[0], f[1], f[2], f[3])); }
__device__ __forceinline__ void st_tok4(__nv_bfloat16* p, const float (&f)[4]) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
}

// One token for each of S slots; thread i takes channels 4i' .. 4i' + 3 of
// the flat [S][C] index 4i (C % 4 == 0, so the four share a slot).
template <class E>
__global__ void __launch_bounds__(kDecThreads) wkv4_decode_kernel(int64_t total, int C, const float* __restrict__ w,
                                                                 const float* __restrict__ u,
                                                                 const E* __restrict__ k, const E* __restrict__ v,
                                                                 E* __restrict__ y, float* __restrict__ state) {
  const int64_t i = ((int64_t)blockIdx.x * kDecThreads + threadIdx.x) * 4;
  if (i >= total) return;
  const int64_t s = i / C;
  const int c = (int)(i - s * C);
  float* sp = state + s * 5 * C + c;
  const float4 aa = ld4(sp), bb = ld4(sp + C), base = ld4(sp + 2 * (int64_t)C), nn = ld4(sp + 3 * (int64_t)C),
               rf = ld4(sp + 4 * (int64_t)C);
  const float4 w4 = ld4(w + c), u4 = ld4(u + c);
  float kk[4], vv[4], yy[4], o[5][4];
  ld_tok4(k + i, kk);
  ld_tok4(v + i, vv);
  float w2c[4], u2c[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    w2c[j] = __fmul_rn(comp(w4, j), kLog2e);
    u2c[j] = __fmul_rn(comp(u4, j), kLog2e);
  }
  // output form per channel pair (c, c + 1), (c + 2, c + 3), as every kernel decides it
  const bool sc01 = wkv4_scaled_pair(u2c[0], w2c[0], u2c[1], w2c[1]);
  const bool sc23 = wkv4_scaled_pair(u2c[2], w2c[2], u2c[3], w2c[3]);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    Wkv4State st = {comp(aa, j), comp(bb, j), comp(base, j), comp(nn, j)};
    // a slot that has absorbed nothing yet takes its reference from this token
    const float ref = st.base == kEmptyPP ? wkv4_ref(kk[j]) : comp(rf, j);
    yy[j] = wkv4_token(st, wkv4_key(kk[j], ref), vv[j], u2c[j], w2c[j], j < 2 ? sc01 : sc23,
                       wkv4_out_scale(u2c[j], w2c[j]));
    o[0][j] = st.aa;
    o[1][j] = st.bb;
    o[2][j] = st.base;
    o[3][j] = st.n;
    o[4][j] = ref;
  }
  st_tok4(y + i, yy);
#pragma unroll
  for (int r = 0; r < 5; ++r) st4(sp + r * (int64_t)C, make_float4(o[r][0], o[r][1], o[r][2], o[r][3]));
}

}  // namespace

wkv_status launch_wkv4_decode_step(int64_t S, int64_t C, int dtype, const float* w, const float* u, const void* k,
                                   const void* v, void* y, float* state, cudaStream_t stream, const char** why) {
  const int64_t total = S * C;
  const unsigned grid = (unsigned)ceil_div(total / 4, kDecThreads);
  if (dtype == WKV_BF16)
    wkv4_decode_kernel<__nv_bfloat16><<<grid, kDecThreads, 0, stream>>>(
        total, (int)C, w, u, static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
        static_cast<__nv_bfloat16*>(y), state);
  else
    wkv4_decode_kernel<float><<<grid, kDecThreads, 0, stream>>>(total, (int)C, w, u, static_cast<const float*>(k),
                                                                static_cast<const float*>(v), static_cast<float*>(y),
                                                                state);
  if (cudaGetLastError() != cudaSuccess) {
    *why = "wkv4_decode_step kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

}  // namespace wkv
