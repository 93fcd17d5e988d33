// wkv4_chunk.cu -- RWKV-4 WKV as a state-carrying step over batched,
// variable-length inference slots (web-rwkv crate page, section "批量推理" /
// batched inference: num_batch slots, at most token_chunk_size tokens per
// run() call, empty slots skipped, state persisting between calls).
//
// One warp serves 32 channels of one slot: it loads the slot's
// (aa, bb, base, n, ref) from the persistent state, runs the same float32
// step as wkv4_forward over the slot's tokens of this call, writes y and stores the state back. A call
// moves at most a few tens of MB, so the kernel is latency bound: each warp
// issues the loads of a whole group of tokens before it starts computing.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

constexpr int kChunkGroup = 8;

template <class E>
__global__ void __launch_bounds__(32) wkv4_chunk_kernel(int C, int ncb, const float* __restrict__ w,
                                                        const float* __restrict__ u, const E* __restrict__ k,
                                                        const E* __restrict__ v, E* __restrict__ y,
                                                        int64_t n_tokens, const int32_t* __restrict__ cu,
                                                        float* __restrict__ state, unsigned* err) {
  const int lane = threadIdx.x;
  const int cb = blockIdx.x % ncb;
  const int s = blockIdx.x / ncb;
  const int c = cb * 32 + lane;
  const int64_t beg = cu[s];
  const int64_t end = cu[s + 1];
  if (end == beg) return;  // empty slot: skipped, state untouched
  if (end < beg || beg < 0 || end > n_tokens) {
    if (lane == 0 && cb == 0) record_error(err, WKV_DEVERR_BAD_SLOT);
    return;
  }
  if (c >= C) return;

  float* sp = state + (int64_t)s * 5 * C + c;
  Wkv4State st = {sp[0], sp[C], sp[2 * (int64_t)C], sp[3 * (int64_t)C]};
  // a slot that has absorbed nothing yet takes its reference from this call's first token
  const float ref = st.base == kEmptyPP ? wkv4_ref(Elem<E>::to_f32(k[beg * C + c])) : sp[4 * (int64_t)C];
  const float w2 = __fmul_rn(w[c], kLog2e);
  const float u2 = __fmul_rn(u[c], kLog2e);
  const E* kp = k + beg * C + c;
  const E* vp = v + beg * C + c;
  E* yp = y + beg * C + c;
  const int64_t n = end - beg;
  for (int64_t t0 = 0; t0 < n; t0 += kChunkGroup) {
    float kk[kChunkGroup], vv[kChunkGroup];
#pragma unroll
    for (int j = 0; j < kChunkGroup; ++j) {
      if (t0 + j < n) {
        kk[j] = Elem<E>::to_f32(kp[(t0 + j) * C]);
        vv[j] = Elem<E>::to_f32(vp[(t0 + j) * C]);
      }
    }
#pragma unroll
    for (int j = 0; j < kChunkGroup; ++j) {
      if (t0 + j < n) {
        const float k2 = wkv4_key(kk[j], ref);
        const float yv = wkv4_token(st, k2, vv[j], u2, w2);
        yp[(t0 + j) * C] = Elem<E>::from_f32(yv);
      }
    }
  }
  sp[0] = st.aa;
  sp[C] = st.bb;
  sp[2 * (int64_t)C] = st.base;
  sp[3 * (int64_t)C] = st.n;
  sp[4 * (int64_t)C] = ref;
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
  const int ncb = (int)ceil_div(a.C, 32);
  const unsigned grid = (unsigned)(ncb * a.S);
  if (a.dtype == WKV_BF16)
    wkv4_chunk_kernel<__nv_bfloat16><<<grid, 32, 0, stream>>>(
        (int)a.C, ncb, a.w, a.u, static_cast<const __nv_bfloat16*>(a.k), static_cast<const __nv_bfloat16*>(a.v),
        static_cast<__nv_bfloat16*>(a.y), a.n_tokens, a.cu_tokens, a.state, err);
  else
    wkv4_chunk_kernel<float><<<grid, 32, 0, stream>>>((int)a.C, ncb, a.w, a.u, static_cast<const float*>(a.k),
                                                      static_cast<const float*>(a.v), static_cast<float*>(a.y),
                                                      a.n_tokens, a.cu_tokens, a.state, err);
  if (cudaGetLastError() != cudaSuccess) {
    *why = "wkv4_chunk_step kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

}  // namespace wkv
