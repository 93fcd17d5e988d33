// wkv6_fwd.cu -- RWKV-6 head-state WKV forward on sm_100a.
//
// Operator: RWKV6_OP (rwkv-ops package page, section "rwkv6op 使用方法", call
// and argument tables). Per (sample b, head h), key index i, value index j:
//   o_t[j]    = sum_i r_t[i] (S_{t-1}[i][j] + u[i] k_t[i] v_t[j])
//   S_t[i][j] = w_t[i] S_{t-1}[i][j] + k_t[i] v_t[j]
// with S_{-1} = 0 or init_state[state_map[b]] (n_state = 1: shared;
// n_state = B: one per sample).
//
// This kernel walks the tokens in order: one CTA per (b, h), thread j keeps
// column j of the fp32 state (64 registers). Tokens arrive in tiles of
// kTok6 steps staged in shared memory as fp32.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

constexpr int kHead = 64;
constexpr int kTok6 = 32;

__global__ void __launch_bounds__(kHead) wkv6_fwd_seq_kernel(int T, int H, const __nv_bfloat16* __restrict__ r,
                                                            const __nv_bfloat16* __restrict__ k,
                                                            const __nv_bfloat16* __restrict__ v,
                                                            const __nv_bfloat16* __restrict__ w,
                                                            const float* __restrict__ u,
                                                            const float* __restrict__ init_state,
                                                            const int32_t* __restrict__ state_map, int n_state,
                                                            float* __restrict__ final_state,
                                                            __nv_bfloat16* __restrict__ o, unsigned* err) {
  __shared__ __align__(16) float sr[kTok6][kHead];
  __shared__ __align__(16) float sk[kTok6][kHead];
  __shared__ __align__(16) float sw[kTok6][kHead];
  __shared__ __align__(16) float sv[kTok6][kHead];
  __shared__ __align__(16) float su[kHead];

  const int j = threadIdx.x;
  const int h = blockIdx.x % H;
  const int b = blockIdx.x / H;
  const int64_t HK = (int64_t)H * kHead;
  const int64_t base = (int64_t)b * T * HK + (int64_t)h * kHead;

  float S[kHead];
  const float* s0 = nullptr;
  if (init_state) {
    int sidx = state_map ? state_map[b] : (n_state == 1 ? 0 : b);
    if (sidx < 0 || sidx >= n_state) {
      if (j == 0) record_error(err, WKV_DEVERR_BAD_STATE);
    } else {
      s0 = init_state + ((int64_t)sidx * H + h) * kHead * kHead;
    }
  }
#pragma unroll
  for (int i = 0; i < kHead; ++i) S[i] = s0 ? s0[i * kHead + j] : 0.f;
  su[j] = u[h * kHead + j];

  for (int t0 = 0; t0 < T; t0 += kTok6) {
    const int n = min(kTok6, T - t0);
    __syncthreads();
    for (int q = 0; q < n; ++q) {
      const int64_t row = base + (int64_t)(t0 + q) * HK + j;
      sr[q][j] = __bfloat162float(r[row]);
      sk[q][j] = __bfloat162float(k[row]);
      sw[q][j] = __bfloat162float(w[row]);
      sv[q][j] = __bfloat162float(v[row]);
    }
    __syncthreads();
    for (int q = 0; q < n; ++q) {
      const float vj = sv[q][j];
      float acc = 0.f, bonus = 0.f;
#pragma unroll
      for (int i = 0; i < kHead; ++i) {
        acc = fmaf(sr[q][i], S[i], acc);
        bonus = fmaf(sr[q][i] * su[i], sk[q][i], bonus);
      }
      o[base + (int64_t)(t0 + q) * HK + j] = __float2bfloat16_rn(fmaf(bonus, vj, acc));
#pragma unroll
      for (int i = 0; i < kHead; ++i) S[i] = fmaf(sw[q][i], S[i], sk[q][i] * vj);
    }
  }
  if (final_state) {
    float* fs = final_state + ((int64_t)b * H + h) * kHead * kHead;
#pragma unroll
    for (int i = 0; i < kHead; ++i) fs[i * kHead + j] = S[i];
  }
}

wkv_status launch_wkv6_forward(const Wkv6FwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  wkv6_fwd_seq_kernel<<<(unsigned)(a.B * a.H), kHead, 0, stream>>>(
      (int)a.T, (int)a.H, static_cast<const __nv_bfloat16*>(a.r), static_cast<const __nv_bfloat16*>(a.k),
      static_cast<const __nv_bfloat16*>(a.v), static_cast<const __nv_bfloat16*>(a.w), a.u, a.init_state,
      a.state_map, (int)a.n_state, a.final_state, static_cast<__nv_bfloat16*>(a.o), err);
  if (cudaGetLastError() != cudaSuccess) {
    *why = "wkv6_forward kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

}  // namespace wkv
