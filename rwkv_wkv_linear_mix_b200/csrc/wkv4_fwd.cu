// wkv4_fwd.cu -- RWKV-4 WKV forward on sm_100a.
//
// Operator: the WKV of RWKV_TimeMix.forward, RUN_CUDA(B, T, C, time_decay,
// time_first, k, v) ("代码连连看——RWKV", section RWKV_TimeMix), evaluated as the
// running-max recurrence of wkv_device.cuh.
//
// Design. The recurrence is sequential in t and independent per lane (b, c),
// so one thread owns one lane and keeps its state in registers for the
// whole sequence. A CTA is one warp = 32 consecutive channels of one sample.
// The warp streams its [T x 32] slices of k and v through a ring of STAGES
// shared-memory tiles of LT time steps, filled by 3-D TMA loads (box
// {32 ch, LT steps, 1 sample}; rows past T are zero-filled and ignored) that
// complete on per-stage mbarriers. Lane 0 refills a stage as soon as the warp
// has consumed it, so STAGES-1 tiles are always in flight per warp. y is
// written straight from registers (one 64/128-byte row segment per warp and
// step). Every WKV4_CKPT_LEN steps the state is written to the checkpoint
// buffer that the backward pass restarts from; its exponent P is relative to the
// lane reference fl(k[b][0][c] * log2e), which the backward recomputes.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

template <class E, int LT, int STAGES>
struct Wkv4FwdSmem {
  E k[STAGES][LT][32];
  E v[STAGES][LT][32];
  uint64_t full[STAGES];
};

template <class E, int LT, int STAGES>
__global__ void __launch_bounds__(32) wkv4_fwd_kernel(const __grid_constant__ CUtensorMap tk,
                                                      const __grid_constant__ CUtensorMap tv, int T, int C,
                                                      int ncb, const float* __restrict__ w,
                                                      const float* __restrict__ u, E* __restrict__ y,
                                                      float* __restrict__ ckpt, unsigned* err) {
  static_assert(WKV4_CKPT_LEN % LT == 0, "checkpoint interval must be a whole number of tiles");
  __shared__ __align__(128) Wkv4FwdSmem<E, LT, STAGES> sm;
  constexpr uint32_t kStageBytes = 2u * LT * 32u * sizeof(E);

  const int lane = threadIdx.x;
  const int cb = blockIdx.x % ncb;
  const int b = blockIdx.x / ncb;
  const int c0 = cb * 32;
  const int c = c0 + lane;
  const bool valid = c < C;
  const int nchunk = (T + LT - 1) / LT;

  if (lane == 0) {
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    for (int s = 0; s < STAGES; ++s) mbar_init(&sm.full[s], 1);
    mbar_init_fence();
    for (int s = 0; s < STAGES && s < nchunk; ++s) {
      mbar_arrive_expect_tx(&sm.full[s], kStageBytes);
      tma_load_3d(&sm.k[s][0][0], &tk, &sm.full[s], c0, s * LT, b);
      tma_load_3d(&sm.v[s][0][0], &tv, &sm.full[s], c0, s * LT, b);
    }
  }
  __syncwarp();

  const float w2 = valid ? __fmul_rn(w[c], kLog2e) : 0.f;
  const float u2 = valid ? __fmul_rn(u[c], kLog2e) : 0.f;
  Wkv4State st = wkv4_empty_state();
  float ref = 0.f;  // set from the lane's first key once the first tile lands
  E* yl = y ? y + (int64_t)b * T * C + c : nullptr;
  const int64_t nck = (T + WKV4_CKPT_LEN - 1) / WKV4_CKPT_LEN;
  float* ckl = ckpt ? ckpt + (int64_t)b * nck * 3 * C + c : nullptr;

  int i = 0;
  for (; i < nchunk; ++i) {
    const int s = i % STAGES;
    const int t0 = i * LT;
    if (ckl && valid && (t0 % WKV4_CKPT_LEN) == 0) {
      float* p = ckl + (int64_t)(t0 / WKV4_CKPT_LEN) * 3 * C;
      p[0] = st.aa;
      p[C] = st.bb;
      p[2 * (int64_t)C] = wkv4_exponent(st, w2);
    }
    const bool ok = mbar_wait_bounded(&sm.full[s], (i / STAGES) & 1, err);
    if (!__all_sync(0xffffffffu, ok)) break;
    if (i == 0) ref = wkv4_ref(Elem<E>::to_f32(sm.k[0][0][lane]));
    const int n = min(LT, T - t0);
    if (valid) {
      E* yt = yl ? yl + (int64_t)t0 * C : nullptr;
      if (n == LT) {
#pragma unroll 8
        for (int j = 0; j < LT; ++j) {
          const float k2 = wkv4_key(Elem<E>::to_f32(sm.k[s][j][lane]), ref);
          const float vv = Elem<E>::to_f32(sm.v[s][j][lane]);
          const float yv = wkv4_token(st, k2, vv, u2, w2);
          if (yt) yt[(int64_t)j * C] = Elem<E>::from_f32(yv);
        }
      } else {
        for (int j = 0; j < n; ++j) {
          const float k2 = wkv4_key(Elem<E>::to_f32(sm.k[s][j][lane]), ref);
          const float vv = Elem<E>::to_f32(sm.v[s][j][lane]);
          const float yv = wkv4_token(st, k2, vv, u2, w2);
          if (yt) yt[(int64_t)j * C] = Elem<E>::from_f32(yv);
        }
      }
    }
    __syncwarp();
    if (lane == 0 && i + STAGES < nchunk) {
      const int tn = (i + STAGES) * LT;
      mbar_arrive_expect_tx(&sm.full[s], kStageBytes);
      tma_load_3d(&sm.k[s][0][0], &tk, &sm.full[s], c0, tn, b);
      tma_load_3d(&sm.v[s][0][0], &tv, &sm.full[s], c0, tn, b);
    }
  }
  if (i < nchunk && lane == 0) {
    // A wait gave up: let the copies still in flight land before the CTA's
    // shared memory is released (each wait is itself bounded).
    for (int j = i; j < nchunk && j < i + STAGES; ++j) mbar_wait_bounded(&sm.full[j % STAGES], (j / STAGES) & 1, err);
  }
}

template <class E, int LT, int STAGES>
static wkv_status run_fwd(const Wkv4FwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  CUtensorMap tk, tv;
  const CUtensorMapDataType ty = Elem<E>::tma_type;
  if (!encode_tmap_3d(&tk, a.k, ty, sizeof(E), a.C, a.T, a.B, 32, LT, 1, why) ||
      !encode_tmap_3d(&tv, a.v, ty, sizeof(E), a.C, a.T, a.B, 32, LT, 1, why))
    return WKV_ERR_INVALID_ARG;
  const int ncb = (int)ceil_div(a.C, 32);
  const dim3 grid((unsigned)(ncb * a.B));
  wkv4_fwd_kernel<E, LT, STAGES><<<grid, 32, 0, stream>>>(tk, tv, (int)a.T, (int)a.C, ncb, a.w, a.u,
                                                          static_cast<E*>(a.y), a.ckpt, err);
  if (cudaGetLastError() != cudaSuccess) {
    *why = "wkv4_forward kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

wkv_status launch_wkv4_forward(const Wkv4FwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  if (a.dtype == WKV_BF16) return run_fwd<__nv_bfloat16, 32, 3>(a, stream, err, why);
  return run_fwd<float, 16, 3>(a, stream, err, why);
}

}  // namespace wkv
