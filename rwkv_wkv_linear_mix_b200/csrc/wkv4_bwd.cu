// wkv4_bwd.cu -- RWKV-4 WKV backward on sm_100a.
//
// Gradients of L = sum(gy * y) for the WKV of RWKV_TimeMix.forward
// ("代码连连看——RWKV", section RWKV_TimeMix; the parameters time_decay and
// time_first are trained, so the operator needs its backward).
//
// With D_t = b_t + e^{u+k_t}, alpha_t = gy_t / D_t, beta_t = gy_t y_t / D_t:
//   direct terms     gv_t = gy_t rho_t, gk_t = gy_t rho_t (v_t - y_t),
//                    gu  += gy_t rho_t (v_t - y_t),  rho_t = e^{u+k_t} / D_t
//   future terms     A_i = sum_{t>i} alpha_t e^{-(t-1-i) w} (B_i with beta),
//                    gv_i += e^{k_i} A_i, gk_i += e^{k_i} (v_i A_i - B_i)
//   decay gradient   A'_i = sum_{t>i} (t-1-i) alpha_t e^{-(t-1-i) w},
//                    gw -= e^{k_i} (v_i A'_i - B'_i)
// A, B, A', B' follow the reverse recurrences A_{i-1} = alpha_i + e^{-w} A_i,
// A'_{i-1} = e^{-w} (A'_i + A_i). They are carried as mantissas under one
// shared base-2 exponent R (A = Am * 2^R) that is a running max of the term
// exponents -q_t - (t-1-i) w, kept like the forward's exponent as a base and
// an exact step count; then the factor e^{k_i} * 2^R has exponent <= 0
// because q_t >= P_t >= k_i - (t-1-i) w.
//
// Kernel shape. One thread per lane, one warp = 32 channels of one sample.
// Time is walked in reverse, one checkpoint interval (WKV4_CKPT_LEN = 32
// steps) at a time: the warp restarts the forward recurrence from the
// interval's checkpoint, keeps the 32 states in registers, then runs the 32
// reverse steps. k, v and gy of the interval arrive as TMA tiles (in reverse
// interval order) in a ring of STAGES stages. Per-lane gw/gu sums go to a
// [B][C] scratch and are added over the batch in a fixed order afterwards.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

constexpr int kBwdL = WKV4_CKPT_LEN;

template <class E, int STAGES>
struct Wkv4BwdSmem {
  E k[STAGES][kBwdL][32];
  E v[STAGES][kBwdL][32];
  E gy[STAGES][kBwdL][32];
  uint64_t full[STAGES];
};

template <class E, int STAGES>
__global__ void __launch_bounds__(32) wkv4_bwd_kernel(const __grid_constant__ CUtensorMap tk,
                                                      const __grid_constant__ CUtensorMap tv,
                                                      const __grid_constant__ CUtensorMap tg, int T, int C,
                                                      int ncb, const float* __restrict__ w,
                                                      const float* __restrict__ u,
                                                      const E* __restrict__ kraw,
                                                      const float* __restrict__ ckpt, E* __restrict__ gk,
                                                      E* __restrict__ gv, float* __restrict__ part_gw,
                                                      float* __restrict__ part_gu, unsigned* err) {
  __shared__ __align__(128) Wkv4BwdSmem<E, STAGES> sm;
  constexpr uint32_t kStageBytes = 3u * kBwdL * 32u * sizeof(E);

  const int lane = threadIdx.x;
  const int cb = blockIdx.x % ncb;
  const int b = blockIdx.x / ncb;
  const int c0 = cb * 32;
  const int c = c0 + lane;
  const bool valid = c < C;
  const int nck = (T + kBwdL - 1) / kBwdL;

  auto issue = [&](int it, int s) {
    const int t0 = (nck - 1 - it) * kBwdL;
    mbar_arrive_expect_tx(&sm.full[s], kStageBytes);
    tma_load_3d(&sm.k[s][0][0], &tk, &sm.full[s], c0, t0, b);
    tma_load_3d(&sm.v[s][0][0], &tv, &sm.full[s], c0, t0, b);
    tma_load_3d(&sm.gy[s][0][0], &tg, &sm.full[s], c0, t0, b);
  };
  if (lane == 0) {
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    tma_prefetch_desc(&tg);
    for (int s = 0; s < STAGES; ++s) mbar_init(&sm.full[s], 1);
    mbar_init_fence();
    for (int s = 0; s < STAGES && s < nck; ++s) issue(s, s);
  }
  __syncwarp();

  const float w2 = valid ? __fmul_rn(w[c], kLog2e) : 0.f;
  const float u2 = valid ? __fmul_rn(u[c], kLog2e) : 0.f;
  const int64_t lane_off = (int64_t)b * T * C + c;
  // lane reference exponent: the same value the forward derived from token 0
  const float ref = valid ? wkv4_ref(Elem<E>::to_f32(kraw[lane_off])) : 0.f;
  const float* ckl = ckpt + (int64_t)b * nck * 3 * C + c;

  // reverse carry: A = Am 2^R etc. with R = rbase - rn * w2 (counted decay,
  // as in the forward); R starts at the "empty" exponent
  float rbase = kEmptyPP, rn = 0.f, Am = 0.f, Bm = 0.f, Apm = 0.f, Bpm = 0.f;
  float gw_acc = 0.f, gu_acc = 0.f;

  // checkpoint of the interval processed next (prefetched one interval ahead)
  Wkv4State nxt = {0.f, 0.f, 0.f, 0.f};
  if (valid && nck > 0) {
    const float* p = ckl + (int64_t)(nck - 1) * 3 * C;
    nxt = {p[0], p[C], p[2 * (int64_t)C], 0.f};
  }

  int it = 0;
  for (; it < nck; ++it) {
    const int s = it % STAGES;
    const int j = nck - 1 - it;
    const int t0 = j * kBwdL;
    const int n = min(kBwdL, T - t0);
    Wkv4State st = nxt;
    if (valid && j > 0) {
      const float* p = ckl + (int64_t)(j - 1) * 3 * C;
      nxt = {p[0], p[C], p[2 * (int64_t)C], 0.f};
    }
    const bool ok = mbar_wait_bounded(&sm.full[s], (it / STAGES) & 1, err);
    if (!__all_sync(0xffffffffu, ok)) break;

    if (valid) {
      // forward recompute over the interval: state before each token
      float saa[kBwdL], sbb[kBwdL], spp[kBwdL];
#pragma unroll
      for (int jj = 0; jj < kBwdL; ++jj) {
        if (jj < n) {
          saa[jj] = st.aa;
          sbb[jj] = st.bb;
          spp[jj] = wkv4_exponent(st, w2);
          const float k2 = wkv4_key(Elem<E>::to_f32(sm.k[s][jj][lane]), ref);
          const float vv = Elem<E>::to_f32(sm.v[s][jj][lane]);
          wkv4_absorb(st, k2, vv, w2);
        }
      }
      E* gkl = gk + lane_off + (int64_t)t0 * C;
      E* gvl = gv + lane_off + (int64_t)t0 * C;
      // reverse sweep over the interval
#pragma unroll
      for (int jj = kBwdL - 1; jj >= 0; --jj) {
        if (jj < n) {
          const float k2 = wkv4_key(Elem<E>::to_f32(sm.k[s][jj][lane]), ref);
          const float vv = Elem<E>::to_f32(sm.v[s][jj][lane]);
          const float g = Elem<E>::to_f32(sm.gy[s][jj][lane]);
          // output of token jj: D = 2^q * den
          const float cur = __fadd_rn(u2, k2);
          const float d = __fsub_rn(spp[jj], cur);
          const float e = ex2(-fabsf(d));
          const bool past_max = d >= 0.f;
          const float e1 = past_max ? 1.f : e;
          const float e2 = past_max ? e : 1.f;
          const float q = past_max ? spp[jj] : cur;
          const float num = __fmaf_rn(e1, saa[jj], __fmul_rn(e2, vv));
          const float den = __fmaf_rn(e1, sbb[jj], e2);
          const float rd = rcp(den);
          const float yv = __fmul_rn(num, rd);
          const float alpha = __fmul_rn(g, rd);   // alpha_t * 2^q
          const float beta = __fmul_rn(alpha, yv);  // beta_t * 2^q
          const float gloc = __fmul_rn(alpha, e2);  // gy_t rho_t
          // v - y = e1 (bb v - aa) / den: no cancellation against v when the
          // current token dominates (y within rounding of v)
          const float vmy = __fmul_rn(__fmul_rn(e1, __fmaf_rn(sbb[jj], vv, -saa[jj])), rd);
          float gvv = gloc;
          float gkv = __fmul_rn(gloc, vmy);
          gu_acc = __fadd_rn(gu_acc, gkv);
          // tokens after jj, through the carried sums
          const float f = ex2(__fadd_rn(k2, __fmaf_rn(-rn, w2, rbase)));
          gvv = __fmaf_rn(f, Am, gvv);
          gkv = __fmaf_rn(f, __fmaf_rn(vv, Am, -Bm), gkv);
          gw_acc = __fmaf_rn(-f, __fmaf_rn(vv, Apm, -Bpm), gw_acc);
          gkl[(int64_t)jj * C] = Elem<E>::from_f32(gkv);
          gvl[(int64_t)jj * C] = Elem<E>::from_f32(gvv);
          // fold token jj into the carry (new exponent max(R - w, -q))
          const float rn1 = __fadd_rn(rn, 1.f);
          const float dd = __fmaf_rn(-rn1, w2, __fadd_rn(rbase, q));  // (R - w) - (-q)
          const float ef = ex2(-fabsf(dd));
          const bool keep = dd >= 0.f;
          const float fo = keep ? 1.f : ef;
          const float fn = keep ? ef : 1.f;
          Apm = __fmul_rn(fo, __fadd_rn(Apm, Am));
          Bpm = __fmul_rn(fo, __fadd_rn(Bpm, Bm));
          Am = __fmaf_rn(fo, Am, __fmul_rn(fn, alpha));
          Bm = __fmaf_rn(fo, Bm, __fmul_rn(fn, beta));
          rbase = keep ? rbase : -q;
          rn = keep ? rn1 : 0.f;
        }
      }
    }
    __syncwarp();
    if (lane == 0 && it + STAGES < nck) issue(it + STAGES, s);
  }
  if (it < nck) {
    if (lane == 0)
      for (int jt = it; jt < nck && jt < it + STAGES; ++jt)
        mbar_wait_bounded(&sm.full[jt % STAGES], (jt / STAGES) & 1, err);
    return;
  }
  if (valid) {
    part_gw[(int64_t)b * C + c] = gw_acc;
    part_gu[(int64_t)b * C + c] = gu_acc;
  }
}

// gw[c] = sum_b part_gw[b][c] (b ascending), same for gu.
__global__ void wkv4_reduce_kernel(const float* __restrict__ part_gw, const float* __restrict__ part_gu, int B,
                                   int C, float* __restrict__ gw, float* __restrict__ gu) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= C) return;
  float sw = 0.f, su = 0.f;
  for (int b = 0; b < B; ++b) {
    sw += part_gw[(int64_t)b * C + c];
    su += part_gu[(int64_t)b * C + c];
  }
  gw[c] = sw;
  gu[c] = su;
}

template <class E, int STAGES>
static wkv_status run_bwd(const Wkv4BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  CUtensorMap tk, tv, tg;
  const CUtensorMapDataType ty = Elem<E>::tma_type;
  if (!encode_tmap_3d(&tk, a.k, ty, sizeof(E), a.C, a.T, a.B, 32, kBwdL, 1, why) ||
      !encode_tmap_3d(&tv, a.v, ty, sizeof(E), a.C, a.T, a.B, 32, kBwdL, 1, why) ||
      !encode_tmap_3d(&tg, a.gy, ty, sizeof(E), a.C, a.T, a.B, 32, kBwdL, 1, why))
    return WKV_ERR_INVALID_ARG;
  const int ncb = (int)ceil_div(a.C, 32);
  float* part_gw = a.part;
  float* part_gu = a.part + a.B * a.C;
  wkv4_bwd_kernel<E, STAGES><<<(unsigned)(ncb * a.B), 32, 0, stream>>>(
      tk, tv, tg, (int)a.T, (int)a.C, ncb, a.w, a.u, static_cast<const E*>(a.k), a.ckpt,
      static_cast<E*>(a.gk), static_cast<E*>(a.gv),
      part_gw, part_gu, err);
  wkv4_reduce_kernel<<<(unsigned)ceil_div(a.C, 256), 256, 0, stream>>>(part_gw, part_gu, (int)a.B, (int)a.C,
                                                                       a.gw, a.gu);
  if (cudaGetLastError() != cudaSuccess) {
    *why = "wkv4_backward kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

wkv_status launch_wkv4_backward(const Wkv4BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  if (a.dtype == WKV_BF16) return run_bwd<__nv_bfloat16, 2>(a, stream, err, why);
  return run_bwd<float, 2>(a, stream, err, why);
}

}  // namespace wkv
