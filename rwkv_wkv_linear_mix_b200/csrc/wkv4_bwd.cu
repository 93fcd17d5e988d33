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
// Kernel shape. One warp = 32 channels of one sample; time is walked in
// reverse one checkpoint interval (WKV4_CKPT_LEN = 32 steps) at a time: the
// warp restarts the forward recurrence from the interval's checkpoint, keeps
// the 32 states in registers, then runs the 32 reverse steps. k, v, gy of an
// interval arrive as one TMA stage of a ring. When lanes are few, each lane's
// sequence is split into NSEG segments handled by the NSEG one-warp CTAs of a
// cluster: (1) each CTA folds its segment into a local carry starting from an
// empty future; (2) after a cluster barrier CTA r combines the local carries
// of the CTAs after it (each shifted across the segments before it) read
// through distributed shared memory; (3) each CTA reruns its segment with the
// exact incoming carry and writes gk, gv. Per-(sample, segment, channel) gw/gu
// sums go to scratch and are added in a fixed order by a second kernel.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

constexpr int kBwdL = WKV4_CKPT_LEN;

template <class E, int STAGES>
struct alignas(128) Wkv4BwdSmem {
  E k[STAGES][kBwdL][32];
  E v[STAGES][kBwdL][32];
  E gy[STAGES][kBwdL][32];
  uint64_t full[STAGES];
  float carry[5][32];  // this segment's local carry: Am, Bm, Apm, Bpm, R
};

// Carried future sums of one lane: mantissas under the exponent R.
struct Wkv4Carry {
  float Am, Bm, Apm, Bpm, R;
};

// Move a carry `m` steps further back in time: A' gains m A, the exponent
// loses m w2 (A'_{i-m} = e^{-m w} (A'_i + m A_i)).
__device__ __forceinline__ Wkv4Carry wkv4_carry_shift(Wkv4Carry c, float m, float w2) {
  c.Apm = __fmaf_rn(m, c.Am, c.Apm);
  c.Bpm = __fmaf_rn(m, c.Bm, c.Bpm);
  c.R = __fmaf_rn(-m, w2, c.R);
  return c;
}

__device__ __forceinline__ Wkv4Carry wkv4_carry_merge(const Wkv4Carry& x, const Wkv4Carry& y) {
  const float d = __fsub_rn(x.R, y.R);
  const float e = ex2(-fabsf(d));
  const bool xm = d >= 0.f;
  const float fx = xm ? 1.f : e;
  const float fy = xm ? e : 1.f;
  return {__fmaf_rn(fx, x.Am, __fmul_rn(fy, y.Am)), __fmaf_rn(fx, x.Bm, __fmul_rn(fy, y.Bm)),
          __fmaf_rn(fx, x.Apm, __fmul_rn(fy, y.Apm)), __fmaf_rn(fx, x.Bpm, __fmul_rn(fy, y.Bpm)),
          xm ? x.R : y.R};
}

// One checkpoint interval in reverse. FULL: also produce gk, gv, gw, gu;
// otherwise only fold the interval into the carry.
template <bool FULL, class E>
__device__ __forceinline__ void wkv4_bwd_interval(const E (*ks)[32], const E (*vs)[32], const E (*gs)[32], int lane,
                                                  int n, Wkv4State st, float ref, float u2, float w2, float& rbase,
                                                  float& rn, float& Am, float& Bm, float& Apm, float& Bpm,
                                                  float& gw_acc, float& gu_acc, E* gkl, E* gvl, int C) {
  // forward recompute over the interval: state before each token
  float saa[kBwdL], sbb[kBwdL], spp[kBwdL];
#pragma unroll
  for (int jj = 0; jj < kBwdL; ++jj) {
    if (jj < n) {
      saa[jj] = st.aa;
      sbb[jj] = st.bb;
      spp[jj] = wkv4_exponent(st, w2);
      wkv4_absorb(st, wkv4_key(Elem<E>::to_f32(ks[jj][lane]), ref), Elem<E>::to_f32(vs[jj][lane]), w2);
    }
  }
#pragma unroll
  for (int jj = kBwdL - 1; jj >= 0; --jj) {
    if (jj < n) {
      const float k2 = wkv4_key(Elem<E>::to_f32(ks[jj][lane]), ref);
      const float vv = Elem<E>::to_f32(vs[jj][lane]);
      const float g = Elem<E>::to_f32(gs[jj][lane]);
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
      const float alpha = __fmul_rn(g, rd);     // alpha_t * 2^q
      const float beta = __fmul_rn(alpha, yv);  // beta_t * 2^q
      if constexpr (FULL) {
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
      }
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

template <class E, int STAGES, int NSEG, int NW>
__global__ void __launch_bounds__(32 * NW) wkv4_bwd_kernel(const __grid_constant__ CUtensorMap tk,
                                                           const __grid_constant__ CUtensorMap tv,
                                                           const __grid_constant__ CUtensorMap tg, int T, int C,
                                                           int ncb, int ngroups, const float* __restrict__ w,
                                                           const float* __restrict__ u, const E* __restrict__ kraw,
                                                           const float* __restrict__ ckpt, E* __restrict__ gk,
                                                           E* __restrict__ gv, float* __restrict__ part_gw,
                                                           float* __restrict__ part_gu, unsigned* err) {
  extern __shared__ __align__(128) unsigned char wkv4_bwd_dsmem[];
  // each warp is an independent lane group with its own ring and barriers
  Wkv4BwdSmem<E, STAGES>& sm = reinterpret_cast<Wkv4BwdSmem<E, STAGES>*>(wkv4_bwd_dsmem)[threadIdx.x / 32];
  constexpr uint32_t kStageBytes = 3u * kBwdL * 32u * sizeof(E);
  constexpr int kPasses = NSEG > 1 ? 2 : 1;

  const int lane = threadIdx.x % 32;
  const int seg = NSEG > 1 ? (int)(blockIdx.x % NSEG) : 0;  // == cluster rank
  const int group = (blockIdx.x / NSEG) * NW + threadIdx.x / 32;
  const bool active = group < ngroups;  // a warp past the last group only joins the cluster barriers
  const int cb = group % ncb;
  const int b = group / ncb;
  const int c0 = cb * 32;
  const int c = c0 + lane;
  const bool valid = active && c < C;
  const int nck = (T + kBwdL - 1) / kBwdL;
  const int i_beg = wkv4_seg_begin(seg, NSEG, nck);
  const int i_end = wkv4_seg_begin(seg + 1, NSEG, nck);
  const int nloc = active ? i_end - i_beg : 0;  // intervals of this segment, walked last to first
  const int total = kPasses * nloc;
  auto interval = [&](int qq) { return i_end - 1 - (qq % nloc); };

  auto issue = [&](int qq) {
    const int s = qq % STAGES;
    const int t0 = interval(qq) * kBwdL;
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
    for (int qq = 0; qq < STAGES && qq < total; ++qq) issue(qq);
  }
  __syncwarp();

  const float w2 = valid ? __fmul_rn(w[c], kLog2e) : 0.f;
  const float u2 = valid ? __fmul_rn(u[c], kLog2e) : 0.f;
  const int64_t lane_off = valid ? (int64_t)b * T * C + c : 0;
  // lane reference exponent: the same value the forward derived from token 0
  const float ref = valid ? wkv4_ref(Elem<E>::to_f32(kraw[lane_off])) : 0.f;
  const float* ckl = ckpt + (valid ? (int64_t)b * nck * 3 * C + c : 0);
  auto load_ckpt = [&](int i) -> Wkv4State {
    if (!valid) return {0.f, 0.f, 0.f, 0.f};
    const float* p = ckl + (int64_t)i * 3 * C;
    return {p[0], p[C], p[2 * (int64_t)C], 0.f};
  };

  int qq = 0;
  bool ok = true;
  auto acquire = [&](int x) {
    const bool got = mbar_wait_bounded(&sm.full[x % STAGES], (x / STAGES) & 1, err);
    ok = __all_sync(0xffffffffu, got);
    return ok;
  };
  auto release = [&](int x) {
    __syncwarp();
    if (lane == 0 && x + STAGES < total) issue(x + STAGES);
  };

  // reverse carry: A = Am 2^R etc. with R = rbase - rn * w2 (counted decay,
  // as in the forward); R starts at the "empty" exponent
  float rbase = kEmptyPP, rn = 0.f, Am = 0.f, Bm = 0.f, Apm = 0.f, Bpm = 0.f;
  float gw_acc = 0.f, gu_acc = 0.f;

  if constexpr (NSEG > 1) {
    // ---- phase 1: this segment's own carry, from an empty future ----
    Wkv4State nxt = nloc > 0 ? load_ckpt(interval(0)) : Wkv4State{0.f, 0.f, 0.f, 0.f};
    for (; ok && qq < nloc; ++qq) {
      const int i = interval(qq);
      const Wkv4State st = nxt;
      if (qq + 1 < nloc) nxt = load_ckpt(interval(qq + 1));
      if (!acquire(qq)) break;
      const int s = qq % STAGES;
      if (valid)
        wkv4_bwd_interval<false, E>(sm.k[s], sm.v[s], sm.gy[s], lane, min(kBwdL, T - i * kBwdL), st, ref, u2, w2,
                                    rbase, rn, Am, Bm, Apm, Bpm, gw_acc, gu_acc, nullptr, nullptr, C);
      release(qq);
    }
    sm.carry[0][lane] = Am;
    sm.carry[1][lane] = Bm;
    sm.carry[2][lane] = Apm;
    sm.carry[3][lane] = Bpm;
    sm.carry[4][lane] = __fmaf_rn(-rn, w2, rbase);
    cluster_arrive_release();
    cluster_wait_acquire();
    // ---- phase 2: the exact carry entering this segment from the later ones ----
    Wkv4Carry in = {0.f, 0.f, 0.f, 0.f, kEmptyPP};
    for (int r = NSEG - 1; r > seg; --r) {
      const int len = min(T, wkv4_seg_begin(r + 1, NSEG, nck) * kBwdL) - wkv4_seg_begin(r, NSEG, nck) * kBwdL;
      const Wkv4Carry own = {ld_shared_cluster(map_shared_rank(&sm.carry[0][lane], r)),
                             ld_shared_cluster(map_shared_rank(&sm.carry[1][lane], r)),
                             ld_shared_cluster(map_shared_rank(&sm.carry[2][lane], r)),
                             ld_shared_cluster(map_shared_rank(&sm.carry[3][lane], r)),
                             ld_shared_cluster(map_shared_rank(&sm.carry[4][lane], r))};
      in = wkv4_carry_merge(own, wkv4_carry_shift(in, (float)len, w2));
    }
    cluster_arrive_release();  // done reading peers; waited for before exit
    Am = in.Am;
    Bm = in.Bm;
    Apm = in.Apm;
    Bpm = in.Bpm;
    rbase = in.R;
    rn = 0.f;
  }

  // ---- last pass: gradients ----
  Wkv4State nxt = nloc > 0 ? load_ckpt(interval(0)) : Wkv4State{0.f, 0.f, 0.f, 0.f};
  for (; ok && qq < total; ++qq) {
    const int i = interval(qq);
    const Wkv4State st = nxt;
    if (qq + 1 < total) nxt = load_ckpt(interval(qq + 1));
    if (!acquire(qq)) break;
    const int s = qq % STAGES;
    if (valid) {
      const int64_t off = lane_off + (int64_t)i * kBwdL * C;
      wkv4_bwd_interval<true, E>(sm.k[s], sm.v[s], sm.gy[s], lane, min(kBwdL, T - i * kBwdL), st, ref, u2, w2, rbase,
                                 rn, Am, Bm, Apm, Bpm, gw_acc, gu_acc, gk + off, gv + off, C);
    }
    release(qq);
  }
  if (!ok) {
    if (lane == 0)
      for (int x = qq; x < total && x < qq + STAGES; ++x) mbar_wait_bounded(&sm.full[x % STAGES], (x / STAGES) & 1, err);
  } else if (valid) {
    const int64_t pi = ((int64_t)b * NSEG + seg) * C + c;
    part_gw[pi] = gw_acc;
    part_gu[pi] = gu_acc;
  }
  if constexpr (NSEG > 1) cluster_wait_acquire();  // peers may still read this CTA's carry
}

// gw[c] = sum over (b, segment) of the partials, in ascending order; same for gu.
__global__ void wkv4_reduce_kernel(const float* __restrict__ part_gw, const float* __restrict__ part_gu, int rows,
                                   int C, float* __restrict__ gw, float* __restrict__ gu) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= C) return;
  float sw = 0.f, su = 0.f;
  for (int r = 0; r < rows; ++r) {
    sw += part_gw[(int64_t)r * C + c];
    su += part_gu[(int64_t)r * C + c];
  }
  gw[c] = sw;
  gu[c] = su;
}

template <class E, int STAGES, int NSEG, int NW>
static wkv_status run_bwd(const Wkv4BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  CUtensorMap tk, tv, tg;
  const CUtensorMapDataType ty = Elem<E>::tma_type;
  if (!encode_tmap_3d(&tk, a.k, ty, sizeof(E), a.C, a.T, a.B, 32, kBwdL, 1, why) ||
      !encode_tmap_3d(&tv, a.v, ty, sizeof(E), a.C, a.T, a.B, 32, kBwdL, 1, why) ||
      !encode_tmap_3d(&tg, a.gy, ty, sizeof(E), a.C, a.T, a.B, 32, kBwdL, 1, why))
    return WKV_ERR_INVALID_ARG;
  const int ncb = (int)ceil_div(a.C, 32);
  const int ngroups = (int)(ncb * a.B);
  const int64_t rows = a.B * NSEG;
  float* part_gw = a.part;
  float* part_gu = a.part + rows * a.C;
  auto kern = wkv4_bwd_kernel<E, STAGES, NSEG, NW>;
  const size_t smem = NW * sizeof(Wkv4BwdSmem<E, STAGES>);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
    *why = "wkv4_backward: shared memory configuration failed";
    return WKV_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(ceil_div(ngroups, NW) * NSEG));
  cfg.blockDim = dim3(32 * NW);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (NSEG > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = NSEG;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tk, tv, tg, (int)a.T, (int)a.C, ncb, ngroups, a.w, a.u,
                                     static_cast<const E*>(a.k), a.ckpt, static_cast<E*>(a.gk), static_cast<E*>(a.gv),
                                     part_gw, part_gu, err);
  if (e == cudaSuccess) {
    wkv4_reduce_kernel<<<(unsigned)ceil_div(a.C, 256), 256, 0, stream>>>(part_gw, part_gu, (int)rows, (int)a.C,
                                                                         a.gw, a.gu);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    *why = "wkv4_backward kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

// Stages of the k/v/gy ring: two for bf16 (12 KB each); for float32 (24 KB
// a stage) one when the sequence is split, so that the ~10 one-warp CTAs an
// SM then holds still fit in shared memory.
template <class E, int STAGES, int NSEG>
static wkv_status run_bwd_nw(const Wkv4BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  switch (wkv4_warps_per_cta(a.B, a.C, NSEG)) {
    case 4: return run_bwd<E, STAGES, NSEG, 4>(a, stream, err, why);
    case 2: return run_bwd<E, STAGES, NSEG, 2>(a, stream, err, why);
    default: return run_bwd<E, STAGES, NSEG, 1>(a, stream, err, why);
  }
}

#ifndef WKV4_BWD_SPLIT_STAGES_F32
#define WKV4_BWD_SPLIT_STAGES_F32 1
#endif
template <class E>
static wkv_status run_bwd_nseg(const Wkv4BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  constexpr int kSplitStages = sizeof(E) == 2 ? 2 : WKV4_BWD_SPLIT_STAGES_F32;
  switch (wkv4_bwd_segments(a.B, a.T, a.C)) {
    case 8: return run_bwd_nw<E, kSplitStages, 8>(a, stream, err, why);
    case 4: return run_bwd_nw<E, kSplitStages, 4>(a, stream, err, why);
    case 2: return run_bwd_nw<E, kSplitStages, 2>(a, stream, err, why);
    default: return run_bwd<E, 2, 1, 1>(a, stream, err, why);
  }
}

wkv_status launch_wkv4_backward(const Wkv4BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  if (a.dtype == WKV_BF16) return run_bwd_nseg<__nv_bfloat16>(a, stream, err, why);
  return run_bwd_nseg<float>(a, stream, err, why);
}

}  // namespace wkv
