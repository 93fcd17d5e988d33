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
// A'_{i-1} = e^{-w} (A'_i + A_i). They are carried normalised by the
// forward's own exponent after token i: A~_i = A_i 2^{P_{i+1}} (P the
// base-2 exponent of the running-max state, P_{i+1} = max(P_i - w, k_i)).
// Then every coefficient of the reverse scan is a factor the forward step
// already forms, all <= 1 (base 2, w and k pre-scaled by log2 e):
//   absorb of token i   f1_i = 2^{P_i - w - P_{i+1}}, f2_i = 2^{k_i - P_{i+1}}
//   output of token i   e_i = 2^{u + k_i - P_i} (capped at 2^64 as in the
//                       forward), D_i = 2^{P_i} (bb_i + e_i)
// (one of f1/f2 is exactly 1), and walking i downwards
//   gv_i += f2_i A~_i,   gk_i += f2_i (v_i A~_i - B~_i),
//   gw   -= f2_i (v_i A~'_i - B~'_i),
//   A~'_{i-1} = f1_i (A~'_i + A~_i),  A~_{i-1} = f1_i A~_i + gy_i / (bb_i + e_i)
// (B~ the same with gy_i y_i). The carries stay bounded by sum |gy| and need
// no exponent of their own; the loop-carried dependence is one multiply-add.
//
// Kernel shape. One warp = 32 channels of one sample; time is walked in
// reverse one checkpoint interval (WKV4_CKPT_LEN = 16 steps) at a time: the
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

template <bool V>
struct BoolTag {
  static constexpr bool value = V;
};

template <class E, int STAGES>
struct alignas(128) Wkv4BwdSmem {
  E k[STAGES][kBwdL][32];
  E v[STAGES][kBwdL][32];
  E gy[STAGES][kBwdL][32];
  uint64_t full[STAGES];
  float carry[5][32];  // this segment's local carry A, B, A', B' and its product of f1
};

// Carried future sums of one lane, normalised by 2^{P} of the forward state
// at the point they refer to (see above).
struct Wkv4Carry {
  float A, B, Ap, Bp;
};

// One checkpoint interval in reverse. FULL: also produce gk, gv, gw, gu;
// otherwise only fold the interval into the carry.
// fprod (fold-only pass) accumulates the product of the f1 factors. WHOLE
// (n == kBwdL): the reverse steps are not predicated, so the compiler can
// overlap the independent parts of consecutive steps; the recompute loop
// always is (unpredicated, both loops together need too many registers).
template <bool FULL, bool WHOLE, class E>
__device__ __forceinline__ void wkv4_bwd_interval(const E (*ks)[32], const E (*vs)[32], const E (*gs)[32], int lane,
                                                  int n, Wkv4State st, float ref, float u2, float w2, Wkv4Carry& cr,
                                                  float& fprod, float& gw_acc, float& gu_acc, E* gkl, E* gvl,
                                                  int C) {
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
  float A = cr.A, B = cr.B, Ap = cr.Ap, Bp = cr.Bp;
#pragma unroll
  for (int jj = kBwdL - 1; jj >= 0; --jj) {
    if (WHOLE || jj < n) {
      const float k2 = wkv4_key(Elem<E>::to_f32(ks[jj][lane]), ref);
      const float vv = Elem<E>::to_f32(vs[jj][lane]);
      const float g = Elem<E>::to_f32(gs[jj][lane]);
      const float P = spp[jj];
      // output of token jj, in units of the past's exponent P: weight
      // e = 2^{u + k - P} of the current token (capped as in the forward),
      // D = 2^P (bb + e), y = (aa + e v) / (bb + e)
      const float e = ex2(fminf(__fsub_rn(__fadd_rn(u2, k2), P), 64.f));
      const float rd = rcp(__fadd_rn(sbb[jj], e));
      const float yv = __fmul_rn(__fmaf_rn(e, vv, saa[jj]), rd);
      // absorb pair of token jj: P' = max(P - w, k)
      const float z = __fsub_rn(k2, __fsub_rn(P, w2));
      const float ea = ex2(-fabsf(z));
      const bool keep = z <= 0.f;
      const float f1 = keep ? 1.f : ea;
      const float f2 = keep ? ea : 1.f;
      const float ag = __fmul_rn(g, rd);  // gy 2^P / D
      if constexpr (FULL) {
        const float rg = __fmul_rn(ag, e);  // gy rho, rho = e^{u+k} / D
        // v - y = (bb v - aa) / (bb + e): no cancellation against v when the
        // current token dominates (y within rounding of v)
        const float vmy = __fmul_rn(__fmaf_rn(sbb[jj], vv, -saa[jj]), rd);
        const float gvv = __fmaf_rn(f2, A, rg);
        const float gkv = __fmaf_rn(rg, vmy, __fmul_rn(f2, __fmaf_rn(vv, A, -B)));
        gu_acc = __fmaf_rn(rg, vmy, gu_acc);
        gw_acc = __fmaf_rn(-f2, __fmaf_rn(vv, Ap, -Bp), gw_acc);
        gkl[(int64_t)jj * C] = Elem<E>::from_f32(gkv);
        gvl[(int64_t)jj * C] = Elem<E>::from_f32(gvv);
      }
      if constexpr (!FULL) fprod = __fmul_rn(fprod, f1);
      // carries for token jj - 1
      Ap = __fmul_rn(f1, __fadd_rn(Ap, A));
      Bp = __fmul_rn(f1, __fadd_rn(Bp, B));
      A = __fmaf_rn(f1, A, ag);
      B = __fmaf_rn(f1, B, __fmul_rn(ag, yv));
    }
  }
  cr = {A, B, Ap, Bp};
}

template <class E, int STAGES, int NSEG, int NW>
__global__ void __launch_bounds__(32 * NW, NSEG == 1 ? 16 : 1) wkv4_bwd_kernel(const __grid_constant__ CUtensorMap tk,
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

  // reverse carries (normalised by the forward exponent, see above)
  Wkv4Carry cr = {0.f, 0.f, 0.f, 0.f};
  float gw_acc = 0.f, gu_acc = 0.f;
  auto run_interval = [&](auto full_tag, int s, int i, const Wkv4State& st, float& fprod) {
    constexpr bool kFull = decltype(full_tag)::value;
    const int n = min(kBwdL, T - i * kBwdL);
    const int64_t off = lane_off + (int64_t)i * kBwdL * C;
    E* gkp = kFull ? gk + off : nullptr;
    E* gvp = kFull ? gv + off : nullptr;
    // unpredicated steps for whole bf16 intervals (float32 would spill)
    if (sizeof(E) == 2 && n == kBwdL)
      wkv4_bwd_interval<kFull, sizeof(E) == 2, E>(sm.k[s], sm.v[s], sm.gy[s], lane, n, st, ref, u2, w2, cr, fprod, gw_acc,
                                        gu_acc, gkp, gvp, C);
    else
      wkv4_bwd_interval<kFull, false, E>(sm.k[s], sm.v[s], sm.gy[s], lane, n, st, ref, u2, w2, cr, fprod, gw_acc,
                                         gu_acc, gkp, gvp, C);
  };

  if constexpr (NSEG > 1) {
    // ---- phase 1: this segment's own carry, from an empty future ----
    float fprod = 1.f;
    Wkv4State nxt = nloc > 0 ? load_ckpt(interval(0)) : Wkv4State{0.f, 0.f, 0.f, 0.f};
    for (; ok && qq < nloc; ++qq) {
      const int i = interval(qq);
      const Wkv4State st = nxt;
      if (qq + 1 < nloc) nxt = load_ckpt(interval(qq + 1));
      if (!acquire(qq)) break;
      if (valid) run_interval(BoolTag<false>{}, qq % STAGES, i, st, fprod);
      release(qq);
    }
    sm.carry[0][lane] = cr.A;
    sm.carry[1][lane] = cr.B;
    sm.carry[2][lane] = cr.Ap;
    sm.carry[3][lane] = cr.Bp;
    sm.carry[4][lane] = fprod;
    cluster_arrive_release();
    cluster_wait_acquire();
    // ---- phase 2: the exact carry entering this segment from the later ones ----
    Wkv4Carry in = {0.f, 0.f, 0.f, 0.f};
    for (int r = NSEG - 1; r > seg; --r) {
      const int len = min(T, wkv4_seg_begin(r + 1, NSEG, nck) * kBwdL) - wkv4_seg_begin(r, NSEG, nck) * kBwdL;
      const float f = ld_shared_cluster(map_shared_rank(&sm.carry[4][lane], r));
      const float m = (float)len;
      in = {__fmaf_rn(f, in.A, ld_shared_cluster(map_shared_rank(&sm.carry[0][lane], r))),
            __fmaf_rn(f, in.B, ld_shared_cluster(map_shared_rank(&sm.carry[1][lane], r))),
            __fmaf_rn(f, __fmaf_rn(m, in.A, in.Ap), ld_shared_cluster(map_shared_rank(&sm.carry[2][lane], r))),
            __fmaf_rn(f, __fmaf_rn(m, in.B, in.Bp), ld_shared_cluster(map_shared_rank(&sm.carry[3][lane], r)))};
    }
    cluster_arrive_release();  // done reading peers; waited for before exit
    cr = in;
    gw_acc = 0.f;
    gu_acc = 0.f;
  }

  // ---- last pass: gradients ----
  {
    float unused = 1.f;
    Wkv4State nxt = nloc > 0 ? load_ckpt(interval(0)) : Wkv4State{0.f, 0.f, 0.f, 0.f};
    for (; ok && qq < total; ++qq) {
      const int i = interval(qq);
      const Wkv4State st = nxt;
      if (qq + 1 < total) nxt = load_ckpt(interval(qq + 1));
      if (!acquire(qq)) break;
      if (valid) run_interval(BoolTag<true>{}, qq % STAGES, i, st, unused);
      release(qq);
    }
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

// gw[c] = sum over (b, segment) of the partials; same for gu. A block of
// 8 warps takes 32 channels: warp q adds rows q, q + 8, q + 16, ... in
// ascending order, then warp 0 adds the 8 warp sums in order 0..7, so the
// result does not depend on timing.
constexpr int kReduceWarps = 8;
__global__ void __launch_bounds__(32 * kReduceWarps) wkv4_reduce_kernel(const float* __restrict__ part_gw,
                                                                       const float* __restrict__ part_gu, int rows,
                                                                       int C, float* __restrict__ gw,
                                                                       float* __restrict__ gu) {
  __shared__ float sw[kReduceWarps][32], su[kReduceWarps][32];
  const int lane = threadIdx.x % 32, q = threadIdx.x / 32;
  const int c = blockIdx.x * 32 + lane;
  float aw = 0.f, au = 0.f;
  if (c < C) {
    for (int r = q; r < rows; r += kReduceWarps) {
      aw += part_gw[(int64_t)r * C + c];
      au += part_gu[(int64_t)r * C + c];
    }
  }
  sw[q][lane] = aw;
  su[q][lane] = au;
  __syncthreads();
  if (q == 0 && c < C) {
    float tw = 0.f, tu = 0.f;
#pragma unroll
    for (int i = 0; i < kReduceWarps; ++i) {
      tw += sw[i][lane];
      tu += su[i][lane];
    }
    gw[c] = tw;
    gu[c] = tu;
  }
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
    // clusters above 8 CTAs are a non-portable size that must be opted into
    if (NSEG > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
      *why = "non-portable cluster size refused";
      return WKV_ERR_CUDA;
    }
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
    wkv4_reduce_kernel<<<(unsigned)ceil_div(a.C, 32), 32 * kReduceWarps, 0, stream>>>(part_gw, part_gu, (int)rows,
                                                                                     (int)a.C, a.gw, a.gu);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    *why = "wkv4_backward kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

// Stages of the k/v/gy ring (one checkpoint interval each): four for bf16
// (3 KB a stage), two for float32 (6 KB), so that the 14-16 one-warp CTAs an
// SM holds still fit in shared memory.
template <class E, int STAGES, int NSEG>
static wkv_status run_bwd_nw(const Wkv4BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  switch (wkv4_warps_per_cta(a.B, a.C, NSEG)) {
    case 4: return run_bwd<E, STAGES, NSEG, 4>(a, stream, err, why);
    case 2: return run_bwd<E, STAGES, NSEG, 2>(a, stream, err, why);
    default: return run_bwd<E, STAGES, NSEG, 1>(a, stream, err, why);
  }
}

template <class E>
static wkv_status run_bwd_nseg(const Wkv4BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  constexpr int kStages = sizeof(E) == 2 ? 4 : 2;
  switch (wkv4_bwd_segments(a.B, a.T, a.C)) {
#if WKV4_MAX_SEGMENTS_ANY > 8
    case 16: return run_bwd_nw<E, kStages, 16>(a, stream, err, why);
#endif
    case 8: return run_bwd_nw<E, kStages, 8>(a, stream, err, why);
    case 4: return run_bwd_nw<E, kStages, 4>(a, stream, err, why);
    case 2: return run_bwd_nw<E, kStages, 2>(a, stream, err, why);
    default: return run_bwd<E, kStages, 1, 1>(a, stream, err, why);
  }
}

wkv_status launch_wkv4_backward(const Wkv4BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  if (a.dtype == WKV_BF16) return run_bwd_nseg<__nv_bfloat16>(a, stream, err, why);
  return run_bwd_nseg<float>(a, stream, err, why);
}

}  // namespace wkv
