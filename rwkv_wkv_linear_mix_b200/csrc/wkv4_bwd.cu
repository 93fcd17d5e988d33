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
// Kernel shape. One warp = 64 channels of one sample, a channel pair per
// lane on the packed fp32 pair instructions; time is walked in reverse one
// checkpoint interval (WKV4_CKPT_LEN = 16 steps) at a time: the warp restarts
// the forward recurrence from the interval's checkpoint, keeps the 16 states
// in registers, then runs the 16 reverse steps. k, v, gy of an
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

// 1: whole intervals take an unpredicated copy of the reverse steps (more
// overlap between steps, more registers).
#ifndef WKV4_BWD_WHOLE
#define WKV4_BWD_WHOLE 1
#endif

constexpr int kBwdL = WKV4_CKPT_LEN;
constexpr int kBwdCh = WKV4_WARP_CH;  // channels of one warp: a pair per lane

// Where the recompute leaves the per-step forward quantities (state aa, bb
// before the step and the absorb exponent z1) for the reverse steps: in
// registers, or (bf16) in shared memory, which frees ~100 registers per
// thread for the unpredicated reverse steps (float32 keeps them in registers:
// its larger stages leave no room for the stash at 7 warps per SM).
// Ring depth of the bf16 kernel next to the 16 KB stash (7 warps per SM).
#ifndef WKV4_BWD_STAGES_STASH
#define WKV4_BWD_STAGES_STASH 2
#endif
#ifndef WKV4_BWD_WHOLE_RECOMPUTE
#define WKV4_BWD_WHOLE_RECOMPUTE 1
#endif
// Tokens whose exponent chain the shared-memory-stash recompute runs ahead of
// their value updates.
#ifndef WKV4_BWD_RECOMP_GROUP
#define WKV4_BWD_RECOMP_GROUP 8
#endif
#ifndef WKV4_BWD_SMEM_STASH_F32
#define WKV4_BWD_SMEM_STASH_F32 0
#endif
#ifndef WKV4_BWD_SMEM_STASH
#define WKV4_BWD_SMEM_STASH 1
#endif
template <class E>
constexpr bool bwd_smem_stash() {
  return WKV4_BWD_SMEM_STASH && (sizeof(E) == 2 || WKV4_BWD_SMEM_STASH_F32);
}
// GATE: the gated kernel's ring carries a fourth tile (r); its stash drops
// v (read again from the ring) so that a warp's shared memory stays the same.
template <bool S, bool GATE>
struct Wkv4Stash {
  float4 ab[kBwdL][32];  // (aa.x, aa.y, bb.x, bb.y) of each step, per lane
  float4 zv[kBwdL][32];  // (z1.x, z1.y, v.x, v.y): v unpacked once
};
template <>
struct Wkv4Stash<true, true> {
  float4 ab[kBwdL][32];
  float2 zv[kBwdL][32];  // z1 only
};
template <bool GATE>
struct Wkv4Stash<false, GATE> {};

template <class E, int STAGES, bool GATE>
struct Wkv4BwdGateRing {
  E r[STAGES][kBwdL][kBwdCh];
};
template <class E, int STAGES>
struct Wkv4BwdGateRing<E, STAGES, false> {};

template <class E, int STAGES, bool GATE>
struct alignas(128) Wkv4BwdSmem {
  E k[STAGES][kBwdL][kBwdCh];
  E v[STAGES][kBwdL][kBwdCh];
  E gy[STAGES][kBwdL][kBwdCh];
  Wkv4BwdGateRing<E, STAGES, GATE> g;
  Wkv4Stash<bwd_smem_stash<E>(), GATE> stash;
  uint64_t full[STAGES];
  float2 carry[5][32];  // this segment's local carry A, B, A', B' and its product of f1
};

// Carried future sums of a lane's channel pair, normalised by 2^{P} of the
// forward state at the point they refer to (see above).
struct Wkv4Carry2 {
  float2 A, B, Ap, Bp;
};

__device__ __forceinline__ float2 neg2(float2 a) { return make_float2(-a.x, -a.y); }

// One reverse step of a lane's channel pair (token t, walking down), from
// the forward quantities of the token: the state (aa, bb) before it, its
// absorb factors f1, f2 (and absorb exponent z, for the exact output form),
// v and gy. The output weight e = 2^{u + k - P} = 2^{z1 + u - w} of the token
// (in units of the past's exponent P; D = 2^P (bb + e), y = (aa + e v) /
// (bb + e)) is formed as in the forward: SCALED from f1, f2 and the channel
// constants E2 = 2^{u - w} (den = f1 (bb + e) = f1 bb + f2 E, so 1/(bb + e) =
// f1 / den and e/(bb + e) = f2 E / den), otherwise from a second ex2 of
// z + uw2, capped as in the forward. FULL: also write gk, gv at gkp, gvp and
// add the token's gw, gu terms (gwn holds -gw); otherwise only fold the token
// into the carries and fprod. GATE: gy is the gradient of the gated output
// sigmoid(r) * y; the step writes dL/dr = gy y s (1 - s) at grp
// (s = sigmoid(r)) and carries gy s on as y's.
template <bool FULL, bool GATE, bool SCALED, class E>
__device__ __forceinline__ void wkv4_bwd_rstep(float2& A, float2& B, float2& Ap, float2& Bp, float2& fprod,
                                               float2& gwn, float2& gu_acc, float2 vv, float2 g, float2 rr,
                                               float2 aa, float2 bb, float2 z, float2 f1, float2 f2, float2 uw2,
                                               float2 E2, E* gkp, E* gvp, E* grp) {
  float2 yv, rd, e, rc, g2, t1, t2;
  if constexpr (SCALED) {
    t1 = mul2(f1, aa);
    t2 = mul2(f1, bb);
    g2 = mul2(f2, E2);
    rc = rcp2(fma2(f1, bb, g2));
    yv = mul2(fma2(g2, vv, t1), rc);
  } else {
    const float2 zo = add2(z, uw2);
    e = make_float2(ex2(fminf(zo.x, 64.f)), ex2(fminf(zo.y, 64.f)));
    rd = rcp2(add2(bb, e));
    yv = mul2(fma2(e, vv, aa), rd);
  }
  if constexpr (GATE) {
    const float2 sg = sigmoid2(rr);
    if constexpr (FULL) st_pair(grp, mul2(mul2(g, yv), mul2(sg, sub2(splat2(1.f), sg))));
    g = mul2(g, sg);
  }
  float2 ag, rg, vmy;  // gy 2^P / D; gy rho with rho = e^{u+k} / D; v - y
  if constexpr (SCALED) {
    const float2 q = mul2(g, rc);
    ag = mul2(q, f1);
    rg = mul2(q, g2);
    // v - y = (bb v - aa) / (bb + e) = (t2 v - t1) / den
    vmy = mul2(fma2(t2, vv, neg2(t1)), rc);
  } else {
    ag = mul2(g, rd);
    rg = mul2(ag, e);
    // v - y = (bb v - aa) / (bb + e): no cancellation against v when the
    // current token dominates (y within rounding of v)
    vmy = mul2(fma2(bb, vv, neg2(aa)), rd);
  }
  if constexpr (FULL) {
    const float2 gvv = fma2(f2, A, rg);
    const float2 gkv = fma2(rg, vmy, mul2(f2, fma2(vv, A, neg2(B))));
    gu_acc = fma2(rg, vmy, gu_acc);
    gwn = fma2(f2, fma2(vv, Ap, neg2(Bp)), gwn);
    st_pair(gkp, gkv);
    st_pair(gvp, gvv);
  }
  if constexpr (!FULL) fprod = mul2(fprod, f1);
  // carries for the token before
  Ap = mul2(f1, add2(Ap, A));
  Bp = mul2(f1, add2(Bp, B));
  A = fma2(f1, A, ag);
  B = fma2(f1, B, mul2(ag, yv));
}

// One checkpoint interval in reverse for a lane's channel pair. FULL: also
// produce gk, gv, gw, gu; otherwise only fold the interval into the carry.
// fprod (fold-only pass) accumulates the product of the f1 factors; gwn
// accumulates -gw. WHOLE (n == kBwdL): the reverse steps are not
// predicated, so the compiler can overlap the independent parts of
// consecutive steps. The recompute runs the exponent chain of the interval's
// tokens first and their value updates after it (the split of
// wkv4_chain2 / wkv4_factors2; the same operations as wkv4_absorb2).
template <bool FULL, bool WHOLE, bool GATE, bool SCALED, class E, bool S>
__device__ __forceinline__ void wkv4_bwd_interval(const E (*ks)[kBwdCh], const E (*vs)[kBwdCh],
                                                  const E (*gs)[kBwdCh], const E (*rs)[kBwdCh],
                                                  Wkv4Stash<S, GATE>& sx, int lane, int n, Wkv4State2 st,
                                                  float2 ref, float2 uw2, float2 w2, float2 E2, Wkv4Carry2& cr,
                                                  float2& fprod, float2& gwn, float2& gu_acc, E* gkl, E* gvl, E* grl,
                                                  int C) {
  // the stash holds f1, f2 (scaled form, ungated, shared memory) or z1
  constexpr bool kStashF = S && SCALED && !GATE;
  constexpr int kReg = S ? 1 : kBwdL;
  float2 saa[kReg], sbb[kReg], sz[kReg];
  if constexpr (S) {
    // groups of kGrp tokens: the exponent chain of the group, then its value
    // updates and stash writes (z of one group in registers)
    constexpr int kGrp = WKV4_BWD_RECOMP_GROUP;
#pragma unroll
    for (int j0 = 0; j0 < kBwdL; j0 += kGrp) {
      float2 z[kGrp];
#pragma unroll
      for (int j = 0; j < kGrp; ++j) {
        if (WKV4_BWD_WHOLE_RECOMPUTE && WHOLE || j0 + j < n) {
          float2 unused;
          z[j] = wkv4_chain2<true, false>(st, wkv4_key2(ld_pair(&ks[j0 + j][2 * lane]), ref), splat2(0.f), w2, unused);
        }
      }
#pragma unroll
      for (int j = 0; j < kGrp; ++j) {
        const int jj = j0 + j;
        if (WKV4_BWD_WHOLE_RECOMPUTE && WHOLE || jj < n) {
          const float2 aa = st.aa, bb = st.bb;
          const float2 vj = ld_pair(&vs[jj][2 * lane]);
          float2 f1, f2;
          wkv4_factors2<false>(z[j], f1, f2);
          st.aa = fma2(f2, vj, mul2(f1, st.aa));
          st.bb = fma2(f1, st.bb, f2);
          sx.ab[jj][lane] = make_float4(aa.x, aa.y, bb.x, bb.y);
          if constexpr (GATE)
            sx.zv[jj][lane] = z[j];
          else if constexpr (kStashF)
            sx.zv[jj][lane] = make_float4(f1.x, f1.y, f2.x, f2.y);
          else
            sx.zv[jj][lane] = make_float4(z[j].x, z[j].y, vj.x, vj.y);
        }
      }
    }
  } else {
    // register stash: one token at a time (the stash already holds ~100
    // registers)
#pragma unroll
    for (int jj = 0; jj < kBwdL; ++jj) {
      if (WKV4_BWD_WHOLE_RECOMPUTE && WHOLE || jj < n) {
        saa[jj] = st.aa;
        sbb[jj] = st.bb;
        sz[jj] = wkv4_absorb2<false>(st, wkv4_key2(ld_pair(&ks[jj][2 * lane]), ref), ld_pair(&vs[jj][2 * lane]), w2);
      }
    }
  }
  float2 A = cr.A, B = cr.B, Ap = cr.Ap, Bp = cr.Bp;
#pragma unroll
  for (int jj = kBwdL - 1; jj >= 0; --jj) {
    if (WHOLE || jj < n) {
      const float2 g = ld_pair(&gs[jj][2 * lane]);
      const float2 rr = GATE ? ld_pair(&rs[jj][2 * lane]) : splat2(0.f);
      float2 aa, bb, zz = splat2(0.f), vv, f1, f2;
      if constexpr (S) {
        const float4 ab = sx.ab[jj][lane];
        aa = make_float2(ab.x, ab.y);
        bb = make_float2(ab.z, ab.w);
        if constexpr (GATE) {
          zz = sx.zv[jj][lane];
          vv = ld_pair(&vs[jj][2 * lane]);
          wkv4_factors2<false>(zz, f1, f2);
        } else if constexpr (kStashF) {
          const float4 ff = sx.zv[jj][lane];
          f1 = make_float2(ff.x, ff.y);
          f2 = make_float2(ff.z, ff.w);
          vv = ld_pair(&vs[jj][2 * lane]);
        } else {
          const float4 zv = sx.zv[jj][lane];
          zz = make_float2(zv.x, zv.y);
          vv = make_float2(zv.z, zv.w);
          wkv4_factors2<false>(zz, f1, f2);
        }
      } else {
        aa = saa[jj];
        bb = sbb[jj];
        zz = sz[jj];
        vv = ld_pair(&vs[jj][2 * lane]);
        wkv4_factors2<false>(zz, f1, f2);
      }
      wkv4_bwd_rstep<FULL, GATE, SCALED>(A, B, Ap, Bp, fprod, gwn, gu_acc, vv, g, rr, aa, bb, zz, f1, f2, uw2, E2,
                                         gkl + (int64_t)jj * C, gvl + (int64_t)jj * C,
                                         GATE ? grl + (int64_t)jj * C : nullptr);
    }
  }
  cr = {A, B, Ap, Bp};
}

// One carry merge for one channel: the carry `in` entering segment r from
// the later ones, folded through segment r (len steps, its local carry `own`
// and product of f1 `f`).
__device__ __forceinline__ void wkv4_carry_fold(float& A, float& B, float& Ap, float& Bp, float f, float m,
                                                float oA, float oB, float oAp, float oBp) {
  const float nA = __fmaf_rn(f, A, oA), nB = __fmaf_rn(f, B, oB);
  const float nAp = __fmaf_rn(f, __fmaf_rn(m, A, Ap), oAp), nBp = __fmaf_rn(f, __fmaf_rn(m, B, Bp), oBp);
  A = nA;
  B = nB;
  Ap = nAp;
  Bp = nBp;
}

template <class E, int STAGES, int NSEG, int NW, bool GATE>
__global__ void __launch_bounds__(32 * NW, NSEG == 1 ? 8 : 1) wkv4_bwd_kernel(const __grid_constant__ CUtensorMap tk,
                                                           const __grid_constant__ CUtensorMap tv,
                                                           const __grid_constant__ CUtensorMap tg,
                                                           const __grid_constant__ CUtensorMap tr, int T, int C,
                                                           int ncb, int ngroups, const float* __restrict__ w,
                                                           const float* __restrict__ u, const E* __restrict__ kraw,
                                                           const float* __restrict__ ckpt, E* __restrict__ gk,
                                                           E* __restrict__ gv, E* __restrict__ gr,
                                                           float* __restrict__ part_gw,
                                                           float* __restrict__ part_gu, unsigned* err) {
  extern __shared__ __align__(128) unsigned char wkv4_bwd_dsmem[];
  // each warp is an independent lane group with its own ring and barriers
  Wkv4BwdSmem<E, STAGES, GATE>& sm =
      reinterpret_cast<Wkv4BwdSmem<E, STAGES, GATE>*>(wkv4_bwd_dsmem)[threadIdx.x / 32];
  constexpr uint32_t kStageBytes = (GATE ? 4u : 3u) * kBwdL * kBwdCh * sizeof(E);
  constexpr int kPasses = NSEG > 1 ? 2 : 1;

  const int lane = threadIdx.x % 32;
  const int seg = NSEG > 1 ? (int)(blockIdx.x % NSEG) : 0;  // == cluster rank
  const int group = (blockIdx.x / NSEG) * NW + threadIdx.x / 32;
  const bool active = group < ngroups;  // a warp past the last group only joins the cluster barriers
  const int cb = group % ncb;
  const int b = group / ncb;
  const int c0 = cb * kBwdCh;
  const int c = c0 + 2 * lane;  // this lane's channels c, c + 1
  const bool valid = active && c < C;
  const int nck = (T + kBwdL - 1) / kBwdL;
  const int i_beg = wkv4_seg_begin(seg, NSEG, nck);
  const int i_end = wkv4_seg_begin(seg + 1, NSEG, nck);
  const int nloc = active ? i_end - i_beg : 0;  // intervals of this segment, walked last to first
  // segment 0's own carry is read by no other segment: no phase 1 there
  const bool own_pass = kPasses > 1 && seg > 0;
  const int total = (own_pass ? 2 : 1) * nloc;
  auto interval = [&](int qq) { return i_end - 1 - (qq % nloc); };

  auto issue = [&](int qq) {
    const int s = qq % STAGES;
    const int t0 = interval(qq) * kBwdL;
    mbar_arrive_expect_tx(&sm.full[s], kStageBytes);
    tma_load_3d(&sm.k[s][0][0], &tk, &sm.full[s], c0, t0, b);
    tma_load_3d(&sm.v[s][0][0], &tv, &sm.full[s], c0, t0, b);
    tma_load_3d(&sm.gy[s][0][0], &tg, &sm.full[s], c0, t0, b);
    if constexpr (GATE) tma_load_3d(&sm.g.r[s][0][0], &tr, &sm.full[s], c0, t0, b);
  };
  if (lane == 0) {
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    tma_prefetch_desc(&tg);
    if constexpr (GATE) tma_prefetch_desc(&tr);
    for (int s = 0; s < STAGES; ++s) mbar_init(&sm.full[s], 1);
    mbar_init_fence();
    for (int qq = 0; qq < STAGES && qq < total; ++qq) issue(qq);
  }
  __syncwarp();

  const float2 w2 = valid ? mul2(ld_pair(w + c), splat2(kLog2e)) : splat2(0.f);
  const float2 u2 = valid ? mul2(ld_pair(u + c), splat2(kLog2e)) : splat2(0.f);
  const float2 uw2 = sub2(u2, w2);  // output exponent minus absorb exponent
  // output form of the pair (wkv4_scaled_pair) and its channel constants 2^{u2 - w2}
  const bool scaled = wkv4_scaled_pair2(u2, w2);
  const float2 E2 = wkv4_out_scale2(u2, w2);
  const int64_t lane_off = valid ? (int64_t)b * T * C + c : 0;
  // lane reference exponents: the values the forward derived from token 0
  float2 ref = splat2(0.f);
  if (valid) {
    const float2 kf = ld_pair(kraw + lane_off);
    ref = make_float2(wkv4_ref(kf.x), wkv4_ref(kf.y));
  }
  const float* ckl = ckpt + (valid ? (int64_t)b * nck * 3 * C + c : 0);
  auto load_ckpt = [&](int i) -> Wkv4State2 {
    if (!valid) return {splat2(0.f), splat2(0.f), splat2(0.f), splat2(0.f)};
    const float* p = ckl + (int64_t)i * 3 * C;
    return {ld_pair(p), ld_pair(p + C), ld_pair(p + 2 * (int64_t)C), splat2(0.f)};
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
  Wkv4Carry2 cr = {splat2(0.f), splat2(0.f), splat2(0.f), splat2(0.f)};
  float2 gwn = splat2(0.f), gu_acc = splat2(0.f);
  auto run_interval = [&](auto full_tag, int s, int i, const Wkv4State2& st, float2& fprod) {
    constexpr bool kFull = decltype(full_tag)::value;
    const int n = min(kBwdL, T - i * kBwdL);
    const int64_t off = lane_off + (int64_t)i * kBwdL * C;
    E* gkp = kFull ? gk + off : nullptr;
    E* gvp = kFull ? gv + off : nullptr;
    E* grp = kFull && GATE ? gr + off : nullptr;
    const E (*rs)[kBwdCh] = nullptr;
    if constexpr (GATE) rs = sm.g.r[s];
    auto go = [&](auto whole_tag, auto scaled_tag) {
      wkv4_bwd_interval<kFull, decltype(whole_tag)::value, GATE, decltype(scaled_tag)::value>(
          sm.k[s], sm.v[s], sm.gy[s], rs, sm.stash, lane, n, st, ref, uw2, w2, E2, cr, fprod, gwn, gu_acc, gkp, gvp,
          grp, C);
    };
    if (WKV4_BWD_WHOLE && n == kBwdL) {
      if (scaled)
        go(BoolConst<true>{}, BoolConst<true>{});
      else
        go(BoolConst<true>{}, BoolConst<false>{});
    } else {
      if (scaled)
        go(BoolConst<false>{}, BoolConst<true>{});
      else
        go(BoolConst<false>{}, BoolConst<false>{});
    }
  };

  if constexpr (NSEG > 1) {
    // ---- phase 1: this segment's own carry, from an empty future ----
    float2 fprod = splat2(1.f);
    Wkv4State2 nxt = nloc > 0 ? load_ckpt(interval(0)) : Wkv4State2{splat2(0.f), splat2(0.f), splat2(0.f), splat2(0.f)};
    for (; own_pass && ok && qq < nloc; ++qq) {
      const int i = interval(qq);
      const Wkv4State2 st = nxt;
      if (qq + 1 < nloc) nxt = load_ckpt(interval(qq + 1));
      if (!acquire(qq)) break;
      if (valid) run_interval(BoolConst<false>{}, qq % STAGES, i, st, fprod);
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
    // every later segment's carry is requested first (independent remote
    // loads in flight together), then they are folded in order
    float2 pc[NSEG][5];
#pragma unroll
    for (int r = 1; r < NSEG; ++r)
      if (r > seg)
#pragma unroll
        for (int comp = 0; comp < 5; ++comp) pc[r][comp] = ld_shared_cluster_f2(map_shared_rank(&sm.carry[comp][lane], r));
    float in[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int r = NSEG - 1; r >= 1; --r) {
      if (r > seg) {
        const int len = min(T, wkv4_seg_begin(r + 1, NSEG, nck) * kBwdL) - wkv4_seg_begin(r, NSEG, nck) * kBwdL;
        const float m = (float)len;
        wkv4_carry_fold(in[0][0], in[0][1], in[0][2], in[0][3], pc[r][4].x, m, pc[r][0].x, pc[r][1].x, pc[r][2].x,
                        pc[r][3].x);
        wkv4_carry_fold(in[1][0], in[1][1], in[1][2], in[1][3], pc[r][4].y, m, pc[r][0].y, pc[r][1].y, pc[r][2].y,
                        pc[r][3].y);
      }
    }
    cluster_arrive_release();  // done reading peers; waited for before exit
    cr = {make_float2(in[0][0], in[1][0]), make_float2(in[0][1], in[1][1]), make_float2(in[0][2], in[1][2]),
          make_float2(in[0][3], in[1][3])};
    gwn = splat2(0.f);
    gu_acc = splat2(0.f);
  }

  // ---- last pass: gradients ----
  {
    float2 unused = splat2(1.f);
    Wkv4State2 nxt = nloc > 0 ? load_ckpt(interval(0)) : Wkv4State2{splat2(0.f), splat2(0.f), splat2(0.f), splat2(0.f)};
    for (; ok && qq < total; ++qq) {
      const int i = interval(qq);
      const Wkv4State2 st = nxt;
      if (qq + 1 < total) nxt = load_ckpt(interval(qq + 1));
      if (!acquire(qq)) break;
      if (valid) run_interval(BoolConst<true>{}, qq % STAGES, i, st, unused);
      release(qq);
    }
  }
  if (!ok && lane == 0)
    for (int x = qq; x < total && x < qq + STAGES; ++x) mbar_wait_bounded(&sm.full[x % STAGES], (x / STAGES) & 1, err);
  if (valid) {
    // after a wait that gave up (recorded in the device error word) the
    // partial sums are written as zeros, so the batch sum never reads a
    // value left in the scratch by an earlier call
    const int64_t pi = ((int64_t)b * NSEG + seg) * C + c;
    st_pair(part_gw + pi, ok ? neg2(gwn) : splat2(0.f));
    st_pair(part_gu + pi, ok ? gu_acc : splat2(0.f));
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

template <class E, int STAGES, int NSEG, int NW, bool GATE>
static wkv_status run_bwd(const Wkv4BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  CUtensorMap tk, tv, tg, tr;
  const CUtensorMapDataType ty = Elem<E>::tma_type;
  if (!encode_tmap_3d(&tk, a.k, ty, sizeof(E), a.C, a.T, a.B, kBwdCh, kBwdL, 1, why) ||
      !encode_tmap_3d(&tv, a.v, ty, sizeof(E), a.C, a.T, a.B, kBwdCh, kBwdL, 1, why) ||
      !encode_tmap_3d(&tg, a.gy, ty, sizeof(E), a.C, a.T, a.B, kBwdCh, kBwdL, 1, why))
    return WKV_ERR_INVALID_ARG;
  if (!GATE)
    tr = tk;  // unused
  else if (!encode_tmap_3d(&tr, a.r, ty, sizeof(E), a.C, a.T, a.B, kBwdCh, kBwdL, 1, why))
    return WKV_ERR_INVALID_ARG;
  const int ncb = (int)ceil_div(a.C, kBwdCh);
  const int ngroups = (int)(ncb * a.B);
  const int64_t rows = a.B * NSEG;
  float* part_gw = a.part;
  float* part_gu = a.part + rows * a.C;
  auto kern = wkv4_bwd_kernel<E, STAGES, NSEG, NW, GATE>;
  const size_t smem = NW * sizeof(Wkv4BwdSmem<E, STAGES, GATE>);
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
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tk, tv, tg, tr, (int)a.T, (int)a.C, ncb, ngroups, a.w, a.u,
                                     static_cast<const E*>(a.k), a.ckpt, static_cast<E*>(a.gk), static_cast<E*>(a.gv),
                                     static_cast<E*>(a.gr), part_gw, part_gu, err);
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

// Stages of the k/v/gy ring (one checkpoint interval each): two for bf16
// next to the stash (6 KB a stage, 8 KB gated), two for float32 (12 KB,
// 16 KB gated), so that the 6-7 one-warp CTAs an SM holds still fit in
// shared memory.
template <class E, int STAGES, int NSEG, bool GATE>
static wkv_status run_bwd_nw(const Wkv4BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  switch (wkv4_warps_per_cta(a.B, a.C, NSEG)) {
    case 4: return run_bwd<E, STAGES, NSEG, 4, GATE>(a, stream, err, why);
    case 2: return run_bwd<E, STAGES, NSEG, 2, GATE>(a, stream, err, why);
    default: return run_bwd<E, STAGES, NSEG, 1, GATE>(a, stream, err, why);
  }
}

template <class E, bool GATE>
static wkv_status run_bwd_nseg(const Wkv4BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  constexpr int kStages = sizeof(E) == 2 ? (bwd_smem_stash<E>() ? WKV4_BWD_STAGES_STASH : 4) : 2;
  switch (wkv4_bwd_segments(a.B, a.T, a.C)) {
#if WKV4_MAX_SEGMENTS_ANY > 8
    case 16: return run_bwd_nw<E, kStages, 16, GATE>(a, stream, err, why);
#endif
    case 8: return run_bwd_nw<E, kStages, 8, GATE>(a, stream, err, why);
    case 4: return run_bwd_nw<E, kStages, 4, GATE>(a, stream, err, why);
    case 2: return run_bwd_nw<E, kStages, 2, GATE>(a, stream, err, why);
    default: return run_bwd<E, kStages, 1, 1, GATE>(a, stream, err, why);
  }
}

wkv_status launch_wkv4_backward(const Wkv4BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  if (a.r) {
    if (a.dtype == WKV_BF16) return run_bwd_nseg<__nv_bfloat16, true>(a, stream, err, why);
    return run_bwd_nseg<float, true>(a, stream, err, why);
  }
  if (a.dtype == WKV_BF16) return run_bwd_nseg<__nv_bfloat16, false>(a, stream, err, why);
  return run_bwd_nseg<float, false>(a, stream, err, why);
}

}  // namespace wkv
