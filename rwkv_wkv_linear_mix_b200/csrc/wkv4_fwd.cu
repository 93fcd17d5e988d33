// wkv4_fwd.cu -- RWKV-4 WKV forward on sm_100a.
//
// Operator: the WKV of RWKV_TimeMix.forward, RUN_CUDA(B, T, C, time_decay,
// time_first, k, v) ("代码连连看——RWKV", section RWKV_TimeMix), evaluated as the
// running-max recurrence of wkv_device.cuh.
//
// Design. The recurrence is sequential in t and independent per lane (b, c).
// A warp owns 64 consecutive channels of one sample, a pair per thread, and
// keeps their states in registers; the pair runs on the packed fp32
// instructions (wkv4_token2). When there are too few lanes to fill the GPU, each lane's
// sequence is split into NSEG segments of whole checkpoint intervals, one
// one-warp CTA per segment, the NSEG CTAs forming a thread-block cluster:
//   1. every CTA runs its segment from the empty past (absorb only) and leaves
//      the segment's own state in shared memory;
//   2. after a cluster barrier, CTA r reads the states of CTAs 0..r-1 through
//      distributed shared memory and folds them, each decayed across the
//      segments after it, into its exact incoming state;
//   3. every CTA reruns its segment from that state, writing y and the
//      checkpoints (the second read of k, v mostly hits L2).
// With NSEG = 1 phases 1-2 vanish and the kernel is the plain sequential scan
// (most such launches run it as wkv4_fwd_seq_kernel, below: the same tile in
// a one-warp CTA with static shared arrays).
// k and v stream through a ring of STAGES shared-memory tiles of LT steps,
// filled by 3-D TMA loads (box {64 ch, LT steps, 1 sample}; rows past the
// segment are ignored) that complete on per-stage mbarriers; lane 0 refills a
// stage as soon as the warp has consumed it. y is written straight from
// registers. Every WKV4_CKPT_LEN steps the state (aa, bb, P) goes to the
// checkpoint buffer the backward restarts from; P is relative to the lane
// reference fl(k[b][0][c] * log2e), which the backward recomputes.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

// Channels one warp covers: 32 lanes x a pair each.
constexpr int kFwdCh = WKV4_WARP_CH;

// Output form of the tiles of each kernel (kYTest, or kYNone / kYStore
// chosen per launch). Measured on the B200 at B = 16, T = 4096, C = 4096
// (bf16): the general kernel 0.307 ms with the per-token test, 0.337 ms with
// the fixed forms; gated, 0.487 against 0.448 ms the other way round; the
// sequential kernel at the 3B width 0.274 ms with the fixed forms, 0.298 ms
// with the test.
#ifndef WKV4_FWD_GENERAL_YTEST
#define WKV4_FWD_GENERAL_YTEST 1
#endif

// The gate input r rides in the same ring when the output is gated.
template <class E, int LT, int STAGES, bool GATE>
struct Wkv4GateRing {
  E r[STAGES][LT][kFwdCh];
};
template <class E, int LT, int STAGES>
struct Wkv4GateRing<E, LT, STAGES, false> {};

template <class E, int LT, int STAGES, bool GATE>
struct alignas(128) Wkv4FwdSmem {
  E k[STAGES][LT][kFwdCh];
  E v[STAGES][LT][kFwdCh];
  Wkv4GateRing<E, LT, STAGES, GATE> g;
  uint64_t full[STAGES];
  float2 seg_aa[32], seg_bb[32], seg_P[32];  // this segment's own state (phase 1)
};

// State (aa, bb, P) before a token to its checkpoint slot p ([3][C] floats).
__device__ __forceinline__ void wkv4_write_ckpt(float* p, const Wkv4State2& st, float2 w2, int C) {
  st_pair(p, st.aa);
  st_pair(p + C, st.bb);
  st_pair(p + 2 * (int64_t)C, wkv4_exponent2(st, w2));
}

// A whole tile of N tokens (N a multiple of WKV4_CKPT_LEN) for a lane's
// channel pair, one checkpoint interval at a time: the exponent chain of the
// interval's tokens runs first (z1, and zo for the exact form, kept in
// registers), then their value updates and outputs. The chain is cheap and
// serial; the second half's ex2/rcp of different tokens are independent, so
// the split lets them overlap instead of waiting on one token at a time.
// ckt: the tile's first checkpoint slot (null: none written). YM: how the
// outputs are written: kYNone (yt null), kYStore (yt not null) or kYTest
// (yt tested at every token). The two fixed forms and the test compile to
// different schedules; which is faster depends on the kernel around the tile
// (measured on the B200, see the launchers).
constexpr int kYNone = 0, kYStore = 1, kYTest = 2;
template <int V>
struct IntConst {
  static constexpr int value = V;
};
template <bool SCALED, bool GATE, int N, int YM, class E>
__device__ __forceinline__ void wkv4_fwd_tile(Wkv4State2& st, const E (*ks)[kFwdCh], const E (*vs)[kFwdCh],
                                              const E (*rs)[kFwdCh], int lane, float2 ref, float2 u2, float2 w2,
                                              float2 E2, E* yt, float* ckt, int C) {
  constexpr int L = WKV4_CKPT_LEN;
#pragma unroll
  for (int jc = 0; jc < N; jc += L) {
    if (ckt) wkv4_write_ckpt(ckt + (int64_t)(jc / L) * 3 * C, st, w2, C);
    float2 z[L], zo[L];
#pragma unroll
    for (int j = 0; j < L; ++j) z[j] = wkv4_chain2<SCALED>(st, wkv4_key2(ld_pair(&ks[jc + j][2 * lane]), ref), u2, w2, zo[j]);
#pragma unroll
    for (int j = 0; j < L; ++j) {
      float2 yv = wkv4_values2<SCALED>(st, z[j], zo[j], ld_pair(&vs[jc + j][2 * lane]), E2);
      if constexpr (GATE) yv = mul2(yv, sigmoid2(ld_pair(&rs[jc + j][2 * lane])));
      if constexpr (YM == kYStore)
        st_pair(yt + (int64_t)(jc + j) * C, yv);
      else if constexpr (YM == kYTest)
        if (yt) st_pair(yt + (int64_t)(jc + j) * C, yv);
    }
  }
}

template <class E, int LT, int STAGES, int NSEG, int NW, bool GATE>
__global__ void __launch_bounds__(32 * NW) wkv4_fwd_kernel(const __grid_constant__ CUtensorMap tk,
                                                           const __grid_constant__ CUtensorMap tv,
                                                           const __grid_constant__ CUtensorMap tr,
                                                           const E* __restrict__ kraw, int T, int C, int ncb,
                                                           int ngroups, const float* __restrict__ w,
                                                           const float* __restrict__ u, E* __restrict__ y,
                                                           float* __restrict__ ckpt, unsigned* err) {
  static_assert(LT % WKV4_CKPT_LEN == 0, "a tile must hold whole checkpoint intervals");
  extern __shared__ __align__(128) unsigned char wkv4_fwd_dsmem[];
  // each warp is an independent lane group with its own ring and barriers
  Wkv4FwdSmem<E, LT, STAGES, GATE>& sm =
      reinterpret_cast<Wkv4FwdSmem<E, LT, STAGES, GATE>*>(wkv4_fwd_dsmem)[threadIdx.x / 32];
  constexpr uint32_t kStageBytes = (GATE ? 3u : 2u) * LT * kFwdCh * sizeof(E);
  constexpr int kPasses = NSEG > 1 ? 2 : 1;

  const int lane = threadIdx.x % 32;
  const int seg = NSEG > 1 ? (int)(blockIdx.x % NSEG) : 0;  // == cluster rank (1-D clusters)
  const int group = (blockIdx.x / NSEG) * NW + threadIdx.x / 32;
  const bool active = group < ngroups;  // a warp past the last group only joins the cluster barriers
  const int cb = group % ncb;
  const int b = group / ncb;
  const int c0 = cb * kFwdCh;
  const int c = c0 + 2 * lane;  // this lane's channels c, c + 1
  const bool valid = active && c < C;
  const int nck = (T + WKV4_CKPT_LEN - 1) / WKV4_CKPT_LEN;
  const int t_beg = wkv4_seg_begin(seg, NSEG, nck) * WKV4_CKPT_LEN;
  const int t_end = min(T, wkv4_seg_begin(seg + 1, NSEG, nck) * WKV4_CKPT_LEN);
  const int ntile = (active && t_end > t_beg) ? (t_end - t_beg + LT - 1) / LT : 0;
  // the last segment's own state is read by no other segment: no phase 1 there
  const bool own_pass = kPasses > 1 && seg < NSEG - 1;
  const int total = (own_pass ? 2 : 1) * ntile;  // tiles streamed through the ring

  auto issue = [&](int q) {
    const int s = q % STAGES;
    const int t = t_beg + (q % ntile) * LT;
    mbar_arrive_expect_tx(&sm.full[s], kStageBytes);
    tma_load_3d(&sm.k[s][0][0], &tk, &sm.full[s], c0, t, b);
    tma_load_3d(&sm.v[s][0][0], &tv, &sm.full[s], c0, t, b);
    if constexpr (GATE) tma_load_3d(&sm.g.r[s][0][0], &tr, &sm.full[s], c0, t, b);
  };
  if (lane == 0) {
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    if constexpr (GATE) tma_prefetch_desc(&tr);
    for (int s = 0; s < STAGES; ++s) mbar_init(&sm.full[s], 1);
    mbar_init_fence();
    for (int q = 0; q < STAGES && q < total; ++q) issue(q);
  }
  __syncwarp();

  const int64_t lane_off = valid ? (int64_t)b * T * C + c : 0;
  const float2 w2 = valid ? mul2(ld_pair(w + c), splat2(kLog2e)) : splat2(0.f);
  const float2 u2 = valid ? mul2(ld_pair(u + c), splat2(kLog2e)) : splat2(0.f);
  float2 ref = splat2(0.f);
  if (valid) {
    const float2 kf = ld_pair(kraw + lane_off);
    ref = make_float2(wkv4_ref(kf.x), wkv4_ref(kf.y));
  }
  float* ckl = ckpt ? ckpt + (int64_t)b * nck * 3 * C + c : nullptr;

  int q = 0;          // next tile to consume
  bool ok = true;     // every wait so far completed
  auto acquire = [&](int qq) {
    const bool got = mbar_wait_bounded(&sm.full[qq % STAGES], (qq / STAGES) & 1, err);
    ok = __all_sync(0xffffffffu, got);
    return ok;
  };
  auto release = [&](int qq) {
    __syncwarp();
    if (lane == 0 && qq + STAGES < total) issue(qq + STAGES);
  };

  Wkv4State2 st = wkv4_empty_state2();
  if constexpr (NSEG > 1) {
    // ---- phase 1: this segment from the empty past ----
    for (; own_pass && ok && q < ntile; ++q) {
      if (!acquire(q)) break;
      const int s = q % STAGES;
      const int n = min(LT, t_end - (t_beg + q * LT));
      if (valid) {
#pragma unroll 4
        for (int j = 0; j < n; ++j)
          wkv4_absorb2(st, wkv4_key2(ld_pair(&sm.k[s][j][2 * lane]), ref), ld_pair(&sm.v[s][j][2 * lane]), w2);
      }
      release(q);
    }
    sm.seg_aa[lane] = st.aa;
    sm.seg_bb[lane] = st.bb;
    sm.seg_P[lane] = wkv4_exponent2(st, w2);
    cluster_arrive_release();
    cluster_wait_acquire();
    // ---- phase 2: fold the segments before this one into the incoming state ----
    // every earlier segment's state is requested first (independent remote
    // loads in flight together), then they are merged in order
    float2 ra[NSEG], rb[NSEG], rp[NSEG];
#pragma unroll
    for (int r = 0; r < NSEG - 1; ++r) {
      if (r < seg) {
        ra[r] = ld_shared_cluster_f2(map_shared_rank(&sm.seg_aa[lane], r));
        rb[r] = ld_shared_cluster_f2(map_shared_rank(&sm.seg_bb[lane], r));
        rp[r] = ld_shared_cluster_f2(map_shared_rank(&sm.seg_P[lane], r));
      }
    }
    Wkv4Sum inx = {0.f, 0.f, kEmptyPP}, iny = inx;
#pragma unroll
    for (int r = 0; r < NSEG - 1; ++r) {
      if (r < seg) {
        const int len = min(T, wkv4_seg_begin(r + 1, NSEG, nck) * WKV4_CKPT_LEN) -
                        wkv4_seg_begin(r, NSEG, nck) * WKV4_CKPT_LEN;
        // decay the earlier part across segment r
        inx.P = __fmaf_rn(-(float)len, w2.x, inx.P);
        iny.P = __fmaf_rn(-(float)len, w2.y, iny.P);
        inx = wkv4_merge(inx, Wkv4Sum{ra[r].x, rb[r].x, rp[r].x});
        iny = wkv4_merge(iny, Wkv4Sum{ra[r].y, rb[r].y, rp[r].y});
      }
    }
    cluster_arrive_release();  // done reading peers; waited for before exit
    st = {make_float2(inx.aa, iny.aa), make_float2(inx.bb, iny.bb), make_float2(inx.P, iny.P), splat2(0.f)};
  }

  // ---- last pass: outputs and checkpoints ----
  E* yl = y ? y + lane_off : nullptr;
  const bool scaled = wkv4_scaled_pair2(u2, w2);
  const float2 E2 = wkv4_out_scale2(u2, w2);
  for (; ok && q < total; ++q) {
    const int t0 = t_beg + (q % ntile) * LT;  // a multiple of WKV4_CKPT_LEN
    if (!acquire(q)) break;
    const int s = q % STAGES;
    const int n = min(LT, t_end - t0);
    if (valid) {
      E* yt = yl ? yl + (int64_t)t0 * C : nullptr;
      float* ckt = ckl ? ckl + (int64_t)(t0 / WKV4_CKPT_LEN) * 3 * C : nullptr;
      const E(*rs)[kFwdCh] = nullptr;
      if constexpr (GATE) rs = sm.g.r[s];
      if (n == LT) {
        auto tile = [&](auto sc, auto ym) {
          wkv4_fwd_tile<decltype(sc)::value, GATE, LT, decltype(ym)::value>(st, sm.k[s], sm.v[s], rs, lane, ref, u2,
                                                                           w2, E2, yt, ckt, C);
        };
        if constexpr (WKV4_FWD_GENERAL_YTEST && !GATE) {
          if (scaled) tile(BoolConst<true>{}, IntConst<kYTest>{});
          else tile(BoolConst<false>{}, IntConst<kYTest>{});
        } else {
          if (scaled) {
            if (yt) tile(BoolConst<true>{}, IntConst<kYStore>{});
            else tile(BoolConst<true>{}, IntConst<kYNone>{});
          } else {
            if (yt) tile(BoolConst<false>{}, IntConst<kYStore>{});
            else tile(BoolConst<false>{}, IntConst<kYNone>{});
          }
        }
      } else {
        for (int j = 0; j < n; ++j) {
          if (j % WKV4_CKPT_LEN == 0 && ckt) wkv4_write_ckpt(ckt + (int64_t)(j / WKV4_CKPT_LEN) * 3 * C, st, w2, C);
          float2 yv = wkv4_token2(st, wkv4_key2(ld_pair(&sm.k[s][j][2 * lane]), ref), ld_pair(&sm.v[s][j][2 * lane]),
                                  u2, w2, scaled, E2);
          if constexpr (GATE) yv = mul2(yv, sigmoid2(ld_pair(&rs[j][2 * lane])));
          if (yt) st_pair(yt + (int64_t)j * C, yv);
        }
      }
    }
    release(q);
  }
  if (!ok && lane == 0) {
    // A wait gave up: let the copies still in flight land before the CTA's
    // shared memory is released (each wait is itself bounded).
    for (int qq = q; qq < total && qq < q + STAGES; ++qq)
      mbar_wait_bounded(&sm.full[qq % STAGES], (qq / STAGES) & 1, err);
  }
  if constexpr (NSEG > 1) cluster_wait_acquire();  // peers may still read this CTA's segment state
}

// The unsplit launch (every lane group runs its whole sequence): one warp
// per CTA, its ring in statically sized shared arrays, and a plain loop of
// wait, tile, refill. The same step as wkv4_fwd_kernel with NSEG = 1; kept
// apart because the compiler schedules the tile's loads and arithmetic
// further apart in this form (a probe of the same tile code on the B200: 57
// cycles per token from static shared arrays, 87 from the dynamic array).
template <class E, int LT, int STAGES, bool GATE>
__global__ void __launch_bounds__(32) wkv4_fwd_seq_kernel(const __grid_constant__ CUtensorMap tk,
                                                          const __grid_constant__ CUtensorMap tv,
                                                          const __grid_constant__ CUtensorMap tr,
                                                          const E* __restrict__ kraw, int T, int C, int ncb,
                                                          const float* __restrict__ w, const float* __restrict__ u,
                                                          E* __restrict__ y, float* __restrict__ ckpt, unsigned* err) {
  static_assert(LT % WKV4_CKPT_LEN == 0, "a tile must hold whole checkpoint intervals");
  constexpr int RS = GATE ? STAGES : 1;
  __shared__ __align__(128) E ks[STAGES][LT][kFwdCh];
  __shared__ __align__(128) E vs[STAGES][LT][kFwdCh];
  __shared__ __align__(128) E rsm[RS][GATE ? LT : 1][kFwdCh];
  __shared__ uint64_t full[STAGES];
  constexpr uint32_t kStageBytes = (GATE ? 3u : 2u) * LT * kFwdCh * sizeof(E);

  const int lane = threadIdx.x;
  const int cb = blockIdx.x % ncb;
  const int b = blockIdx.x / ncb;
  const int c0 = cb * kFwdCh;
  const int c = c0 + 2 * lane;  // this lane's channels c, c + 1
  const bool valid = c < C;
  const int nck = (T + WKV4_CKPT_LEN - 1) / WKV4_CKPT_LEN;
  const int ntile = (T + LT - 1) / LT;

  auto issue = [&](int q) {
    const int s = q % STAGES;
    mbar_arrive_expect_tx(&full[s], kStageBytes);
    tma_load_3d(&ks[s][0][0], &tk, &full[s], c0, q * LT, b);
    tma_load_3d(&vs[s][0][0], &tv, &full[s], c0, q * LT, b);
    if constexpr (GATE) tma_load_3d(&rsm[s % RS][0][0], &tr, &full[s], c0, q * LT, b);
  };
  if (lane == 0) {
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    if constexpr (GATE) tma_prefetch_desc(&tr);
    for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
    mbar_init_fence();
    for (int q = 0; q < STAGES && q < ntile; ++q) issue(q);
  }
  __syncwarp();

  const int64_t lane_off = valid ? (int64_t)b * T * C + c : 0;
  const float2 w2 = valid ? mul2(ld_pair(w + c), splat2(kLog2e)) : splat2(0.f);
  const float2 u2 = valid ? mul2(ld_pair(u + c), splat2(kLog2e)) : splat2(0.f);
  float2 ref = splat2(0.f);
  if (valid) {
    const float2 kf = ld_pair(kraw + lane_off);
    ref = make_float2(wkv4_ref(kf.x), wkv4_ref(kf.y));
  }
  float* ckl = (ckpt && valid) ? ckpt + (int64_t)b * nck * 3 * C + c : nullptr;
  E* yl = (y && valid) ? y + lane_off : nullptr;
  const bool scaled = wkv4_scaled_pair2(u2, w2);
  const float2 E2 = wkv4_out_scale2(u2, w2);

  Wkv4State2 st = wkv4_empty_state2();
  int q = 0;
  bool ok = true;
  for (; q < ntile; ++q) {
    const int s = q % STAGES;
    ok = __all_sync(0xffffffffu, mbar_wait_bounded(&full[s], (q / STAGES) & 1, err));
    if (!ok) break;
    const int t0 = q * LT;
    const int n = min(LT, T - t0);
    if (valid) {
      E* yt = yl ? yl + (int64_t)t0 * C : nullptr;
      float* ckt = ckl ? ckl + (int64_t)(t0 / WKV4_CKPT_LEN) * 3 * C : nullptr;
      const E(*rs)[kFwdCh] = nullptr;
      if constexpr (GATE) rs = rsm[s % RS];
      if (n == LT) {
        auto tile = [&](auto sc, auto ym) {
          wkv4_fwd_tile<decltype(sc)::value, GATE, LT, decltype(ym)::value>(st, ks[s], vs[s], rs, lane, ref, u2, w2,
                                                                           E2, yt, ckt, C);
        };
        if (scaled) {
          if (yt) tile(BoolConst<true>{}, IntConst<kYStore>{});
          else tile(BoolConst<true>{}, IntConst<kYNone>{});
        } else {
          if (yt) tile(BoolConst<false>{}, IntConst<kYStore>{});
          else tile(BoolConst<false>{}, IntConst<kYNone>{});
        }
      } else {
        for (int j = 0; j < n; ++j) {
          if (j % WKV4_CKPT_LEN == 0 && ckt) wkv4_write_ckpt(ckt + (int64_t)(j / WKV4_CKPT_LEN) * 3 * C, st, w2, C);
          float2 yv = wkv4_token2(st, wkv4_key2(ld_pair(&ks[s][j][2 * lane]), ref), ld_pair(&vs[s][j][2 * lane]), u2,
                                  w2, scaled, E2);
          if constexpr (GATE) yv = mul2(yv, sigmoid2(ld_pair(&rs[j][2 * lane])));
          if (yt) st_pair(yt + (int64_t)j * C, yv);
        }
      }
    }
    __syncwarp();
    if (lane == 0 && q + STAGES < ntile) issue(q + STAGES);
  }
  if (!ok && lane == 0) {
    // A wait gave up: let the copies still in flight land before the CTA's
    // shared memory is released (each wait is itself bounded).
    for (int qq = q; qq < ntile && qq < q + STAGES; ++qq) mbar_wait_bounded(&full[qq % STAGES], (qq / STAGES) & 1, err);
  }
}

// Which unsplit launches take wkv4_fwd_seq_kernel. Measured on the B200
// (B = 16, T = 4096): bf16 at the 3B width (640 lane groups, 4.3 warps per
// SM) 0.274 ms against 0.307 ms for wkv4_fwd_kernel, but at C = 4096 (1,024
// groups, 6.9 per SM) 0.356 ms against 0.309 ms; float32 at C = 4096 0.58-
// 0.59 ms against 0.60-0.62 ms. So bf16 launches of more than
// WKV4_FWD_SEQ_MAX_GROUPS lane groups keep the general kernel.
#ifndef WKV4_FWD_SEQ_KERNEL
#define WKV4_FWD_SEQ_KERNEL 1
#endif
#ifndef WKV4_FWD_SEQ_MAX_GROUPS
#define WKV4_FWD_SEQ_MAX_GROUPS (148 * 5)
#endif

template <class E, int LT, int STAGES, int NSEG, int NW, bool GATE>
static wkv_status run_fwd(const Wkv4FwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  CUtensorMap tk, tv, tr;
  const CUtensorMapDataType ty = Elem<E>::tma_type;
  if (!encode_tmap_3d(&tk, a.k, ty, sizeof(E), a.C, a.T, a.B, kFwdCh, LT, 1, why) ||
      !encode_tmap_3d(&tv, a.v, ty, sizeof(E), a.C, a.T, a.B, kFwdCh, LT, 1, why))
    return WKV_ERR_INVALID_ARG;
  if (!GATE)
    tr = tk;  // unused
  else if (!encode_tmap_3d(&tr, a.r, ty, sizeof(E), a.C, a.T, a.B, kFwdCh, LT, 1, why))
    return WKV_ERR_INVALID_ARG;
  const int ncb = (int)ceil_div(a.C, kFwdCh);
  const int ngroups = (int)(ncb * a.B);
  if (NSEG == 1 && NW == 1 && WKV4_FWD_SEQ_KERNEL && (sizeof(E) == 4 || ngroups <= WKV4_FWD_SEQ_MAX_GROUPS)) {
    // all static: without a preference the driver may leave part of the
    // unified L1/shared memory to L1 and fit fewer of these CTAs on an SM
    auto seq = wkv4_fwd_seq_kernel<E, LT, STAGES, GATE>;
    if (cudaFuncSetAttribute(seq, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared) !=
        cudaSuccess) {
      *why = "wkv4_forward: shared memory configuration failed";
      return WKV_ERR_CUDA;
    }
    const unsigned grid = (unsigned)ngroups;
    seq<<<grid, 32, 0, stream>>>(
        tk, tv, tr, static_cast<const E*>(a.k), (int)a.T, (int)a.C, ncb, a.w, a.u, static_cast<E*>(a.y), a.ckpt, err);
    if (cudaGetLastError() != cudaSuccess) {
      *why = "wkv4_forward kernel launch failed";
      return WKV_ERR_CUDA;
    }
    return WKV_OK;
  }
  auto kern = wkv4_fwd_kernel<E, LT, STAGES, NSEG, NW, GATE>;
  const size_t smem = NW * sizeof(Wkv4FwdSmem<E, LT, STAGES, GATE>);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
    *why = "wkv4_forward: shared memory configuration failed";
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tk, tv, tr, static_cast<const E*>(a.k), (int)a.T, (int)a.C, ncb,
                                           ngroups, a.w, a.u, static_cast<E*>(a.y), a.ckpt, err);
  if (e != cudaSuccess) {
    *why = "wkv4_forward kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

template <class E, int LT, int STAGES, int NSEG, bool GATE>
static wkv_status run_fwd_nw(const Wkv4FwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  switch (wkv4_warps_per_cta(a.B, a.C, NSEG)) {
    case 4: return run_fwd<E, LT, STAGES, NSEG, 4, GATE>(a, stream, err, why);
    case 2: return run_fwd<E, LT, STAGES, NSEG, 2, GATE>(a, stream, err, why);
    default: return run_fwd<E, LT, STAGES, NSEG, 1, GATE>(a, stream, err, why);
  }
}

template <class E, int LT, int STAGES, bool GATE = false>
static wkv_status run_fwd_nseg(const Wkv4FwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  switch (wkv4_fwd_segments(a.B, a.T, a.C)) {
#if WKV4_MAX_SEGMENTS_ANY > 8
    case 16: return run_fwd_nw<E, LT, STAGES, 16, GATE>(a, stream, err, why);
#endif
    case 8: return run_fwd_nw<E, LT, STAGES, 8, GATE>(a, stream, err, why);
    case 4: return run_fwd_nw<E, LT, STAGES, 4, GATE>(a, stream, err, why);
    case 2: return run_fwd_nw<E, LT, STAGES, 2, GATE>(a, stream, err, why);
    default: return run_fwd<E, LT, STAGES, 1, 1, GATE>(a, stream, err, why);
  }
}

// Ring depth: each warp consumes its stream quickly relative to the ~1 us
// load latency, so several tiles must be in flight per warp.
#ifndef WKV4_FWD_STAGES_F32
#define WKV4_FWD_STAGES_F32 3
#endif
#ifndef WKV4_FWD_STAGES_BF16
#define WKV4_FWD_STAGES_BF16 3
#endif

wkv_status launch_wkv4_forward(const Wkv4FwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  if (a.r) {
    // gated: a third tile per stage, one stage fewer (same shared memory per warp)
    if (a.dtype == WKV_BF16) return run_fwd_nseg<__nv_bfloat16, 32, 2, true>(a, stream, err, why);
    return run_fwd_nseg<float, 16, 2, true>(a, stream, err, why);
  }
  if (a.dtype == WKV_BF16) return run_fwd_nseg<__nv_bfloat16, 32, WKV4_FWD_STAGES_BF16>(a, stream, err, why);
  return run_fwd_nseg<float, 16, WKV4_FWD_STAGES_F32>(a, stream, err, why);
}

}  // namespace wkv
