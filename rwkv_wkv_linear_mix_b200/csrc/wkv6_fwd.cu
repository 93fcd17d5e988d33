// wkv6_fwd.cu -- RWKV-6 head-state WKV forward on sm_100a, chunked, with the
// intra-chunk contractions on the tcgen05 tensor cores.
//
// Operator: RWKV6_OP (rwkv-ops package page, section "rwkv6op 使用方法", call
// and argument tables). Per (sample b, head h), key index i, value index j:
//   o_t[j]    = sum_i r_t[i] (S_{t-1}[i][j] + u[i] k_t[i] v_t[j])
//   S_t[i][j] = w_t[i] S_{t-1}[i][j] + k_t[i] v_t[j]
// with S_{-1} = 0 or init_state[state_map[b]] (n_state = 1: shared;
// n_state = B: one per sample).
//
// Chunked form. For a chunk of L <= 64 tokens t0 + j and the cumulative decay
// E_j[i] = prod_{tau <= j} w_{t0+tau}[i] (E_{-1} = 1):
//   o_j  = (r_j * E_{j-1}) S_in                                   (inter)
//        + sum_{s<j} [ (r_j * E_{j-1}) . (k_s / E_s) ] v_s
//        + [ r_j . (u * k_j) ] v_j                                (intra)
//   S_out = diag(E_{L-1}) S_in + sum_s (k_s * E_{L-1} / E_s)^T v_s
// The 64x64x64 products run on the tensor cores with fp32 accumulators in
// tensor memory:
//   MMA12 [A | O] = R^ [K~ ; S_in^T]^T   tf32, one N = 128 product:
//                  R^ = r * E_{j-1}, K~ = k / E_s, S_in the fp32 state
//   MMA4  dS = K^^T V       bf16: K^ = k * E_{L-1} / E_s (<= |k|)
//   MMA3  O += mask(A) V    bf16, mask(A) split hi = bf16(x), lo = bf16(x - hi)
//                           (two passes: bf16 alone would lose the 2e-2 bound)
// mask keeps s < j and puts the bonus r_j . (u * k_j) on s = j. E is a
// running product of the decays (no logarithms, no exponentials): R^ and K^
// never exceed |r|, |k|. K~ = k / E_s grows as the chunk decays, so a chunk
// whose total decay falls below 2^-96 in some channel is processed as
// sub-chunks of 16, then 4, then 1 token(s) (the same code with the tokens
// outside the sub-chunk masked: r = k = 0, w = 1). A single token needs no
// K~, so every w in (0, 1] is handled.
//
// For the backward the kernel can also write the state entering every
// 64-token chunk (ck_state, [B*H][chunks][64][64] fp32, [i][jv]), skip o,
// and run the time-reversed recurrence (REV: chunks last to first, each
// chunk's tokens in descending order; its output row t is the reversed
// recurrence's output for token t and ck_state[c] the state entering chunk c
// from above).
//
// Kernel shape: one CTA of 256 threads per (b, h), walking its chunks (and
// sub-chunks: "units") in order; two CTAs share an SM. Per unit n:
//   B. pass 1: product of w over each warp's 8 tokens, totals, split check
//   C. pass 2: R^, K~ (fp32), K^ = K~ E_{L-1} (bf16) and the bonus
//   D. TMA starts the next chunk's r, k tiles; MMA12 and MMA4 issued
//   E. epilogue of unit n - 1 (its O buffer) while those MMAs run
//   F. mask(A) -> am tiles; S = diag(E) S + dS -> registers and the S^T rows
//   G. MMA3 issued into unit n's O buffer (two buffers alternate)
// Warp g prepares tokens 8g .. 8g + 7 (lane = two channels, the bonus summed
// over the warp by shuffles); one thread issues the MMAs; accumulators are
// read back by warps 0-3 (columns 0-31) and 4-7 (columns 32-63) of the TMEM
// sub-partition warp % 4, all 32 lanes busy (16x256b loads), and the same
// threads keep the fp32 state, 16 values each. Waits are bounded (2 s): a wait that gives up records
// WKV_DEVERR_WAIT_TIMEOUT, the CTA drains its copies and MMAs in flight,
// frees its tensor memory and exits.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {


constexpr int kHead6 = 64;                         // head size K = V
constexpr int kChunk6 = 64;                        // tokens per chunk
constexpr int kThreads6 = 256;                     // 8 warps
constexpr uint32_t kTile6 = 8192;                  // 64 x 64 bf16, or one 64 x 32 fp32 panel
constexpr uint32_t kTmemCols6 = 256;               // tensor-memory columns allocated
constexpr uint32_t kColA = 0, kColO = 64, kColS = 128;  // A, O (adjacent: one N = 128 MMA), dS
constexpr float kMinChunkDecay6 = 1.2621774e-29f;  // 2^-96

struct alignas(1024) Wkv6Smem {
  uint8_t r[kTile6];      // bf16 r   [j][i]   of the current chunk
  uint8_t k[kTile6];      // bf16 k   [s][i]
  uint8_t w[kTile6];      // bf16 w   [j][i]
  uint8_t v[2][kTile6];   // bf16 v   [s][jv]  of the p-th chunk processed in v[p & 1]
  uint8_t rf[2][kTile6];  // R^ fp32, panels [i / 32][j][i % 32]            (A of MMA12)
  uint8_t bt[2][2 * kTile6];  // B of MMA12, fp32, panels [i / 32][128 rows][i % 32]:
                              // rows 0-63 K~ [s], rows 64-127 S_in^T [jv]; after
                              // MMA12 rows 0-63 of panel 0 / 1 hold hi / lo of
                              // mask(A), bf16 [j][s] (A of MMA3)
  uint8_t kh[kTile6];     // K^ bf16 [s][i] (A of MMA4); in pass 1 the w products
  float u[kHead6];
  float dec[kHead6];      // E_{L-1}: decay of the state across the unit
  float bonus[kHead6];    // r_j . (u * k_j)
  uint64_t w_bar, rk_bar, v_bar[2], mma_bar;
  uint32_t tmem_base;
};

// bf16 pair (channels 2 * lane, 2 * lane + 1) of row j of a swizzled bf16 tile.
__device__ __forceinline__ uint32_t tile_ld2(const uint8_t* tile, int j, int lane) {
  return *reinterpret_cast<const uint32_t*>(tile + j * 128 + ((((lane >> 2) ^ (j & 7)) & 7) << 4) + 4 * (lane & 3));
}
__device__ __forceinline__ void tile_st2(uint8_t* tile, int j, int lane, uint32_t v) {
  *reinterpret_cast<uint32_t*>(tile + j * 128 + ((((lane >> 2) ^ (j & 7)) & 7) << 4) + 4 * (lane & 3)) = v;
}
// Byte offset of the fp32 pair (columns 2 * lane, 2 * lane + 1) of row j of a
// two-panel swizzled fp32 tile whose panels are `panel` bytes apart.
__device__ __forceinline__ int f32_pair_off(int j, int lane, int panel) {
  return (lane >> 4) * panel + j * 128 + (((((lane & 15) >> 1) ^ (j & 7)) & 7) << 4) + (lane & 1) * 8;
}
// bf16 pair (columns col, col + 1; col even) of row `row` of a swizzled bf16 tile.
__device__ __forceinline__ void tile_st_pair(uint8_t* tile, int row, int col, uint32_t v) {
  *reinterpret_cast<uint32_t*>(tile + row * 128 + ((((col >> 3) ^ (row & 7)) & 7) << 4) + (col & 7) * 2) = v;
}
// Columns 16 q .. 16 q + 15 (q in 0..3) of row `row` of a bf16 tile.
__device__ __forceinline__ void tile_st_row16(uint8_t* tile, int row, int q, const uint32_t (&p)[8]) {
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int phys = ((2 * q + c) ^ (row & 7)) & 7;
    *reinterpret_cast<uint4*>(tile + row * 128 + phys * 16) = make_uint4(p[4 * c], p[4 * c + 1], p[4 * c + 2], p[4 * c + 3]);
  }
}
// x ~ hi + lo with hi = bf16(x), lo = bf16(x - hi), for a pair of values.
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(a, b);
  lo = pack_bf16x2(a - bf16lo(hi), b - bf16hi(hi));
}

// Pass 2 for the tokens 8g .. 8g + 7 of warp g: R^ = r E_{j-1} and
// K~ = k / E_s (fp32) from the prefix product `pre`, K^ = K~ E_{L-1} =
// k E_{L-1} / E_s (bf16; `tot` = E_{L-1}), and the bonus r_j . (u * k_j) of
// each token (this lane's two channels, then summed over the warp). FULL: the
// unit is the whole 64-token chunk (no masking).
// REV: the tokens are taken in descending order (the time-reversed
// recurrence): E runs over the rows after j, pre holds the product over the
// warps after this one.
template <bool FULL, bool REV>
__device__ __forceinline__ void wkv6_prepare(Wkv6Smem& sm, int g, int lane, int lo, int hi, const float (&w0)[8],
                                             const float (&w1)[8], float pre0, float pre1, float tot0, float tot1,
                                             float u0, float u1) {
  const bool need_kb = FULL || hi - lo > 1;  // one token has no s < j pair
  float e0 = pre0, e1 = pre1;
  float pb[8];  // this lane's part of each token's bonus
#pragma unroll
  for (int step = 0; step < 8; ++step) {
    const int jj = REV ? 7 - step : step;
    const int j = 8 * g + jj;
    const bool in = FULL || (j >= lo && j < hi);
    const uint32_t rx = tile_ld2(sm.r, j, lane), kx = tile_ld2(sm.k, j, lane);
    pb[jj] = in ? fmaf(bf16lo(rx) * u0, bf16lo(kx), bf16hi(rx) * u1 * bf16hi(kx)) : 0.f;
    float2 rh = make_float2(bf16lo(rx) * e0, bf16hi(rx) * e1);
    e0 *= w0[jj];
    e1 *= w1[jj];
    float2 kb = make_float2(bf16lo(kx) * rcp(e0), bf16hi(kx) * rcp(e1));
    // one token: E_{L-1} / E_s = 1, and K~ is not needed
    uint32_t kh = need_kb ? pack_bf16x2(kb.x * tot0, kb.y * tot1) : kx;
    if (!FULL) {
      if (!in) {
        rh = make_float2(0.f, 0.f);
        kh = 0u;
      }
      if (!(in && need_kb)) kb = make_float2(0.f, 0.f);
    }
    *reinterpret_cast<float2*>(sm.rf[0] + f32_pair_off(j, lane, kTile6)) = rh;
    *reinterpret_cast<float2*>(sm.bt[0] + f32_pair_off(j, lane, 2 * kTile6)) = kb;
    tile_st2(sm.kh, j, lane, kh);
  }
  // sum the 8 bonus parts over the warp's 32 lanes at once: each exchange
  // halves the tokens a lane keeps, so lane l ends with token (l / 4) % 8
  {
    float q4[4], q2[2];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const bool hi = lane & 16;
      q4[m] = (hi ? pb[m + 4] : pb[m]) + __shfl_xor_sync(0xffffffffu, hi ? pb[m] : pb[m + 4], 16);
    }
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const bool hi = lane & 8;
      q2[m] = (hi ? q4[m + 2] : q4[m]) + __shfl_xor_sync(0xffffffffu, hi ? q4[m] : q4[m + 2], 8);
    }
    const bool hi = lane & 4;
    float q1 = (hi ? q2[1] : q2[0]) + __shfl_xor_sync(0xffffffffu, hi ? q2[0] : q2[1], 4);
    q1 += __shfl_xor_sync(0xffffffffu, q1, 2);
    q1 += __shfl_xor_sync(0xffffffffu, q1, 1);
    if ((lane & 3) == 0) sm.bonus[8 * g + ((lane >> 2) & 7)] = q1;
  }
}

template <bool REV>
__global__ void __launch_bounds__(kThreads6, 2)
    wkv6_fwd_chunk_kernel(const __grid_constant__ CUtensorMap tr, const __grid_constant__ CUtensorMap tk,
                          const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tw, int T, int H,
                          const float* __restrict__ u, const float* __restrict__ init_state,
                          const int32_t* __restrict__ state_map, int n_state, float* __restrict__ final_state,
                          __nv_bfloat16* __restrict__ o, float* __restrict__ ck_state, unsigned* err) {
  extern __shared__ uint8_t wkv6_dsmem[];
  Wkv6Smem& sm = *reinterpret_cast<Wkv6Smem*>((reinterpret_cast<uintptr_t>(wkv6_dsmem) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x % H, b = blockIdx.x / H;
  const int64_t HK = (int64_t)H * kHead6;
  const int nch = (T + kChunk6 - 1) / kChunk6;
  // accumulator read-back: TMEM sub-partition sp, column half ch. With the
  // 32x32b shape lanes 0-15 hold row 16 sp + lane (the epilogue); with the
  // 16x256b shape every thread holds rows r0 = 16 sp + lane / 4 and r0 + 8,
  // columns 32 ch + 8 q + 2 (lane % 4) + {0, 1}, q = 0..3 (mask and state)
  const int sp = warp & 3, ch = warp >> 2;
  const int row = 16 * sp + lane;
  const bool holder = lane < 16;
  const int r0 = 16 * sp + (lane >> 2), r1 = r0 + 8;
  const int cq = 32 * ch + 2 * (lane & 3);  // + 8 q
  const float u0 = u[h * kHead6 + 2 * lane], u1 = u[h * kHead6 + 2 * lane + 1];

  if (tid == 0) {
    if (nch > 0) {
      tma_prefetch_desc(&tr);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      tma_prefetch_desc(&tw);
    }
    mbar_init(&sm.w_bar, 1);
    mbar_init(&sm.rk_bar, 1);
    mbar_init(&sm.v_bar[0], 1);
    mbar_init(&sm.v_bar[1], 1);
    mbar_init(&sm.mma_bar, 1);
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc(&sm.tmem_base, kTmemCols6);
  if (tid < kHead6) sm.u[tid] = u[h * kHead6 + tid];

  // fp32 state in registers, 16 values per thread in the 16x256b layout:
  // S[4q + e] = S[r0][cq + 8q + e], S[4q + 2 + e] = S[r1][cq + 8q + e]; its
  // tf32 operand copy is S^T in rows 64 + jv of bt (K-major: column i)
  float S[16];
  auto store_state = [&]() {
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = (e < 2) ? r0 : r1;
        const int jv = cq + 8 * q + (e & 1);
        *reinterpret_cast<float*>(sm.bt[i >> 5] + (64 + jv) * 128 + (((((i & 31) >> 2) ^ (jv & 7)) & 7) << 4) +
                                  (i & 3) * 4) = S[4 * q + e];
      }
  };
  {
    const float* s0 = nullptr;
    if (init_state) {
      const int sidx = state_map ? state_map[b] : (n_state == 1 ? 0 : b);
      if (sidx < 0 || sidx >= n_state) {
        if (tid == 0) record_error(err, WKV_DEVERR_BAD_STATE);
      } else {
        s0 = init_state + ((int64_t)sidx * H + h) * kHead6 * kHead6;
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float2 x0 = make_float2(0.f, 0.f), x1 = make_float2(0.f, 0.f);
      if (s0) {
        x0 = *reinterpret_cast<const float2*>(s0 + r0 * kHead6 + cq + 8 * q);
        x1 = *reinterpret_cast<const float2*>(s0 + r1 * kHead6 + cq + 8 * q);
      }
      S[4 * q] = x0.x;
      S[4 * q + 1] = x0.y;
      S[4 * q + 2] = x1.x;
      S[4 * q + 3] = x1.y;
    }
    store_state();
  }
  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tm = sm.tmem_base;
  const uint32_t tl = tm + ((uint32_t)(32 * sp) << 16);  // this warp's TMEM lanes

  // copies and MMA commits in flight, as seen by thread 0 (which issues them)
  int w_issued = 0, w_done = 0, rk_issued = 0, rk_done = 0, v_issued = 0, v_done = 0, mma_issued = 0, mma_done = 0;
  // chunks are processed in order (REV: last to first); pp counts them
  auto chunk_of = [&](int pp) { return REV ? nch - 1 - pp : pp; };
  auto load_w = [&](int pp) {
    mbar_arrive_expect_tx(&sm.w_bar, kTile6);
    tma_load_3d(sm.w, &tw, &sm.w_bar, h * kHead6, chunk_of(pp) * kChunk6, b);
    ++w_issued;
  };
  auto load_rk = [&](int pp) {
    mbar_arrive_expect_tx(&sm.rk_bar, 2 * kTile6);
    tma_load_3d(sm.r, &tr, &sm.rk_bar, h * kHead6, chunk_of(pp) * kChunk6, b);
    tma_load_3d(sm.k, &tk, &sm.rk_bar, h * kHead6, chunk_of(pp) * kChunk6, b);
    ++rk_issued;
  };
  auto load_v = [&](int pp) {
    mbar_arrive_expect_tx(&sm.v_bar[pp & 1], kTile6);
    tma_load_3d(sm.v[pp & 1], &tv, &sm.v_bar[pp & 1], h * kHead6, chunk_of(pp) * kChunk6, b);
    ++v_issued;
  };
  if (tid == 0 && nch > 0) {
    load_w(0);
    load_rk(0);
    load_v(0);
  }
  bool ok = true;
  uint32_t mma_phase = 0;
  // every thread waits (bounded) for a barrier phase; thread 0 books it
  auto wait_bar = [&](uint64_t* bar, uint32_t parity, int* done, int upto) {
    const bool got = mbar_wait_bounded(bar, parity, err);
    if (tid == 0 && got) *done = upto;
    ok = ok && got;
  };
  auto wait_mma = [&]() {
    wait_bar(&sm.mma_bar, mma_phase, &mma_done, mma_issued);
    mma_phase ^= 1u;
    tc_fence_after_sync();
  };

  constexpr uint32_t idt_12 = umma_idesc_tf32(64, 128, 0, 0);  // tf32 M64 N128, both K-major
  constexpr uint32_t idb_km = umma_idesc_bf16(64, 64, 0, 1);  // bf16, A K-major, B MN-major
  constexpr uint32_t idb_mm = umma_idesc_bf16(64, 64, 1, 1);  // bf16, A MN-major, B MN-major

  // the previous unit, whose O is still to be written out
  bool prev = false;
  int prev_t0 = 0, prev_lo = 0, prev_hi = 0;
  auto epilogue = [&]() {
    // MMA3 of the previous unit has completed (waited for by the caller)
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float ov[16];
      tmem_ld16(tl + kColO + 32 * ch + 16 * q, ov);
      tmem_wait_ld();
      if (o && ok && holder && row >= prev_lo && row < prev_hi) {
        uint32_t p[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) p[e / 2] = pack_bf16x2(ov[e], ov[e + 1]);
        uint4* dst = reinterpret_cast<uint4*>(o + ((int64_t)b * T + prev_t0 + row) * HK + h * kHead6 + 32 * ch + 16 * q);
        dst[0] = make_uint4(p[0], p[1], p[2], p[3]);
        dst[1] = make_uint4(p[4], p[5], p[6], p[7]);
      }
    }
    tc_fence_before_sync();
  };

  bool failed = false;
  for (int p = 0; p < nch && !failed; ++p) {
    const int c = chunk_of(p);
    const int t0 = c * kChunk6;
    const int valid = min(kChunk6, T - t0);
    const uint32_t vt = smem_u32(sm.v[p & 1]);
    int off = 0, size = kChunk6;
    bool first_unit = true;
    if (ck_state) {
      // the state entering chunk c, [i][jv] fp32, for the backward
      float* cs = ck_state + (((int64_t)b * H + h) * nch + c) * kHead6 * kHead6;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        *reinterpret_cast<float2*>(cs + r0 * kHead6 + cq + 8 * q) = make_float2(S[4 * q], S[4 * q + 1]);
        *reinterpret_cast<float2*>(cs + r1 * kHead6 + cq + 8 * q) = make_float2(S[4 * q + 2], S[4 * q + 3]);
      }
    }
    wait_bar(&sm.w_bar, (uint32_t)p & 1u, &w_done, p + 1);
    while (off < valid) {
      const int len = min(size, valid - off);
      const bool full = len == kChunk6;
      // the unit's rows: [off, off + len) in time order, or counted from the
      // chunk's last row for the reversed recurrence
      const int lo = REV ? valid - off - len : off, hi = lo + len;
      // ---- B. pass 1: product of w over this warp's 8 tokens (w = 1 outside) ----
      float w0[8], w1[8];
      {
        float p0 = 1.f, p1 = 1.f;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int j = 8 * warp + jj;
          const bool in = full || (j >= lo && j < hi);
          const uint32_t x = tile_ld2(sm.w, j, lane);
          w0[jj] = in ? bf16lo(x) : 1.f;
          w1[jj] = in ? bf16hi(x) : 1.f;
          p0 *= w0[jj];
          p1 *= w1[jj];
        }
        float* wq = reinterpret_cast<float*>(sm.kh);  // [8][64]
        *reinterpret_cast<float2*>(wq + warp * kHead6 + 2 * lane) = make_float2(p0, p1);
      }
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      float pre0 = 1.f, pre1 = 1.f, tot0 = 1.f, tot1 = 1.f;
      {
        const float* wq = reinterpret_cast<const float*>(sm.kh);
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const float2 q = *reinterpret_cast<const float2*>(wq + g * kHead6 + 2 * lane);
          if (REV ? g > warp : g < warp) {
            pre0 *= q.x;
            pre1 *= q.y;
          }
          tot0 *= q.x;
          tot1 *= q.y;
        }
      }
      // a unit that decays below 2^-96 is split (K~ = k / E could overflow);
      // nothing has been written yet, so it simply starts again smaller
      const bool deep = !(tot0 >= kMinChunkDecay6 && tot1 >= kMinChunkDecay6);
      if (__syncthreads_or(deep) && size > 1) {
        size >>= 2;
        continue;
      }
      const bool last_unit = off + len == valid;
      // the w tile is consumed: bring the next chunk's
      if (tid == 0 && last_unit && p + 1 < nch) load_w(p + 1);
      if (warp == 0) *reinterpret_cast<float2*>(&sm.dec[2 * lane]) = make_float2(tot0, tot1);
      // ---- E. write out the previous unit (its MMA3 overlapped pass 1) ----
      if (prev) {
        wait_mma();
        epilogue();
      }
      // the v buffer of the chunk before is free now: bring the next chunk's
      if (tid == 0 && first_unit && p + 1 < nch) load_v(p + 1);
      if (first_unit) {
        wait_bar(&sm.rk_bar, (uint32_t)p & 1u, &rk_done, p + 1);
        wait_bar(&sm.v_bar[p & 1], (uint32_t)(p >> 1) & 1u, &v_done, p + 1);
      }
      // ---- C. pass 2 ----
      if (full)
        wkv6_prepare<true, REV>(sm, warp, lane, lo, hi, w0, w1, pre0, pre1, tot0, tot1, u0, u1);
      else
        wkv6_prepare<false, REV>(sm, warp, lane, lo, hi, w0, w1, pre0, pre1, tot0, tot1, u0, u1);
      fence_proxy_async_smem();
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      // ---- D. next chunk's r, k; MMA1 A = R^ K~^T, MMA2 O = R^ S_in, MMA4 dS = K^^T V ----
      if (tid == 0) {
        if (last_unit && p + 1 < nch) load_rk(p + 1);
        tc_fence_after_sync();
        // descriptors advance by whole 16-byte units in their low bits
        const uint64_t da = umma_desc_sw128(smem_u32(sm.rf[0]), 16, 1024);
        const uint64_t db = umma_desc_sw128(smem_u32(sm.bt[0]), 16, 1024);
        const uint64_t dk = umma_desc_sw128(smem_u32(sm.kh), 8192, 1024);
        const uint64_t dv = umma_desc_sw128(vt, 8192, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_tf32(tm + kColA, da + ((kk >> 2) * kTile6 + (kk & 3) * 32) / 16,
                    db + ((kk >> 2) * 2 * kTile6 + (kk & 3) * 32) / 16, idt_12, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_bf16(tm + kColS, dk + kk * 128, dv + kk * 128, idb_mm, kk > 0);
        umma_commit(&sm.mma_bar);
        ++mma_issued;
      }
      // ---- F. mask(A) -> hi / lo tiles over K~; S = diag(E) S + dS ----
      wait_mma();
      {
        float a[16];
        tmem_ld16x256b_x4(tl + kColA + 32 * ch, a);
        tmem_wait_ld();
        const float b0 = sm.bonus[r0], b1 = sm.bonus[r1];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int s0 = cq + 8 * q;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int rr = hh ? r1 : r0;
            const float bb = hh ? b1 : b0;
            // earlier tokens only (REV: the later ones), the bonus on the diagonal
            const bool k0 = REV ? s0 > rr : s0 < rr, k1 = REV ? s0 + 1 > rr : s0 + 1 < rr;
            const float x0 = k0 ? a[4 * q + 2 * hh] : (s0 == rr ? bb : 0.f);
            const float x1 = k1 ? a[4 * q + 2 * hh + 1] : (s0 + 1 == rr ? bb : 0.f);
            uint32_t ph, pl;
            split_bf16x2(x0, x1, ph, pl);
            tile_st_pair(sm.bt[0], rr, s0, ph);
            tile_st_pair(sm.bt[1], rr, s0, pl);
          }
        }
        float d[16];
        tmem_ld16x256b_x4(tl + kColS + 32 * ch, d);
        tmem_wait_ld();
        const float d0 = sm.dec[r0], d1 = sm.dec[r1];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          S[4 * q] = fmaf(d0, S[4 * q], d[4 * q]);
          S[4 * q + 1] = fmaf(d0, S[4 * q + 1], d[4 * q + 1]);
          S[4 * q + 2] = fmaf(d1, S[4 * q + 2], d[4 * q + 2]);
          S[4 * q + 3] = fmaf(d1, S[4 * q + 3], d[4 * q + 3]);
        }
        store_state();
      }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      // ---- G. MMA3 O += mask(A) V (hi and lo passes); written out next unit ----
      if (tid == 0) {
        tc_fence_after_sync();
        const uint64_t dh = umma_desc_sw128(smem_u32(sm.bt[0]), 16, 1024);
        const uint64_t dl = umma_desc_sw128(smem_u32(sm.bt[1]), 16, 1024);
        const uint64_t dv = umma_desc_sw128(vt, 8192, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_bf16(tm + kColO, dh + kk * 2, dv + kk * 128, idb_km, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_bf16(tm + kColO, dl + kk * 2, dv + kk * 128, idb_km, true);
        umma_commit(&sm.mma_bar);
        ++mma_issued;
      }
      prev = true;
      prev_t0 = t0;
      prev_lo = lo;
      prev_hi = hi;
      first_unit = false;
      off += len;
    }
  }
  if (!failed && prev) {
    wait_mma();
    epilogue();
  }
  if (!failed && __syncthreads_or(!ok)) failed = true;
  if (failed) {
    // let every copy and MMA still in flight land before the shared and
    // tensor memory are released (each wait is itself bounded)
    if (tid == 0) {
      if (w_done < w_issued) mbar_wait_bounded(&sm.w_bar, (uint32_t)(w_issued - 1) & 1u, err);
      if (rk_done < rk_issued) mbar_wait_bounded(&sm.rk_bar, (uint32_t)(rk_issued - 1) & 1u, err);
      for (int cc = v_done; cc < v_issued; ++cc) mbar_wait_bounded(&sm.v_bar[cc & 1], (uint32_t)(cc >> 1) & 1u, err);
      if (mma_done < mma_issued) mbar_wait_bounded(&sm.mma_bar, (uint32_t)(mma_issued - 1) & 1u, err);
    }
  } else if (final_state) {
    float* fs = final_state + ((int64_t)b * H + h) * kHead6 * kHead6;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      *reinterpret_cast<float2*>(fs + r0 * kHead6 + cq + 8 * q) = make_float2(S[4 * q], S[4 * q + 1]);
      *reinterpret_cast<float2*>(fs + r1 * kHead6 + cq + 8 * q) = make_float2(S[4 * q + 2], S[4 * q + 3]);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tm, kTmemCols6);
  }
}

wkv_status launch_wkv6_forward(const Wkv6FwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  CUtensorMap maps[4];
  memset(maps, 0, sizeof(maps));
  const uint64_t HK = (uint64_t)a.H * kHead6;
  if (a.T > 0) {
    const void* src[4] = {a.r, a.k, a.v, a.w};
    for (int q = 0; q < 4; ++q)
      if (!encode_tmap_3d(&maps[q], src[q], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HK, (uint64_t)a.T, (uint64_t)a.B,
                          kHead6, kChunk6, 1, why, /*swizzle128=*/true))
        return WKV_ERR_INVALID_ARG;
  }
  const size_t smem = sizeof(Wkv6Smem) + 1024;  // + room to align the base to 1024 bytes
  auto kern = a.reverse ? wkv6_fwd_chunk_kernel<true> : wkv6_fwd_chunk_kernel<false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
    *why = "wkv6_forward: shared memory configuration failed";
    return WKV_ERR_CUDA;
  }
  kern<<<(unsigned)(a.B * a.H), kThreads6, smem, stream>>>(
      maps[0], maps[1], maps[2], maps[3], (int)a.T, (int)a.H, a.u, a.init_state, a.state_map, (int)a.n_state,
      a.final_state, static_cast<__nv_bfloat16*>(a.o), a.ck_state, err);
  if (cudaGetLastError() != cudaSuccess) {
    *why = "wkv6_forward kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

}  // namespace wkv
