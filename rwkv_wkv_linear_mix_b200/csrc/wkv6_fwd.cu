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
// The 64x64x64 products run on the tensor cores (bf16 operands, fp32
// accumulators in tensor memory). A bf16 operand keeps 8 significant bits;
// where that is not enough for the 2e-2 bound the operand x is split into
// hi = bf16(x) and lo = bf16(x - hi) and the product taken in two or three
// passes (x y ~ xh yh + xl yh + xh yl), which keeps ~16 bits:
//   MMA1  A  = R^ K~^T        R^ = r * E_{j-1}, K~ = k / E_s   (3 passes)
//   MMA2  O  = R^ S_in        S_in split hi/lo                 (2 passes)
//   MMA4  dS = K^^T V         K^ = k * E_{L-1} / E_s (<= |k|)  (1 pass)
//   MMA3  O += mask(A) V      mask keeps s < j and puts the bonus on s = j,
//                             split hi/lo                      (2 passes)
// The fp32 state itself stays in registers. E is a running product of the
// decays (no logarithms, no exponentials): R^ and K^ never exceed |r|, |k|.
// K~ = k / E_s grows as the chunk decays, so a chunk whose total decay falls
// below 2^-96 in some channel is processed as sub-chunks of 16, then 4, then
// 1 token(s) (the same code with the tokens outside the sub-chunk masked:
// r = k = 0, w = 1). A single token needs no K~, so every w in (0, 1] is
// handled.
//
// Kernel shape: one CTA of 256 threads per (b, h), walking its chunks in
// order; two CTAs share an SM. TMA brings the r, k, w tiles (64 tokens x 64
// channels, 128-byte swizzled) of the next (sub)chunk as soon as the current
// one's are consumed, and the v tile of chunk c + 1 (double-buffered) while
// chunk c is processed. Warp g prepares the operands of tokens 8g .. 8g + 7
// (lane = two channels) and writes the lo halves of R^ and K~ over the r and
// k tiles it has just read; one thread issues the MMAs; accumulators are read
// back by warps 0-3 (columns 0-31) and 4-7 (columns 32-63), whose lanes 0-15
// also keep the fp32 state (32 values each). Waits are bounded (2 s): a wait
// that gives up records WKV_DEVERR_WAIT_TIMEOUT, the CTA drains its copies
// and MMAs in flight, frees its tensor memory and exits.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

constexpr int kHead6 = 64;                         // head size K = V
constexpr int kChunk6 = 64;                        // tokens per chunk
constexpr int kThreads6 = 256;                     // 8 warps
constexpr uint32_t kTile6 = 64u * 64u * 2u;        // one 64 x 64 bf16 tile
constexpr uint32_t kTmemCols6 = 256;               // A: 0-63, O: 64-127, dS: 128-191
constexpr float kMinChunkDecay6 = 1.2621774e-29f;  // 2^-96

struct alignas(1024) Wkv6Smem {
  uint8_t r[kTile6];     // r of the (sub)chunk; then lo(R^)   [j][i]
  uint8_t k[kTile6];     // k of the (sub)chunk; then lo(K~)   [s][i]
  uint8_t w[kTile6];     // w of the (sub)chunk
  uint8_t v[2][kTile6];  // v of chunks c, c + 1               [s][jv]
  uint8_t rh[kTile6];    // hi(R^)                             [j][i]
  uint8_t kb[kTile6];    // hi(K~); then hi(mask(A))           [s][i] / [j][s]
  uint8_t kh[kTile6];    // K^; then lo(mask(A))               [s][i] / [j][s]
  uint8_t sh[kTile6];    // hi(S_in)                           [i][jv]
  uint8_t sl[kTile6];    // lo(S_in)                           [i][jv]
  float u[kHead6];
  float wq[8][kHead6];  // product of w over each warp's 8 tokens
  float dec[kHead6];    // E_{L-1}: decay of the state across the (sub)chunk
  float bonus[kHead6];  // r_j . (u * k_j)
  uint64_t rkw_bar;     // r, k, w tiles landed
  uint64_t v_bar[2];    // v tiles landed
  uint64_t mma_bar;     // tensor-core completion barrier
  uint32_t tmem_base;
};

// bf16 pair (channels 2 * lane, 2 * lane + 1) of row j of a swizzled tile.
__device__ __forceinline__ uint32_t tile_ld2(const uint8_t* tile, int j, int lane) {
  return *reinterpret_cast<const uint32_t*>(tile + j * 128 + ((((lane >> 2) ^ (j & 7)) & 7) << 4) + 4 * (lane & 3));
}
__device__ __forceinline__ void tile_st2(uint8_t* tile, int j, int lane, uint32_t v) {
  *reinterpret_cast<uint32_t*>(tile + j * 128 + ((((lane >> 2) ^ (j & 7)) & 7) << 4) + 4 * (lane & 3)) = v;
}
// Columns 16 q .. 16 q + 15 (q in 0..3) of row `row`: 8 packed bf16 pairs.
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

__global__ void __launch_bounds__(kThreads6, 2)
    wkv6_fwd_chunk_kernel(const __grid_constant__ CUtensorMap tr, const __grid_constant__ CUtensorMap tk,
                          const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tw, int T, int H,
                          const float* __restrict__ u, const float* __restrict__ init_state,
                          const int32_t* __restrict__ state_map, int n_state, float* __restrict__ final_state,
                          __nv_bfloat16* __restrict__ o, unsigned* err) {
  extern __shared__ uint8_t wkv6_dsmem[];
  Wkv6Smem& sm = *reinterpret_cast<Wkv6Smem*>((reinterpret_cast<uintptr_t>(wkv6_dsmem) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x % H, b = blockIdx.x / H;
  const int64_t HK = (int64_t)H * kHead6;
  const int nch = (T + kChunk6 - 1) / kChunk6;
  // accumulator read-back: TMEM sub-partition sp, column half ch; lanes 0-15
  // hold row 16 sp + lane (a token j of A and O, a key i of dS and S)
  const int sp = warp & 3, ch = warp >> 2;
  const int row = 16 * sp + lane;
  const bool holder = lane < 16;

  if (tid == 0) {
    if (nch > 0) {
      tma_prefetch_desc(&tr);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      tma_prefetch_desc(&tw);
    }
    mbar_init(&sm.rkw_bar, 1);
    mbar_init(&sm.v_bar[0], 1);
    mbar_init(&sm.v_bar[1], 1);
    mbar_init(&sm.mma_bar, 1);
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc(&sm.tmem_base, kTmemCols6);
  if (tid < kHead6) sm.u[tid] = u[h * kHead6 + tid];

  // fp32 state S[row][32 ch .. 32 ch + 31] in registers; hi/lo copy in sh, sl
  float S[32];
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
    for (int e = 0; e < 32; e += 4) {
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (s0 && holder) x = *reinterpret_cast<const float4*>(s0 + row * kHead6 + 32 * ch + e);
      S[e] = x.x;
      S[e + 1] = x.y;
      S[e + 2] = x.z;
      S[e + 3] = x.w;
    }
    if (holder) {
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t ph[8], pl[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) split_bf16x2(S[16 * q + e], S[16 * q + e + 1], ph[e / 2], pl[e / 2]);
        tile_st_row16(sm.sh, row, 2 * ch + q, ph);
        tile_st_row16(sm.sl, row, 2 * ch + q, pl);
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tm = sm.tmem_base;
  const uint32_t tl = tm + ((uint32_t)(32 * sp) << 16);  // this warp's TMEM lanes

  // copies in flight, as seen by thread 0 (the only thread that issues them)
  int rkw_issued = 0, rkw_done = 0, v_issued = 0, v_done = 0;
  auto load_rkw = [&](int cc) {
    mbar_arrive_expect_tx(&sm.rkw_bar, 3 * kTile6);
    tma_load_3d(sm.r, &tr, &sm.rkw_bar, h * kHead6, cc * kChunk6, b);
    tma_load_3d(sm.k, &tk, &sm.rkw_bar, h * kHead6, cc * kChunk6, b);
    tma_load_3d(sm.w, &tw, &sm.rkw_bar, h * kHead6, cc * kChunk6, b);
    ++rkw_issued;
  };
  auto load_v = [&](int cc) {
    mbar_arrive_expect_tx(&sm.v_bar[cc & 1], kTile6);
    tma_load_3d(sm.v[cc & 1], &tv, &sm.v_bar[cc & 1], h * kHead6, cc * kChunk6, b);
    ++v_issued;
  };
  if (tid == 0 && nch > 0) {
    load_rkw(0);
    load_v(0);
  }

  constexpr uint32_t id_kk = umma_idesc_bf16(64, 64, 0, 0);  // A K-major, B K-major
  constexpr uint32_t id_km = umma_idesc_bf16(64, 64, 0, 1);  // A K-major, B MN-major
  constexpr uint32_t id_mm = umma_idesc_bf16(64, 64, 1, 1);  // A MN-major, B MN-major
  uint32_t rkw_phase = 0, mma_phase = 0;
  bool mma_pending = false;  // (thread 0) an MMA commit not yet confirmed complete
  bool ok = true, failed = false;
  bool wait_rkw = true;  // the next (sub)chunk's r, k, w tiles are still loading
  for (int c = 0; c < nch && !failed; ++c) {
    const int t0 = c * kChunk6;
    const int valid = min(kChunk6, T - t0);
    const uint32_t vt = smem_u32(sm.v[c & 1]);
    if (tid == 0 && c + 1 < nch) load_v(c + 1);
    bool v_ready = false;
    int off = 0, size = kChunk6;
    while (off < valid) {
      if (wait_rkw) {
        const bool got = mbar_wait_bounded(&sm.rkw_bar, rkw_phase, err);
        if (tid == 0 && got) rkw_done = rkw_issued;
        ok = got && ok;
        rkw_phase ^= 1u;
        wait_rkw = false;
      }
      const int len = min(size, valid - off);
      // ---- pass 1: product of w over this warp's 8 tokens (w = 1 outside) ----
      float w0[8], w1[8];
      float p0 = 1.f, p1 = 1.f;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const int j = 8 * warp + jj;
        const bool in = j >= off && j < off + len;
        const uint32_t x = tile_ld2(sm.w, j, lane);
        w0[jj] = in ? bf16lo(x) : 1.f;
        w1[jj] = in ? bf16hi(x) : 1.f;
        p0 *= w0[jj];
        p1 *= w1[jj];
      }
      sm.wq[warp][2 * lane] = p0;
      sm.wq[warp][2 * lane + 1] = p1;
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      float pre0 = 1.f, pre1 = 1.f, post0 = 1.f, post1 = 1.f, tot0 = 1.f, tot1 = 1.f;
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const float2 q = *reinterpret_cast<const float2*>(&sm.wq[g][2 * lane]);
        if (g < warp) {
          pre0 *= q.x;
          pre1 *= q.y;
        }
        if (g > warp) {
          post0 *= q.x;
          post1 *= q.y;
        }
        tot0 *= q.x;
        tot1 *= q.y;
      }
      // a chunk that decays below 2^-96 is split (K~ = k / E could overflow);
      // nothing has been written yet, so the tiles are still intact
      const bool deep = !(tot0 >= kMinChunkDecay6 && tot1 >= kMinChunkDecay6);
      if (__syncthreads_or(deep) && size > 1) {
        size >>= 2;
        continue;
      }
      if (warp == 0) {
        sm.dec[2 * lane] = tot0;
        sm.dec[2 * lane + 1] = tot1;
      }
      // ---- bonus r_j . (u * k_j): the four lanes 4m .. 4m + 3 of warp g take
      // token 8g + m, 16 channels each (rows this warp owns) ----
      {
        const int j = tid >> 2, part = tid & 3;
        float acc = 0.f;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int chunk = 2 * part + cc;
          const int phys = (chunk ^ (j & 7)) & 7;
          const uint4 rv = *reinterpret_cast<const uint4*>(sm.r + j * 128 + phys * 16);
          const uint4 kv = *reinterpret_cast<const uint4*>(sm.k + j * 128 + phys * 16);
          const uint32_t rr[4] = {rv.x, rv.y, rv.z, rv.w}, kk[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int i = chunk * 8 + 2 * q;
            acc = fmaf(bf16lo(rr[q]) * sm.u[i], bf16lo(kk[q]), acc);
            acc = fmaf(bf16hi(rr[q]) * sm.u[i + 1], bf16hi(kk[q]), acc);
          }
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        if (part == 0) sm.bonus[j] = (j >= off && j < off + len) ? acc : 0.f;
      }
      __syncwarp();
      // ---- pass 2: K^ (suffix products, backwards); then R^ and K~ with
      // their lo halves written over the r and k rows just read ----
      {
        float g0 = post0, g1 = post1;
#pragma unroll
        for (int jj = 7; jj >= 0; --jj) {
          const int j = 8 * warp + jj;
          const bool in = j >= off && j < off + len;
          const uint32_t kx = tile_ld2(sm.k, j, lane);
          tile_st2(sm.kh, j, lane, in ? pack_bf16x2(bf16lo(kx) * g0, bf16hi(kx) * g1) : 0u);
          g0 *= w0[jj];
          g1 *= w1[jj];
        }
        float e0 = pre0, e1 = pre1;
        const bool need_kb = len > 1;  // one token has no s < j pair
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int j = 8 * warp + jj;
          const bool in = j >= off && j < off + len;
          const uint32_t rx = tile_ld2(sm.r, j, lane), kx = tile_ld2(sm.k, j, lane);
          uint32_t rh, rl, kbh, kbl;
          split_bf16x2(bf16lo(rx) * e0, bf16hi(rx) * e1, rh, rl);
          e0 *= w0[jj];
          e1 *= w1[jj];
          split_bf16x2(bf16lo(kx) * rcp(e0), bf16hi(kx) * rcp(e1), kbh, kbl);
          const bool kin = in && need_kb;
          tile_st2(sm.rh, j, lane, in ? rh : 0u);
          tile_st2(sm.r, j, lane, in ? rl : 0u);
          tile_st2(sm.kb, j, lane, kin ? kbh : 0u);
          tile_st2(sm.k, j, lane, kin ? kbl : 0u);
        }
      }
      if (!v_ready) {
        ok = mbar_wait_bounded(&sm.v_bar[c & 1], (c >> 1) & 1, err) && ok;
        if (tid == 0 && ok) v_done = c + 1;
        v_ready = true;
      }
      fence_proxy_async_smem();
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      // ---- MMA1 A = R^ K~^T, MMA2 O = R^ S_in, MMA4 dS = K^^T V ----
      if (tid == 0) {
        tc_fence_after_sync();
        const uint32_t rh = smem_u32(sm.rh), rl = smem_u32(sm.r), kbh = smem_u32(sm.kb), kbl = smem_u32(sm.k);
        const uint32_t kh = smem_u32(sm.kh), sh = smem_u32(sm.sh), sl = smem_u32(sm.sl);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_bf16(tm + 0, umma_kmajor(rh, kk), umma_kmajor(kbh, kk), id_kk, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_bf16(tm + 0, umma_kmajor(rl, kk), umma_kmajor(kbh, kk), id_kk, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_bf16(tm + 0, umma_kmajor(rh, kk), umma_kmajor(kbl, kk), id_kk, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_bf16(tm + 64, umma_kmajor(rh, kk), umma_mnmajor(sh, kk), id_km, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_bf16(tm + 64, umma_kmajor(rh, kk), umma_mnmajor(sl, kk), id_km, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_bf16(tm + 128, umma_mnmajor(kh, kk), umma_mnmajor(vt, kk), id_mm, kk > 0);
        umma_commit(&sm.mma_bar);
        mma_pending = true;
      }
      {
        const bool got = mbar_wait_bounded(&sm.mma_bar, mma_phase, err);
        if (tid == 0 && got) mma_pending = false;
        ok = got && ok;
        mma_phase ^= 1u;
      }
      tc_fence_after_sync();
      // r, k, w tiles are free: bring those of the next (sub)chunk
      if (tid == 0 && ok) {
        const int next = off + len < valid ? c : c + 1;
        if (next < nch) load_rkw(next);
      }
      wait_rkw = true;
      // ---- mask(A) split hi/lo into kb, kh; S = diag(E) S + dS into sh, sl ----
      {
        const float bj = holder ? sm.bonus[row] : 0.f;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float a[16];
          tmem_ld16(tl + 0 + 32 * ch + 16 * q, a);
          tmem_wait_ld();
          if (holder) {
            uint32_t ph[8], pl[8];
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              const int s = 32 * ch + 16 * q + e;
              const float a0 = s < row ? a[e] : (s == row ? bj : 0.f);
              const float a1 = s + 1 < row ? a[e + 1] : (s + 1 == row ? bj : 0.f);
              split_bf16x2(a0, a1, ph[e / 2], pl[e / 2]);
            }
            tile_st_row16(sm.kb, row, 2 * ch + q, ph);
            tile_st_row16(sm.kh, row, 2 * ch + q, pl);
          }
        }
        const float dj = holder ? sm.dec[row] : 0.f;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float d[16];
          tmem_ld16(tl + 128 + 32 * ch + 16 * q, d);
          tmem_wait_ld();
          if (holder) {
            uint32_t ph[8], pl[8];
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              float& s0 = S[16 * q + e];
              float& s1 = S[16 * q + e + 1];
              s0 = fmaf(dj, s0, d[e]);
              s1 = fmaf(dj, s1, d[e + 1]);
              split_bf16x2(s0, s1, ph[e / 2], pl[e / 2]);
            }
            tile_st_row16(sm.sh, row, 2 * ch + q, ph);
            tile_st_row16(sm.sl, row, 2 * ch + q, pl);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      // ---- MMA3 O += mask(A) V ----
      if (tid == 0) {
        tc_fence_after_sync();
        const uint32_t amh = smem_u32(sm.kb), aml = smem_u32(sm.kh);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_bf16(tm + 64, umma_kmajor(amh, kk), umma_mnmajor(vt, kk), id_km, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_bf16(tm + 64, umma_kmajor(aml, kk), umma_mnmajor(vt, kk), id_km, true);
        umma_commit(&sm.mma_bar);
        mma_pending = true;
      }
      {
        const bool got = mbar_wait_bounded(&sm.mma_bar, mma_phase, err);
        if (tid == 0 && got) mma_pending = false;
        ok = got && ok;
        mma_phase ^= 1u;
      }
      tc_fence_after_sync();
      // ---- epilogue: this (sub)chunk's rows of o ----
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float ov[16];
        tmem_ld16(tl + 64 + 32 * ch + 16 * q, ov);
        tmem_wait_ld();
        if (ok && holder && row >= off && row < off + len) {
          uint32_t p[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) p[e / 2] = pack_bf16x2(ov[e], ov[e + 1]);
          uint4* dst = reinterpret_cast<uint4*>(o + ((int64_t)b * T + t0 + row) * HK + h * kHead6 + 32 * ch + 16 * q);
          dst[0] = make_uint4(p[0], p[1], p[2], p[3]);
          dst[1] = make_uint4(p[4], p[5], p[6], p[7]);
        }
      }
      tc_fence_before_sync();
      off += len;
    }
  }
  if (!failed && __syncthreads_or(!ok)) failed = true;
  if (failed) {
    // let every copy and MMA still in flight land before the shared and
    // tensor memory are released (each wait is itself bounded)
    if (tid == 0) {
      if (rkw_done < rkw_issued) mbar_wait_bounded(&sm.rkw_bar, (uint32_t)(rkw_issued - 1) & 1u, err);
      for (int cc = v_done; cc < v_issued; ++cc) mbar_wait_bounded(&sm.v_bar[cc & 1], (uint32_t)(cc >> 1) & 1u, err);
      if (mma_pending) mbar_wait_bounded(&sm.mma_bar, mma_phase ^ 1u, err);
    }
  } else if (final_state && holder) {
    float* fs = final_state + ((int64_t)b * H + h) * kHead6 * kHead6 + row * kHead6 + 32 * ch;
#pragma unroll
    for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(fs + e) = make_float4(S[e], S[e + 1], S[e + 2], S[e + 3]);
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
  if (cudaFuncSetAttribute(wkv6_fwd_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess) {
    *why = "wkv6_forward: shared memory configuration failed";
    return WKV_ERR_CUDA;
  }
  wkv6_fwd_chunk_kernel<<<(unsigned)(a.B * a.H), kThreads6, smem, stream>>>(
      maps[0], maps[1], maps[2], maps[3], (int)a.T, (int)a.H, a.u, a.init_state, a.state_map, (int)a.n_state,
      a.final_state, static_cast<__nv_bfloat16*>(a.o), err);
  if (cudaGetLastError() != cudaSuccess) {
    *why = "wkv6_forward kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

}  // namespace wkv
