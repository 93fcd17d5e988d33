// wkv6_bwd.cu -- RWKV-6 head-state WKV backward on sm_100a.
//
// Gradients of L = sum(dout * o) + sum(g_final * S_final) for the forward of
// wkv6_fwd.cu (RWKV6_OP on the rwkv-ops package page; the operator is
// trained, and its PyTorch CUDA implementation is listed there), per head
// with K = 64 (S indexed [i][j], i the key index, j the value index):
//   S_t = diag(w_t) S_{t-1} + k_t^T v_t,   o_t = r_t (S_{t-1} + diag(u) k_t^T v_t)
// With G_t = dL/dS_t (G_{T-1} = g_final):
//   G_{t-1} = diag(w_t) G_t + r_t^T do_t
//   gr_t = S_{t-1} do_t + u o k_t (v_t . do_t)
//   gk_t = G_t v_t + u o r_t (v_t . do_t)
//   gv_t = k_t G_t + (r_t . (u o k_t)) do_t
//   gu   = sum_t r_t o k_t (v_t . do_t)
// and for the decay, with P_t[i] = sum_j G_t[i][j] S_t[i][j]:
//   w_t o gw_t = P_t - k_t o (G_t v_t)
//   P_{t-1}    = P_t - k_t o (G_t v_t) + r_t o (S_{t-1} do_t)
// (expand S_t and G_{t-1} by their recurrences). These give the gradient
// with respect to log w without S_{t-1} and G_t at the same step: P starts
// from sum_j g_final S_final and walks down on two row products the passes
// form anyway. The kernel returns glogw = w o gw (what w = exp(-exp(d))
// consumes: dL/dd = -exp(d) glogw); it stays accurate where w_t is tiny,
// where gw itself would be a difference of large terms divided by w_t.
//
// Two passes, one CTA of 128 threads per (b, h); thread (p = tid / 4,
// q = tid % 4) holds rows 2p and 2p + 1, columns 16q .. 16q + 15 (each slice
// of a token's vectors it reads serves two rows):
//   pass 1 (t up):   S; writes gr and, per token, x_t = r_t o (S_{t-1} do_t)
//                    and (c_t = r_t . (u o k_t), v_t . do_t) to the workspace;
//                    at the end P_{T-1} = sum_j g_final S_{T-1}.
//   pass 2 (t down): G in two copies, by rows (G v, the P walk, g_init) and
//                    by columns 2p, 2p + 1 (rows 16q ..: k G becomes a row
//                    product as well, so no 64-way reduction across
//                    threads); writes gk, gv, glogw and per-(b, h) gu
//                    partials.
// Inputs arrive per 32-token chunk by TMA into two stages (the next chunk
// loads while this one runs). Each step reads its 16-wide slices as bf16 (32
// bytes per vector) one step ahead of use and widens them in registers.
// Outputs leave through shared-memory tiles as coalesced 16-byte stores. The
// 16-wide row work runs on packed fp32 pairs. gu is summed over samples by a
// fixed-order reduction.
#include <string.h>

#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

constexpr int kK6b = 64;       // head size
constexpr int kL6b = 32;       // tokens per chunk
constexpr int kT6b = 128;      // threads per CTA (2 rows per thread)
constexpr int kIn6b = 5;       // r, k, v, w, do
enum { kR = 0, kKk = 1, kV = 2, kW = 3, kDo = 4 };

struct alignas(128) Wkv6Bwd1Smem {
  __nv_bfloat16 in[2][kIn6b][kL6b][kK6b];  // two TMA stages
  float cv[2][kL6b][4];                    // per stage and token: c_t, v_t . do_t
  float xo[kL6b][kK6b];                    // x_t rows for the workspace
  __nv_bfloat16 gro[kL6b][kK6b];           // gr tile
  uint64_t full[2];
};

struct alignas(128) Wkv6Bwd2Stage {
  __nv_bfloat16 in[kIn6b][kL6b][kK6b];
  float x[kL6b][kK6b];   // x_t rows
  float cv[kL6b][4];     // (c_t, v_t . do_t, -, -)
};

struct alignas(128) Wkv6Bwd2Smem {
  Wkv6Bwd2Stage st[2];                  // two TMA stages
  __nv_bfloat16 out[3][kL6b][kK6b];     // gk, gv, glogw tiles
  uint64_t full[2];
};

// 16 consecutive bf16 of shared memory (two 16-byte loads), and their
// widening to 8 fp32 pairs (element 2m in the low half of word m).
struct Bf16x16 {
  uint4 a, b;
};
__device__ __forceinline__ Bf16x16 ld16b(const __nv_bfloat16* p) {
  const uint4* p4 = reinterpret_cast<const uint4*>(p);
  return {p4[0], p4[1]};
}
__device__ __forceinline__ void widen16(const Bf16x16& x, float2 (&y)[8]) {
  const uint32_t wds[8] = {x.a.x, x.a.y, x.a.z, x.a.w, x.b.x, x.b.y, x.b.z, x.b.w};
#pragma unroll
  for (int m = 0; m < 8; ++m) y[m] = make_float2(bf16lo(wds[m]), bf16hi(wds[m]));
}
__device__ __forceinline__ float bf(const __nv_bfloat16& x) { return __bfloat162float(x); }

// 16 consecutive fp32 of global memory as 8 pairs.
__device__ __forceinline__ void ld16(const float* p, float2 (&x)[8]) {
  const float4* p4 = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const float4 a = p4[m];
    x[2 * m] = make_float2(a.x, a.y);
    x[2 * m + 1] = make_float2(a.z, a.w);
  }
}

// Sum over the 4 threads of a row (lanes 4m .. 4m + 3).
__device__ __forceinline__ float row_sum4(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

__device__ __forceinline__ float dot16(const float2 (&a)[8], const float2 (&b)[8]) {
  float2 s0 = make_float2(0.f, 0.f), s1 = s0;
#pragma unroll
  for (int m = 0; m < 8; m += 2) {
    s0 = fma2(a[m], b[m], s0);
    s1 = fma2(a[m + 1], b[m + 1], s1);
  }
  const float2 s = add2(s0, s1);
  return __fadd_rn(s.x, s.y);
}

// Two adjacent bf16 of shared memory as a pair.
__device__ __forceinline__ float2 ld2b(const __nv_bfloat16* p) {
  const uint32_t x = *reinterpret_cast<const uint32_t*>(p);
  return make_float2(bf16lo(x), bf16hi(x));
}

// Store a [kL6b][kK6b] bf16 tile to rows t0 .. t0 + n - 1 of a [B][T][HK]
// tensor at column h * 64 (16-byte pieces).
__device__ __forceinline__ void wkv6_store_tile(const __nv_bfloat16 (*tile)[kK6b], __nv_bfloat16* dst, int b, int T,
                                                int HK, int h, int t0, int n, int tid) {
  for (int g = tid; g < kL6b * 8; g += kT6b) {
    const int row = g / 8, piece = g % 8;
    if (row < n) {
      const uint4 val = reinterpret_cast<const uint4*>(&tile[row][0])[piece];
      *reinterpret_cast<uint4*>(dst + ((int64_t)b * T + t0 + row) * HK + (int64_t)h * kK6b + piece * 8) = val;
    }
  }
}

__global__ void __launch_bounds__(kT6b, 2) wkv6_bwd_pass1_kernel(
    const __grid_constant__ CUtensorMap tr, const __grid_constant__ CUtensorMap tk,
    const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tw,
    const __grid_constant__ CUtensorMap tdo, int T, int H, const float* __restrict__ u,
    const float* __restrict__ init_state, const int32_t* __restrict__ state_map, int n_state,
    const float* __restrict__ g_final, __nv_bfloat16* __restrict__ gr, float* __restrict__ xws,
    float* __restrict__ cvws, float* __restrict__ p0, unsigned* err) {
  extern __shared__ __align__(128) unsigned char wkv6_bwd1_dsmem[];
  Wkv6Bwd1Smem& sm = *reinterpret_cast<Wkv6Bwd1Smem*>(wkv6_bwd1_dsmem);
  const int tid = threadIdx.x, q = tid & 3, i0 = 2 * (tid >> 2);  // rows i0, i0 + 1
  const int bh = (int)blockIdx.x, b = bh / H, h = bh % H;
  const int HK = H * kK6b;
  const int nchunk = (T + kL6b - 1) / kL6b;
  constexpr uint32_t kStageBytes = kIn6b * kL6b * kK6b * sizeof(__nv_bfloat16);
  const CUtensorMap* maps[kIn6b] = {&tr, &tk, &tv, &tw, &tdo};
  auto issue = [&](int ch) {
    const int s = ch & 1;
    mbar_arrive_expect_tx(&sm.full[s], kStageBytes);
    for (int m = 0; m < kIn6b; ++m) tma_load_3d(&sm.in[s][m][0][0], maps[m], &sm.full[s], h * kK6b, ch * kL6b, b);
  };
  if (tid == 0) {
    mbar_init(&sm.full[0], 1);
    mbar_init(&sm.full[1], 1);
    mbar_init_fence();
    if (nchunk > 0)
      for (int m = 0; m < kIn6b; ++m) tma_prefetch_desc(maps[m]);
    for (int ch = 0; ch < 2 && ch < nchunk; ++ch) issue(ch);
  }
  // S_{-1}: init_state[state_map[b]] (or the n_state rule), else zero
  float2 S0[8], S1[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) S0[m] = S1[m] = make_float2(0.f, 0.f);
  if (init_state) {
    const int sidx = state_map ? state_map[b] : (n_state == 1 ? 0 : b);
    if (sidx < 0 || sidx >= n_state) {
      if (tid == 0) record_error(err, WKV_DEVERR_BAD_STATE);
    } else {
      const float* base = init_state + (((int64_t)sidx * H + h) * kK6b + i0) * kK6b + 16 * q;
      ld16(base, S0);
      ld16(base + kK6b, S1);
    }
  }
  const float2 uu = make_float2(u[h * kK6b + i0], u[h * kK6b + i0 + 1]);
  __syncthreads();

  bool ok = true;
  int ch = 0;
  for (; ch < nchunk; ++ch) {
    const int s = ch & 1;
    const int t0 = ch * kL6b, n = min(kL6b, T - t0);
    const bool got = mbar_wait_bounded(&sm.full[s], (ch >> 1) & 1, err);
    if (!__syncthreads_and(got)) {
      ok = false;
      break;
    }
    const __nv_bfloat16(*in)[kL6b][kK6b] = sm.in[s];
    {
      // per token: c_t = r . (u o k) and v . do, 4 threads per token
      const int jt = tid >> 2, part = tid & 3;
      float c = 0.f, vd = 0.f;
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        const int e = part * 16 + m;
        c = __fmaf_rn(bf(in[kR][jt][e]) * u[h * kK6b + e], bf(in[kKk][jt][e]), c);
        vd = __fmaf_rn(bf(in[kV][jt][e]), bf(in[kDo][jt][e]), vd);
      }
      c = row_sum4(c);
      vd = row_sum4(vd);
      if (part == 0) reinterpret_cast<float4*>(&sm.cv[s][jt][0])[0] = make_float4(c, vd, 0.f, 0.f);
    }
    __syncthreads();
    // the step's vectors are fetched one step ahead
    Bf16x16 vn = ld16b(&in[kV][0][16 * q]), dn = ld16b(&in[kDo][0][16 * q]);
    float2 wn = ld2b(&in[kW][0][i0]), kn = ld2b(&in[kKk][0][i0]), rn = ld2b(&in[kR][0][i0]);
    float vdn = sm.cv[s][0][1];
    for (int jt = 0; jt < n; ++jt) {
      const Bf16x16 vc = vn, dc = dn;
      const float2 w2 = wn, k2 = kn, r2 = rn;
      const float vdo = vdn;
      if (jt + 1 < n) {
        vn = ld16b(&in[kV][jt + 1][16 * q]);
        dn = ld16b(&in[kDo][jt + 1][16 * q]);
        wn = ld2b(&in[kW][jt + 1][i0]);
        kn = ld2b(&in[kKk][jt + 1][i0]);
        rn = ld2b(&in[kR][jt + 1][i0]);
        vdn = sm.cv[s][jt + 1][1];
      }
      float2 vv[8], dd[8];
      widen16(vc, vv);
      widen16(dc, dd);
      // (S_{t-1} do_t) for both rows
      const float a0 = row_sum4(dot16(S0, dd)), a1 = row_sum4(dot16(S1, dd));
      if (q == 0) {
        *reinterpret_cast<__nv_bfloat162*>(&sm.gro[jt][i0]) =
            __floats2bfloat162_rn(__fmaf_rn(uu.x * k2.x, vdo, a0), __fmaf_rn(uu.y * k2.y, vdo, a1));
        *reinterpret_cast<float2*>(&sm.xo[jt][i0]) = make_float2(__fmul_rn(r2.x, a0), __fmul_rn(r2.y, a1));
      }
      const float2 wa = make_float2(w2.x, w2.x), ka = make_float2(k2.x, k2.x);
      const float2 wb = make_float2(w2.y, w2.y), kb = make_float2(k2.y, k2.y);
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        S0[m] = fma2(S0[m], wa, mul2(ka, vv[m]));
        S1[m] = fma2(S1[m], wb, mul2(kb, vv[m]));
      }
    }
    __syncthreads();
    if (tid == 0 && ch + 2 < nchunk) issue(ch + 2);  // every read of stage s is done
    wkv6_store_tile(sm.gro, gr, b, T, HK, h, t0, n, tid);
    float* xrow = xws + ((int64_t)bh * T + t0) * kK6b;
    for (int g = tid; g < kL6b * kK6b / 4; g += kT6b) {
      const int row = g / (kK6b / 4);
      if (row < n) reinterpret_cast<float4*>(xrow)[g] = reinterpret_cast<const float4*>(&sm.xo[0][0])[g];
    }
    if (tid < n) reinterpret_cast<float4*>(cvws + ((int64_t)bh * T + t0) * 4)[tid] =
        reinterpret_cast<const float4*>(&sm.cv[s][0][0])[tid];
  }
  if (!ok) {
    // a wait gave up: let the copies in flight land before the CTA exits
    if (tid == 0)
      for (int x = ch; x < nchunk && x < ch + 2; ++x) mbar_wait_bounded(&sm.full[x & 1], (x >> 1) & 1, err);
    return;
  }
  // P_{T-1}[i] = sum_j g_final[i][j] S_{T-1}[i][j]
  float p0a = 0.f, p0b = 0.f;
  if (g_final) {
    float2 gf[8];
    const float* base = g_final + ((int64_t)bh * kK6b + i0) * kK6b + 16 * q;
    ld16(base, gf);
    p0a = dot16(gf, S0);
    ld16(base + kK6b, gf);
    p0b = dot16(gf, S1);
  }
  p0a = row_sum4(p0a);
  p0b = row_sum4(p0b);
  if (q == 0) *reinterpret_cast<float2*>(&p0[(int64_t)bh * kK6b + i0]) = make_float2(p0a, p0b);
}

__global__ void __launch_bounds__(kT6b, 2) wkv6_bwd_pass2_kernel(
    const __grid_constant__ CUtensorMap tr, const __grid_constant__ CUtensorMap tk,
    const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tw,
    const __grid_constant__ CUtensorMap tdo, const __grid_constant__ CUtensorMap tx,
    const __grid_constant__ CUtensorMap tcv, int T, int H, const float* __restrict__ u,
    const float* __restrict__ g_final, const float* __restrict__ p0, __nv_bfloat16* __restrict__ gk,
    __nv_bfloat16* __restrict__ gv, __nv_bfloat16* __restrict__ glogw, float* __restrict__ g_init,
    float* __restrict__ gu_part, unsigned* err) {
  extern __shared__ __align__(128) unsigned char wkv6_bwd2_dsmem[];
  Wkv6Bwd2Smem& sm = *reinterpret_cast<Wkv6Bwd2Smem*>(wkv6_bwd2_dsmem);
  // rows i0, i0 + 1 of G and columns i0, i0 + 1 of G (rows 16q .. 16q + 15)
  const int tid = threadIdx.x, q = tid & 3, i0 = 2 * (tid >> 2);
  const int bh = (int)blockIdx.x, b = bh / H, h = bh % H;
  const int HK = H * kK6b;
  const int nchunk = (T + kL6b - 1) / kL6b;
  constexpr uint32_t kStageBytes =
      kIn6b * kL6b * kK6b * sizeof(__nv_bfloat16) + kL6b * kK6b * sizeof(float) + kL6b * 4 * sizeof(float);
  const CUtensorMap* maps[kIn6b] = {&tr, &tk, &tv, &tw, &tdo};
  auto issue = [&](int ch) {  // ch counts chunks from the end
    const int s = ch & 1;
    const int t0 = (nchunk - 1 - ch) * kL6b;
    mbar_arrive_expect_tx(&sm.full[s], kStageBytes);
    for (int m = 0; m < kIn6b; ++m) tma_load_3d(&sm.st[s].in[m][0][0], maps[m], &sm.full[s], h * kK6b, t0, b);
    tma_load_3d(&sm.st[s].x[0][0], &tx, &sm.full[s], 0, t0, bh);
    tma_load_3d(&sm.st[s].cv[0][0], &tcv, &sm.full[s], 0, t0, bh);
  };
  if (tid == 0) {
    mbar_init(&sm.full[0], 1);
    mbar_init(&sm.full[1], 1);
    mbar_init_fence();
    if (nchunk > 0) {
      for (int m = 0; m < kIn6b; ++m) tma_prefetch_desc(maps[m]);
      tma_prefetch_desc(&tx);
      tma_prefetch_desc(&tcv);
    }
    for (int ch = 0; ch < 2 && ch < nchunk; ++ch) issue(ch);
  }
  // G_{T-1} = g_final, by rows (G[i][16q ..]) and by columns (G[16q ..][i])
  float2 G0[8], G1[8], C0[8], C1[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) G0[m] = G1[m] = C0[m] = C1[m] = make_float2(0.f, 0.f);
  if (g_final) {
    const float* gf = g_final + (int64_t)bh * kK6b * kK6b;
    ld16(gf + i0 * kK6b + 16 * q, G0);
    ld16(gf + (i0 + 1) * kK6b + 16 * q, G1);
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const float2 top = *reinterpret_cast<const float2*>(gf + (16 * q + 2 * m) * kK6b + i0);
      const float2 bot = *reinterpret_cast<const float2*>(gf + (16 * q + 2 * m + 1) * kK6b + i0);
      C0[m] = make_float2(top.x, bot.x);
      C1[m] = make_float2(top.y, bot.y);
    }
  }
  float2 P = *reinterpret_cast<const float2*>(&p0[(int64_t)bh * kK6b + i0]);
  const float2 uu = make_float2(u[h * kK6b + i0], u[h * kK6b + i0 + 1]);
  float2 gu2 = make_float2(0.f, 0.f);
  __syncthreads();

  bool ok = true;
  int ch = 0;
  for (; ch < nchunk; ++ch) {
    const int s = ch & 1;
    const int t0 = (nchunk - 1 - ch) * kL6b, n = min(kL6b, T - t0);
    const bool got = mbar_wait_bounded(&sm.full[s], (ch >> 1) & 1, err);
    if (!__syncthreads_and(got)) {
      ok = false;
      break;
    }
    const Wkv6Bwd2Stage& st = sm.st[s];
    struct Tok {
      Bf16x16 v, d, r, k, w;
      float2 w2, r2, k2, d2, cvd, x2;
    };
    auto fetch = [&](int jt) {
      Tok x;
      x.v = ld16b(&st.in[kV][jt][16 * q]);
      x.d = ld16b(&st.in[kDo][jt][16 * q]);
      x.r = ld16b(&st.in[kR][jt][16 * q]);
      x.k = ld16b(&st.in[kKk][jt][16 * q]);
      x.w = ld16b(&st.in[kW][jt][16 * q]);
      x.w2 = ld2b(&st.in[kW][jt][i0]);
      x.r2 = ld2b(&st.in[kR][jt][i0]);
      x.k2 = ld2b(&st.in[kKk][jt][i0]);
      x.d2 = ld2b(&st.in[kDo][jt][i0]);
      x.cvd = *reinterpret_cast<const float2*>(&st.cv[jt][0]);  // (c_t, v_t . do_t)
      x.x2 = *reinterpret_cast<const float2*>(&st.x[jt][i0]);
      return x;
    };
    Tok nx = fetch(n - 1);
    for (int jt = n - 1; jt >= 0; --jt) {
      const Tok cu = nx;
      if (jt > 0) nx = fetch(jt - 1);
      float2 vv[8], dd[8], rr[8], kk[8], ww[8];
      widen16(cu.v, vv);
      widen16(cu.d, dd);
      widen16(cu.r, rr);
      widen16(cu.k, kk);
      widen16(cu.w, ww);
      // (G_t v_t) for rows i0, i0 + 1 and (k_t G_t) for columns i0, i0 + 1
      const float g0 = row_sum4(dot16(G0, vv)), g1 = row_sum4(dot16(G1, vv));
      const float h0 = row_sum4(dot16(kk, C0)), h1 = row_sum4(dot16(kk, C1));
      const float c = cu.cvd.x, vdo = cu.cvd.y;
      const float2 gl = make_float2(__fsub_rn(P.x, __fmul_rn(cu.k2.x, g0)), __fsub_rn(P.y, __fmul_rn(cu.k2.y, g1)));
      P = add2(gl, cu.x2);  // P_{t-1}
      if (q == 0) {
        *reinterpret_cast<__nv_bfloat162*>(&sm.out[0][jt][i0]) =
            __floats2bfloat162_rn(__fmaf_rn(uu.x * cu.r2.x, vdo, g0), __fmaf_rn(uu.y * cu.r2.y, vdo, g1));
        *reinterpret_cast<__nv_bfloat162*>(&sm.out[1][jt][i0]) =
            __floats2bfloat162_rn(__fmaf_rn(c, cu.d2.x, h0), __fmaf_rn(c, cu.d2.y, h1));
        *reinterpret_cast<__nv_bfloat162*>(&sm.out[2][jt][i0]) = __floats2bfloat162_rn(gl.x, gl.y);
      }
      gu2 = fma2(mul2(cu.r2, cu.k2), make_float2(vdo, vdo), gu2);
      const float2 wa = make_float2(cu.w2.x, cu.w2.x), ra = make_float2(cu.r2.x, cu.r2.x);
      const float2 wb = make_float2(cu.w2.y, cu.w2.y), rb = make_float2(cu.r2.y, cu.r2.y);
      const float2 da = make_float2(cu.d2.x, cu.d2.x), db = make_float2(cu.d2.y, cu.d2.y);
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        G0[m] = fma2(G0[m], wa, mul2(ra, dd[m]));
        G1[m] = fma2(G1[m], wb, mul2(rb, dd[m]));
        C0[m] = fma2(C0[m], ww[m], mul2(rr[m], da));
        C1[m] = fma2(C1[m], ww[m], mul2(rr[m], db));
      }
    }
    __syncthreads();
    if (tid == 0 && ch + 2 < nchunk) issue(ch + 2);  // every read of stage s is done
    wkv6_store_tile(sm.out[0], gk, b, T, HK, h, t0, n, tid);
    wkv6_store_tile(sm.out[1], gv, b, T, HK, h, t0, n, tid);
    wkv6_store_tile(sm.out[2], glogw, b, T, HK, h, t0, n, tid);
  }
  if (!ok) {
    if (tid == 0)
      for (int x = ch; x < nchunk && x < ch + 2; ++x) mbar_wait_bounded(&sm.full[x & 1], (x >> 1) & 1, err);
    return;
  }
  if (g_init) {
    float* base = g_init + ((int64_t)bh * kK6b + i0) * kK6b + 16 * q;
    float4* d0 = reinterpret_cast<float4*>(base);
    float4* d1 = reinterpret_cast<float4*>(base + kK6b);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      d0[m] = make_float4(G0[2 * m].x, G0[2 * m].y, G0[2 * m + 1].x, G0[2 * m + 1].y);
      d1[m] = make_float4(G1[2 * m].x, G1[2 * m].y, G1[2 * m + 1].x, G1[2 * m + 1].y);
    }
  }
  if (q == 0) *reinterpret_cast<float2*>(&gu_part[(int64_t)bh * kK6b + i0]) = gu2;
}

// gu[c] = sum over samples b (ascending) of gu_part[b][c]: fixed order.
__global__ void wkv6_gu_reduce_kernel(const float* __restrict__ gu_part, int B, int HK, float* __restrict__ gu) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= HK) return;
  float s = 0.f;
  for (int b = 0; b < B; ++b) s += gu_part[(int64_t)b * HK + c];
  gu[c] = s;
}

size_t wkv6_bwd_workspace_bytes(int64_t B, int64_t T, int64_t H) {
  const int64_t BH = B * H;
  return sizeof(float) * (size_t)(BH * T * kK6b + BH * T * 4 + 2 * BH * kK6b);
}

wkv_status launch_wkv6_backward(const Wkv6BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  const int64_t BH = a.B * a.H, HK = a.H * kK6b;
  float* xws = static_cast<float*>(a.workspace);
  float* cvws = xws + BH * a.T * kK6b;
  float* p0 = cvws + BH * a.T * 4;
  float* gu_part = p0 + BH * kK6b;
  CUtensorMap maps[7];
  memset(maps, 0, sizeof(maps));
  if (a.T > 0) {
    const void* src[kIn6b] = {a.r, a.k, a.v, a.w, a.dout};
    for (int m = 0; m < kIn6b; ++m)
      if (!encode_tmap_3d(&maps[m], src[m], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)HK, (uint64_t)a.T,
                          (uint64_t)a.B, kK6b, kL6b, 1, why))
        return WKV_ERR_INVALID_ARG;
    if (!encode_tmap_3d(&maps[5], xws, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, kK6b, (uint64_t)a.T, (uint64_t)BH, kK6b,
                        kL6b, 1, why) ||
        !encode_tmap_3d(&maps[6], cvws, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 4, (uint64_t)a.T, (uint64_t)BH, 4, kL6b, 1,
                        why))
      return WKV_ERR_INVALID_ARG;
  }
  const size_t smem1 = sizeof(Wkv6Bwd1Smem), smem2 = sizeof(Wkv6Bwd2Smem);
  if (cudaFuncSetAttribute(wkv6_bwd_pass1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1) !=
          cudaSuccess ||
      cudaFuncSetAttribute(wkv6_bwd_pass2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2) !=
          cudaSuccess) {
    *why = "wkv6_backward: shared memory configuration failed";
    return WKV_ERR_CUDA;
  }
  wkv6_bwd_pass1_kernel<<<(unsigned)BH, kT6b, smem1, stream>>>(
      maps[0], maps[1], maps[2], maps[3], maps[4], (int)a.T, (int)a.H, a.u, a.init_state, a.state_map,
      (int)a.n_state, a.g_final, static_cast<__nv_bfloat16*>(a.gr), xws, cvws, p0, err);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) {
    wkv6_bwd_pass2_kernel<<<(unsigned)BH, kT6b, smem2, stream>>>(
        maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], maps[6], (int)a.T, (int)a.H, a.u, a.g_final, p0,
        static_cast<__nv_bfloat16*>(a.gk), static_cast<__nv_bfloat16*>(a.gv), static_cast<__nv_bfloat16*>(a.glogw),
        a.g_init, gu_part, err);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) {
    wkv6_gu_reduce_kernel<<<(unsigned)ceil_div(HK, 256), 256, 0, stream>>>(gu_part, (int)a.B, (int)HK, a.gu);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    *why = "wkv6_backward kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

}  // namespace wkv
