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
// Two passes, one CTA of 256 threads per (b, h); thread (i = tid / 4,
// q = tid % 4) holds row i, columns 16q .. 16q + 15:
//   pass 1 (t up):   S; writes gr and, per token, x_t = r_t o (S_{t-1} do_t)
//                    and (c_t = r_t . (u o k_t), v_t . do_t) to the workspace;
//                    at the end P_{T-1} = sum_j g_final S_{T-1}.
//   pass 2 (t down): G in two copies, by rows (G v, the P walk, g_init) and
//                    by columns (k G becomes a row product as well, so no
//                    64-way reduction across threads); writes gk, gv, glogw
//                    and per-(b, h) gu partials.
// Inputs arrive per 32-token chunk by TMA into two stages (the next chunk
// loads while this one runs). Each step reads its 16-wide slices as bf16
// (32 bytes per vector: the 64 threads that share a slice make shared-memory
// bandwidth, not arithmetic, the limit) one step ahead of use, and widens
// them in registers. Outputs leave through shared-memory tiles as coalesced
// 16-byte stores. The 16-wide row work runs on packed fp32 pairs. gu is
// summed over samples by a fixed-order reduction.
#include <string.h>

#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

constexpr int kK6b = 64;       // head size
constexpr int kL6b = 32;       // tokens per chunk
constexpr int kT6b = 256;      // threads per CTA
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

// Store a [kL6b][kK6b] bf16 tile to rows t0 .. t0 + n - 1 of a [B][T][HK]
// tensor at column h * 64 (one 16-byte piece per thread).
__device__ __forceinline__ void wkv6_store_tile(const __nv_bfloat16 (*tile)[kK6b], __nv_bfloat16* dst, int b, int T,
                                                int HK, int h, int t0, int n, int tid) {
  const int row = tid / 8, piece = tid % 8;
  if (row < n) {
    const uint4 val = reinterpret_cast<const uint4*>(&tile[row][0])[piece];
    *reinterpret_cast<uint4*>(dst + ((int64_t)b * T + t0 + row) * HK + (int64_t)h * kK6b + piece * 8) = val;
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
  const int tid = threadIdx.x, i = tid >> 2, q = tid & 3;
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
  float2 S[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) S[m] = make_float2(0.f, 0.f);
  if (init_state) {
    const int sidx = state_map ? state_map[b] : (n_state == 1 ? 0 : b);
    if (sidx < 0 || sidx >= n_state) {
      if (tid == 0) record_error(err, WKV_DEVERR_BAD_STATE);
    } else {
      ld16(init_state + (((int64_t)sidx * H + h) * kK6b + i) * kK6b + 16 * q, S);
    }
  }
  const float ui = u[h * kK6b + i];
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
      // per token: c_t = r . (u o k) and v . do, 8 threads per token
      const int jt = tid >> 3, part = tid & 7;
      float c = 0.f, vd = 0.f;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int e = part * 8 + m;
        c = __fmaf_rn(bf(in[kR][jt][e]) * u[h * kK6b + e], bf(in[kKk][jt][e]), c);
        vd = __fmaf_rn(bf(in[kV][jt][e]), bf(in[kDo][jt][e]), vd);
      }
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        c += __shfl_xor_sync(0xffffffffu, c, o);
        vd += __shfl_xor_sync(0xffffffffu, vd, o);
      }
      if (part == 0) reinterpret_cast<float4*>(&sm.cv[s][jt][0])[0] = make_float4(c, vd, 0.f, 0.f);
    }
    __syncthreads();
    // the step's vectors are fetched one step ahead
    Bf16x16 vn = ld16b(&in[kV][0][16 * q]), dn = ld16b(&in[kDo][0][16 * q]);
    float wn = bf(in[kW][0][i]), kn = bf(in[kKk][0][i]), rn = bf(in[kR][0][i]), vdn = sm.cv[s][0][1];
    for (int jt = 0; jt < n; ++jt) {
      const Bf16x16 vc = vn, dc = dn;
      const float wi = wn, ki = kn, ri = rn, vdo = vdn;
      if (jt + 1 < n) {
        vn = ld16b(&in[kV][jt + 1][16 * q]);
        dn = ld16b(&in[kDo][jt + 1][16 * q]);
        wn = bf(in[kW][jt + 1][i]);
        kn = bf(in[kKk][jt + 1][i]);
        rn = bf(in[kR][jt + 1][i]);
        vdn = sm.cv[s][jt + 1][1];
      }
      float2 vv[8], dd[8];
      widen16(vc, vv);
      widen16(dc, dd);
      const float acc = row_sum4(dot16(S, dd));  // (S_{t-1} do_t)[i]
      if (q == 0) {
        sm.gro[jt][i] = __float2bfloat16_rn(__fmaf_rn(ui * ki, vdo, acc));
        sm.xo[jt][i] = __fmul_rn(ri, acc);
      }
      const float2 w2 = make_float2(wi, wi), k2 = make_float2(ki, ki);
#pragma unroll
      for (int m = 0; m < 8; ++m) S[m] = fma2(S[m], w2, mul2(k2, vv[m]));
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
  float pp = 0.f;
  if (g_final) {
    float2 gf[8];
    ld16(g_final + ((int64_t)bh * kK6b + i) * kK6b + 16 * q, gf);
    pp = dot16(gf, S);
  }
  pp = row_sum4(pp);
  if (q == 0) p0[(int64_t)bh * kK6b + i] = pp;
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
  const int tid = threadIdx.x, i = tid >> 2, q = tid & 3;  // row i of G; column i of G^T
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
  float2 G[8], Gc[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) G[m] = Gc[m] = make_float2(0.f, 0.f);
  if (g_final) {
    const float* gf = g_final + (int64_t)bh * kK6b * kK6b;
    ld16(gf + i * kK6b + 16 * q, G);
#pragma unroll
    for (int m = 0; m < 8; ++m)
      Gc[m] = make_float2(gf[(16 * q + 2 * m) * kK6b + i], gf[(16 * q + 2 * m + 1) * kK6b + i]);
  }
  float P = p0[(int64_t)bh * kK6b + i];
  const float ui = u[h * kK6b + i];
  float gu_i = 0.f;
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
      float wi, ri, ki, dj, c, vdo, xi;
    };
    auto fetch = [&](int jt) {
      Tok x;
      x.v = ld16b(&st.in[kV][jt][16 * q]);
      x.d = ld16b(&st.in[kDo][jt][16 * q]);
      x.r = ld16b(&st.in[kR][jt][16 * q]);
      x.k = ld16b(&st.in[kKk][jt][16 * q]);
      x.w = ld16b(&st.in[kW][jt][16 * q]);
      x.wi = bf(st.in[kW][jt][i]);
      x.ri = bf(st.in[kR][jt][i]);
      x.ki = bf(st.in[kKk][jt][i]);
      x.dj = bf(st.in[kDo][jt][i]);
      x.c = st.cv[jt][0];
      x.vdo = st.cv[jt][1];
      x.xi = st.x[jt][i];
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
      const float gki = row_sum4(dot16(G, vv));   // (G_t v_t)[i]
      const float gvj = row_sum4(dot16(kk, Gc));  // (k_t G_t)[i]
      const float gl = __fsub_rn(P, __fmul_rn(cu.ki, gki));  // w_t gw_t
      P = __fadd_rn(gl, cu.xi);                              // P_{t-1}
      if (q == 0) {
        sm.out[0][jt][i] = __float2bfloat16_rn(__fmaf_rn(ui * cu.ri, cu.vdo, gki));
        sm.out[1][jt][i] = __float2bfloat16_rn(__fmaf_rn(cu.c, cu.dj, gvj));
        sm.out[2][jt][i] = __float2bfloat16_rn(gl);
      }
      gu_i = __fmaf_rn(cu.ri * cu.ki, cu.vdo, gu_i);
      const float2 w2 = make_float2(cu.wi, cu.wi), r2 = make_float2(cu.ri, cu.ri), d2 = make_float2(cu.dj, cu.dj);
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        G[m] = fma2(G[m], w2, mul2(r2, dd[m]));
        Gc[m] = fma2(Gc[m], ww[m], mul2(rr[m], d2));
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
    float4* d = reinterpret_cast<float4*>(g_init + ((int64_t)bh * kK6b + i) * kK6b + 16 * q);
#pragma unroll
    for (int m = 0; m < 4; ++m) d[m] = make_float4(G[2 * m].x, G[2 * m].y, G[2 * m + 1].x, G[2 * m + 1].y);
  }
  if (q == 0) gu_part[(int64_t)bh * kK6b + i] = gu_i;
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
