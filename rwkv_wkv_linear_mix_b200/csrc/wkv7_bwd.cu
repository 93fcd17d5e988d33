// wkv7_bwd.cu -- RWKV-7 generalized delta rule backward on sm_100a.
//
// Gradients of L = sum(dout * o) + sum(g_final * S_final) for the forward of
// wkv7_fwd.cu (generalized_delta_rule of the rwkv-ops package page, which
// carries gradients; its _inference twin does not). Per head, with G =
// dL/dS_t walked from the last token down (j the key index, i the value
// index, d = e^{w_t}, sa = a_t S_{t-1}):
//   G        += r_t^T dout_t
//   dr_t[j]   = sum_i S_t[j][i] dout_t[i]       dk_t[j] = sum_i G[j][i] v_t[i]
//   db_t[j]   = sum_i G[j][i] sa[i]             dw_t[j] = d[j] sum_i G[j][i] S_{t-1}[j][i]
//   dsa[i]    = sum_j b_t[j] G[j][i]            dv_t[i] = sum_j k_t[j] G[j][i]
//   da_t[j]   = sum_i S_{t-1}[j][i] dsa[i]
//   G        <- diag(d) G + a_t^T dsa
// and d_init = G after token 0.
//
// The reverse walk needs the state before and after every token. The
// forward kernel's checkpoint sweep leaves the state before every 4th token
// in the workspace; per 4-token group, walking down, one CTA per (b, h)
// reloads the group's checkpoint, recomputes the group's states into shared
// memory (5 x 16 KB) with the forward's own step, and then runs the group's
// reverse steps. Thread (g = tid / 8, q = tid % 8) holds G for values
// 4g .. 4g + 3 and keys 8q .. 8q + 7, as the forward holds S: the sums over
// keys (dsa, dv) are three shuffles within the 8 threads of a value group
// and are all the walk itself needs; the five sums over values (dr, dk, db,
// dw, da) leave as per-thread partials in shared memory and are added
// across the 16 value groups in a fixed order once per group, so a group
// costs three barriers, not one per token. A first, exact version: one
// token at a time on CUDA cores.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

namespace {

constexpr int kK7b = 64;               // head size (keys = values)
constexpr int kT7b = 128;              // threads per CTA
constexpr int kL7b = WKV7_CKPT_LEN;    // tokens per checkpoint group
enum { kIR = 0, kID = 1, kIK = 2, kIV = 3, kIA = 4, kIB = 5, kIDo = 6, kInputs = 7 };
enum { kPR = 0, kPK = 1, kPB = 2, kPW = 3, kPA = 4, kParts = 5 };

struct alignas(16) Wkv7BwdSmem {
  float hist[kL7b + 1][kK7b][kK7b];     // state before token jt of the group (hist[jt]) and after the last
  float in[kInputs][kL7b][kK7b];        // r, e^{w}, k, v, a, b, dout of the group
  float sa[kL7b][kK7b];                 // a_t S_{t-1} of each token
  float part[kL7b][16][kParts][kK7b];   // per token and value group: partial sums over its 4 values
};

__device__ __forceinline__ float sum8(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  return x;
}

__device__ __forceinline__ float dot4b(const float2 (&a)[4], const float2 (&s)[4]) {
  float2 acc = mul2(a[0], s[0]);
  acc = fma2(a[1], s[1], acc);
  acc = fma2(a[2], s[2], acc);
  acc = fma2(a[3], s[3], acc);
  return __fadd_rn(acc.x, acc.y);
}

// 8 keys 8q .. 8q + 7 of a row of `src` as 4 pairs. Threads q >= 4 read the
// two halves in the other order, so that within each load the 8 threads of a
// quarter warp fall in 8 different bank groups.
__device__ __forceinline__ void keys8(const float* src, int q, float2 (&x)[4]) {
  const bool sw = q & 4;
  const float4 f0 = *reinterpret_cast<const float4*>(src + 8 * q + (sw ? 4 : 0));
  const float4 f1 = *reinterpret_cast<const float4*>(src + 8 * q + (sw ? 0 : 4));
  const float4 lo = sw ? f1 : f0, hi = sw ? f0 : f1;
  x[0] = make_float2(lo.x, lo.y);
  x[1] = make_float2(lo.z, lo.w);
  x[2] = make_float2(hi.x, hi.y);
  x[3] = make_float2(hi.z, hi.w);
}

// the thread's 32 entries of a [K][K] state, S[c][m] = (S[8q+2m][4g+c], S[8q+2m+1][4g+c])
__device__ __forceinline__ void ld_state(const float* base, int g, int q, float2 (&S)[4][4]) {
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const float4 lo = *reinterpret_cast<const float4*>(base + (8 * q + 2 * m) * kK7b + 4 * g);
    const float4 hi = *reinterpret_cast<const float4*>(base + (8 * q + 2 * m + 1) * kK7b + 4 * g);
    S[0][m] = make_float2(lo.x, hi.x);
    S[1][m] = make_float2(lo.y, hi.y);
    S[2][m] = make_float2(lo.z, hi.z);
    S[3][m] = make_float2(lo.w, hi.w);
  }
}
__device__ __forceinline__ void st_state(float* base, int g, int q, const float2 (&S)[4][4]) {
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    *reinterpret_cast<float4*>(base + (8 * q + 2 * m) * kK7b + 4 * g) =
        make_float4(S[0][m].x, S[1][m].x, S[2][m].x, S[3][m].x);
    *reinterpret_cast<float4*>(base + (8 * q + 2 * m + 1) * kK7b + 4 * g) =
        make_float4(S[0][m].y, S[1][m].y, S[2][m].y, S[3][m].y);
  }
}

// The same slices of a state kept in shared memory, with the 16-byte chunk
// index of row j swizzled by j / 8: the 8 threads of a quarter warp (same g,
// q = 0 .. 7) then touch 8 different bank groups instead of one.
__device__ __forceinline__ void ld_state_sm(const float* base, int g, int q, float2 (&S)[4][4]) {
  const int col = 4 * (g ^ q);
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const float4 lo = *reinterpret_cast<const float4*>(base + (8 * q + 2 * m) * kK7b + col);
    const float4 hi = *reinterpret_cast<const float4*>(base + (8 * q + 2 * m + 1) * kK7b + col);
    S[0][m] = make_float2(lo.x, hi.x);
    S[1][m] = make_float2(lo.y, hi.y);
    S[2][m] = make_float2(lo.z, hi.z);
    S[3][m] = make_float2(lo.w, hi.w);
  }
}
__device__ __forceinline__ void st_state_sm(float* base, int g, int q, const float2 (&S)[4][4]) {
  const int col = 4 * (g ^ q);
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    *reinterpret_cast<float4*>(base + (8 * q + 2 * m) * kK7b + col) =
        make_float4(S[0][m].x, S[1][m].x, S[2][m].x, S[3][m].x);
    *reinterpret_cast<float4*>(base + (8 * q + 2 * m + 1) * kK7b + col) =
        make_float4(S[0][m].y, S[1][m].y, S[2][m].y, S[3][m].y);
  }
}

__global__ void __launch_bounds__(kT7b, 1) wkv7_bwd_kernel(
    int T, int H, const __nv_bfloat16* __restrict__ r, const __nv_bfloat16* __restrict__ w,
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ a,
    const __nv_bfloat16* __restrict__ b, const __nv_bfloat16* __restrict__ dout, const float* __restrict__ ckpt,
    const float* __restrict__ g_final, __nv_bfloat16* __restrict__ dr, __nv_bfloat16* __restrict__ dw,
    __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv, __nv_bfloat16* __restrict__ da,
    __nv_bfloat16* __restrict__ db, float* __restrict__ d_init) {
  extern __shared__ __align__(16) unsigned char wkv7_bwd_dsmem[];
  Wkv7BwdSmem& sm = *reinterpret_cast<Wkv7BwdSmem*>(wkv7_bwd_dsmem);
  const int tid = threadIdx.x, g = tid >> 3, q = tid & 7;
  const int bh = (int)blockIdx.x, bi = bh / H, h = bh % H;
  const int64_t HK = (int64_t)H * kK7b;
  const int nck = (T + kL7b - 1) / kL7b;
  const __nv_bfloat16* srcs[kInputs] = {r, w, k, v, a, b, dout};
  __nv_bfloat16* outs[kParts] = {dr, dk, db, dw, da};

  float2 G[4][4];
  if (g_final) {
    ld_state(g_final + (int64_t)bh * kK7b * kK7b, g, q, G);
  } else {
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int m = 0; m < 4; ++m) G[c][m] = make_float2(0.f, 0.f);
  }
  for (int grp = nck - 1; grp >= 0; --grp) {
    const int t0 = grp * kL7b, n = min(kL7b, T - t0);
    // the group's inputs, widened (e^{w} formed as the forward forms it)
    for (int e = tid; e < kInputs * kL7b * kK7b; e += kT7b) {
      const int x = e / (kL7b * kK7b), jt = (e / kK7b) % kL7b, j = e % kK7b;
      float val = 0.f;
      if (jt < n) {
        val = __bfloat162float(srcs[x][((int64_t)bi * T + t0 + jt) * HK + (int64_t)h * kK7b + j]);
        if (x == kID) val = ex2(__fmul_rn(val, kLog2e));
      }
      sm.in[x][jt][j] = val;
    }
    float2 S[4][4];
    ld_state(ckpt + ((int64_t)bh * nck + grp) * kK7b * kK7b, g, q, S);
    st_state_sm(&sm.hist[0][0][0], g, q, S);
    __syncthreads();
    // recompute the group's states with the forward's step
    for (int jt = 0; jt < n; ++jt) {
      float2 a2[4], b2[4], k2[4], d2[4];
      keys8(sm.in[kIA][jt], q, a2);
      keys8(sm.in[kIB][jt], q, b2);
      keys8(sm.in[kIK][jt], q, k2);
      keys8(sm.in[kID][jt], q, d2);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float sa = sum8(dot4b(a2, S[c]));
        if (q == 0) sm.sa[jt][4 * g + c] = sa;
        const float vc = sm.in[kIV][jt][4 * g + c];
        const float2 sa2 = make_float2(sa, sa), v2 = make_float2(vc, vc);
#pragma unroll
        for (int m = 0; m < 4; ++m) S[c][m] = fma2(S[c][m], d2[m], fma2(b2[m], sa2, mul2(k2[m], v2)));
      }
      st_state_sm(&sm.hist[jt + 1][0][0], g, q, S);
    }
    __syncthreads();
    // reverse steps of the group
    for (int jt = n - 1; jt >= 0; --jt) {
      const int64_t row = ((int64_t)bi * T + t0 + jt) * HK + (int64_t)h * kK7b;
      float2 r2[4], d2[4], k2[4], a2[4], b2[4], Sp[4][4], Sc[4][4];
      keys8(sm.in[kIR][jt], q, r2);
      keys8(sm.in[kID][jt], q, d2);
      keys8(sm.in[kIK][jt], q, k2);
      keys8(sm.in[kIA][jt], q, a2);
      keys8(sm.in[kIB][jt], q, b2);
      ld_state_sm(&sm.hist[jt][0][0], g, q, Sp);
      ld_state_sm(&sm.hist[jt + 1][0][0], g, q, Sc);
      float vv[4], dov[4], sav[4], dsa[4], dvv[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        vv[c] = sm.in[kIV][jt][4 * g + c];
        dov[c] = sm.in[kIDo][jt][4 * g + c];
        sav[c] = sm.sa[jt][4 * g + c];
      }
      // G becomes dL/dS_t: the output of this token reads S_t
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int m = 0; m < 4; ++m) G[c][m] = fma2(r2[m], make_float2(dov[c], dov[c]), G[c][m]);
      // sums over keys
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        dsa[c] = sum8(dot4b(b2, G[c]));
        dvv[c] = sum8(dot4b(k2, G[c]));
      }
      // this thread's partial sums over its 4 values, for its 8 keys
      float2 p[kParts][4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float2 pr = make_float2(0.f, 0.f), pk = pr, pb = pr, pw = pr, pa = pr;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          pr = fma2(Sc[c][m], make_float2(dov[c], dov[c]), pr);
          pk = fma2(G[c][m], make_float2(vv[c], vv[c]), pk);
          pb = fma2(G[c][m], make_float2(sav[c], sav[c]), pb);
          pw = fma2(G[c][m], Sp[c][m], pw);
          pa = fma2(Sp[c][m], make_float2(dsa[c], dsa[c]), pa);
        }
        p[kPR][m] = pr;
        p[kPK][m] = pk;
        p[kPB][m] = pb;
        p[kPW][m] = pw;
        p[kPA][m] = pa;
      }
#pragma unroll
      for (int x = 0; x < kParts; ++x) {
        float* dst = &sm.part[jt][g][x][8 * q];
        const float4 lo = make_float4(p[x][0].x, p[x][0].y, p[x][1].x, p[x][1].y);
        const float4 hi = make_float4(p[x][2].x, p[x][2].y, p[x][3].x, p[x][3].y);
        const bool sw = q & 4;  // halves in the other order, as in keys8
        *reinterpret_cast<float4*>(dst + (sw ? 4 : 0)) = sw ? hi : lo;
        *reinterpret_cast<float4*>(dst + (sw ? 0 : 4)) = sw ? lo : hi;
      }
      if (q == 0) {
        uint2 pk2;
        pk2.x = pack_bf16x2(dvv[0], dvv[1]);
        pk2.y = pack_bf16x2(dvv[2], dvv[3]);
        *reinterpret_cast<uint2*>(dv + row + 4 * g) = pk2;
      }
      // G becomes dL/dS_{t-1}
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int m = 0; m < 4; ++m) G[c][m] = fma2(d2[m], G[c][m], mul2(a2[m], make_float2(dsa[c], dsa[c])));
    }
    __syncthreads();
    // the group's five sums over values (they do not feed the walk), added
    // across the 16 value groups in order
    for (int e = tid; e < n * kParts * kK7b; e += kT7b) {
      const int jt = e / (kParts * kK7b), x = (e / kK7b) % kParts, j = e % kK7b;
      float s = 0.f;
#pragma unroll
      for (int gg = 0; gg < 16; ++gg) s += sm.part[jt][gg][x][j];
      if (x == kPW) s = __fmul_rn(s, sm.in[kID][jt][j]);
      outs[x][((int64_t)bi * T + t0 + jt) * HK + (int64_t)h * kK7b + j] = __float2bfloat16_rn(s);
    }
    __syncthreads();  // the group's inputs, states and partials are read; the next group may overwrite them
  }
  st_state(d_init + (int64_t)bh * kK7b * kK7b, g, q, G);
}

}  // namespace

wkv_status launch_wkv7_backward(const Wkv7BwdArgs& a, cudaStream_t stream, const char** why) {
  const size_t smem = sizeof(Wkv7BwdSmem);
  if (cudaFuncSetAttribute(wkv7_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess) {
    *why = "wkv7_backward: shared memory configuration failed";
    return WKV_ERR_CUDA;
  }
  using bf = __nv_bfloat16;
  wkv7_bwd_kernel<<<(unsigned)(a.B * a.H), kT7b, smem, stream>>>(
      (int)a.T, (int)a.H, static_cast<const bf*>(a.r), static_cast<const bf*>(a.w), static_cast<const bf*>(a.k),
      static_cast<const bf*>(a.v), static_cast<const bf*>(a.a), static_cast<const bf*>(a.b),
      static_cast<const bf*>(a.dout), a.ckpt, a.g_final, static_cast<bf*>(a.dr), static_cast<bf*>(a.dw),
      static_cast<bf*>(a.dk), static_cast<bf*>(a.dv), static_cast<bf*>(a.da), static_cast<bf*>(a.db), a.d_init);
  if (cudaGetLastError() != cudaSuccess) {
    *why = "wkv7_backward kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

}  // namespace wkv
