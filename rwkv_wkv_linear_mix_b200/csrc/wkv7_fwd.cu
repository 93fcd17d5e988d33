// wkv7_fwd.cu -- RWKV-7 generalized delta rule forward on sm_100a.
//
// Operator: generalized_delta_rule / rwkv7_op (rwkv-ops package page): r, w,
// k, v, a, b [B][T][H*K] with w the decay in log space, state [B][H][K][K]
// indexed [key j][value i], output o [B][T][H*K]. Per head, with the
// diagonal-plus-rank-one transition of a generalized delta rule:
//   sa[i]     = sum_j a_t[j] S_{t-1}[j][i]
//   S_t[j][i] = e^{w_t[j]} S_{t-1}[j][i] + b_t[j] sa[i] + k_t[j] v_t[i]
//   o_t[i]    = sum_j r_t[j] S_t[j][i]
// Both products reduce over the key index, so the state is split by keys
// within a row of threads and by values across rows.
//
// Kernel shape: one CTA of 128 threads per (b, h), sequential in t (the
// page's CUDA kernel is the same kind: fp32 inside, fast, but a long
// sequence is one head's serial work). Thread (g = tid / 8, q = tid % 8)
// holds values 4g .. 4g + 3 for keys 8q .. 8q + 7 (32 fp32: 4 columns x 4
// key pairs, on packed fp32 pair instructions); the two key reductions are
// sums over the 8 threads of a column group (lanes 8m .. 8m + 7, three
// shuffles; the output's reduction is transposed, so that after it each of
// the 8 threads holds one column's total and no value is summed twice).
// Inputs arrive per 32-token chunk by TMA into two stages; the
// chunk's decays e^{w} are formed once into shared memory; each step reads
// its key slices as bf16 one step ahead and widens them in registers; o
// leaves through a shared-memory tile as coalesced 16-byte stores. Waits are
// bounded (WKV_DEVERR_WAIT_TIMEOUT, then a clean exit).
#include <string.h>

#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkv {

constexpr int kK7 = 64;    // head size (keys = values)
constexpr int kL7 = 32;    // tokens per chunk
constexpr int kT7 = 128;   // threads per CTA
constexpr int kIn7 = 6;    // r, w, k, v, a, b
enum { kR7 = 0, kW7 = 1, kK7i = 2, kV7 = 3, kA7 = 4, kB7 = 5 };

struct alignas(128) Wkv7Smem {
  __nv_bfloat16 in[2][kIn7][kL7][kK7];  // two TMA stages
  float d[kL7][kK7];                    // e^{w} of the current chunk
  __nv_bfloat16 out[kL7][kK7];          // o tile
  uint64_t full[2];
};

// Sum over the 8 key threads of a column group.
__device__ __forceinline__ float keys_sum8(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  return x;
}

__device__ __forceinline__ float dot4(const float2 (&a)[4], const float2 (&s)[4]) {
  float2 acc = mul2(a[0], s[0]);
  acc = fma2(a[1], s[1], acc);
  acc = fma2(a[2], s[2], acc);
  acc = fma2(a[3], s[3], acc);
  return __fadd_rn(acc.x, acc.y);
}

// The step's raw operands: key slices (bf16, 16 bytes each), decays, values.
struct Wkv7Tok {
  uint4 r, k, a, b;
  float4 d0, d1;
  uint2 v;
};

// CKPT: the backward's forward sweep: no output, the state before every
// WKV7_CKPT_LEN-th token written to ckpt [B*H][ceil(T / WKV7_CKPT_LEN)][K][K].
template <bool CKPT>
__global__ void __launch_bounds__(kT7, 3) wkv7_fwd_kernel(
    const __grid_constant__ CUtensorMap tr, const __grid_constant__ CUtensorMap tw,
    const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
    const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb, int T, int H,
    const float* __restrict__ init_state, float* __restrict__ final_state, __nv_bfloat16* __restrict__ o,
    float* __restrict__ ckpt, unsigned* err) {
  extern __shared__ __align__(128) unsigned char wkv7_dsmem[];
  Wkv7Smem& sm = *reinterpret_cast<Wkv7Smem*>(wkv7_dsmem);
  const int tid = threadIdx.x, g = tid >> 3, q = tid & 7;  // values 4g .., keys 8q ..
  const int bh = (int)blockIdx.x, b = bh / H, h = bh % H;
  const int HK = H * kK7;
  const int nchunk = (T + kL7 - 1) / kL7;
  constexpr uint32_t kStageBytes = kIn7 * kL7 * kK7 * sizeof(__nv_bfloat16);
  const CUtensorMap* maps[kIn7] = {&tr, &tw, &tk, &tv, &ta, &tb};
  auto issue = [&](int ch) {
    const int s = ch & 1;
    mbar_arrive_expect_tx(&sm.full[s], kStageBytes);
    for (int m = 0; m < kIn7; ++m) tma_load_3d(&sm.in[s][m][0][0], maps[m], &sm.full[s], h * kK7, ch * kL7, b);
  };
  if (tid == 0) {
    mbar_init(&sm.full[0], 1);
    mbar_init(&sm.full[1], 1);
    mbar_init_fence();
    if (nchunk > 0)
      for (int m = 0; m < kIn7; ++m) tma_prefetch_desc(maps[m]);
    for (int ch = 0; ch < 2 && ch < nchunk; ++ch) issue(ch);
  }
  // S[c][m] = (S[8q + 2m][4g + c], S[8q + 2m + 1][4g + c])
  float2 S[4][4];
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int m = 0; m < 4; ++m) S[c][m] = make_float2(0.f, 0.f);
  if (init_state) {
    const float* base = init_state + (int64_t)bh * kK7 * kK7 + 4 * g;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const float4 lo = *reinterpret_cast<const float4*>(base + (8 * q + 2 * m) * kK7);
      const float4 hi = *reinterpret_cast<const float4*>(base + (8 * q + 2 * m + 1) * kK7);
      S[0][m] = make_float2(lo.x, hi.x);
      S[1][m] = make_float2(lo.y, hi.y);
      S[2][m] = make_float2(lo.z, hi.z);
      S[3][m] = make_float2(lo.w, hi.w);
    }
  }
  __syncthreads();

  bool ok = true;
  int ch = 0;
  for (; ch < nchunk; ++ch) {
    const int s = ch & 1;
    const int t0 = ch * kL7, n = min(kL7, T - t0);
    const bool got = mbar_wait_bounded(&sm.full[s], (ch >> 1) & 1, err);
    if (!__syncthreads_and(got)) {
      ok = false;
      break;
    }
    const __nv_bfloat16(*in)[kL7][kK7] = sm.in[s];
    // the chunk's decays e^{w} = 2^{w log2 e}
    for (int e = tid; e < kL7 * kK7; e += kT7) {
      const int jt = e / kK7, j = e % kK7;
      sm.d[jt][j] = ex2(__fmul_rn(__bfloat162float(in[kW7][jt][j]), kLog2e));
    }
    __syncthreads();
    auto fetch = [&](int jt) {
      Wkv7Tok x;
      x.r = *reinterpret_cast<const uint4*>(&in[kR7][jt][8 * q]);
      x.k = *reinterpret_cast<const uint4*>(&in[kK7i][jt][8 * q]);
      x.a = *reinterpret_cast<const uint4*>(&in[kA7][jt][8 * q]);
      x.b = *reinterpret_cast<const uint4*>(&in[kB7][jt][8 * q]);
      x.d0 = *reinterpret_cast<const float4*>(&sm.d[jt][8 * q]);
      x.d1 = *reinterpret_cast<const float4*>(&sm.d[jt][8 * q + 4]);
      x.v = *reinterpret_cast<const uint2*>(&in[kV7][jt][4 * g]);
      return x;
    };
    Wkv7Tok nx = fetch(0);
    for (int jt = 0; jt < n; ++jt) {
      const Wkv7Tok cu = nx;
      if (jt + 1 < n) nx = fetch(jt + 1);
      if constexpr (CKPT) {
        const int t = t0 + jt;
        if (t % WKV7_CKPT_LEN == 0) {
          const int nck = (T + WKV7_CKPT_LEN - 1) / WKV7_CKPT_LEN;
          float* base = ckpt + ((int64_t)bh * nck + t / WKV7_CKPT_LEN) * kK7 * kK7 + 4 * g;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            *reinterpret_cast<float4*>(base + (8 * q + 2 * m) * kK7) =
                make_float4(S[0][m].x, S[1][m].x, S[2][m].x, S[3][m].x);
            *reinterpret_cast<float4*>(base + (8 * q + 2 * m + 1) * kK7) =
                make_float4(S[0][m].y, S[1][m].y, S[2][m].y, S[3][m].y);
          }
        }
      }
      auto widen4 = [](const uint4& u, float2 (&x)[4]) {
        x[0] = make_float2(bf16lo(u.x), bf16hi(u.x));
        x[1] = make_float2(bf16lo(u.y), bf16hi(u.y));
        x[2] = make_float2(bf16lo(u.z), bf16hi(u.z));
        x[3] = make_float2(bf16lo(u.w), bf16hi(u.w));
      };
      float2 r2[4], k2[4], a2[4], b2[4];
      widen4(cu.r, r2);
      widen4(cu.k, k2);
      widen4(cu.a, a2);
      widen4(cu.b, b2);
      const float2 d2[4] = {make_float2(cu.d0.x, cu.d0.y), make_float2(cu.d0.z, cu.d0.w),
                            make_float2(cu.d1.x, cu.d1.y), make_float2(cu.d1.z, cu.d1.w)};
      const float vv[4] = {bf16lo(cu.v.x), bf16hi(cu.v.x), bf16lo(cu.v.y), bf16hi(cu.v.y)};
      float po[4] = {0.f, 0.f, 0.f, 0.f};  // this thread's 8-key part of (r_t S_t)[4g + c]
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float sa = keys_sum8(dot4(a2, S[c]));  // (a_t S_{t-1})[4g + c]
        const float2 sa2 = make_float2(sa, sa), v2 = make_float2(vv[c], vv[c]);
#pragma unroll
        for (int m = 0; m < 4; ++m) S[c][m] = fma2(S[c][m], d2[m], fma2(b2[m], sa2, mul2(k2[m], v2)));
        if constexpr (!CKPT) po[c] = dot4(r2, S[c]);
      }
      if constexpr (!CKPT) {
        // transposed sum over the 8 key threads: each exchange passes on the
        // half of the columns this thread does not keep (the same pairwise
        // tree as a butterfly, so the same bits); thread q ends with column
        // 2 (q & 1) + (q & 2) / 2, twice per group
        const bool q0 = q & 1, q1 = q & 2;
        float k0 = q0 ? po[2] : po[0], k1 = q0 ? po[3] : po[1];
        const float s0 = q0 ? po[0] : po[2], s1 = q0 ? po[1] : po[3];
        k0 = __fadd_rn(k0, __shfl_xor_sync(0xffffffffu, s0, 1));
        k1 = __fadd_rn(k1, __shfl_xor_sync(0xffffffffu, s1, 1));
        float kk = q1 ? k1 : k0;
        kk = __fadd_rn(kk, __shfl_xor_sync(0xffffffffu, q1 ? k0 : k1, 2));
        kk = __fadd_rn(kk, __shfl_xor_sync(0xffffffffu, kk, 4));
        if (!(q & 4)) sm.out[jt][4 * g + (q0 ? 2 : 0) + (q1 ? 1 : 0)] = __float2bfloat16_rn(kk);
      }
    }
    __syncthreads();
    if (tid == 0 && ch + 2 < nchunk) issue(ch + 2);  // every read of stage s is done
    if constexpr (!CKPT) {
      for (int p = tid; p < kL7 * 8; p += kT7) {
        const int row = p / 8, piece = p % 8;
        if (row < n)
          *reinterpret_cast<uint4*>(o + ((int64_t)b * T + t0 + row) * HK + (int64_t)h * kK7 + piece * 8) =
              reinterpret_cast<const uint4*>(&sm.out[row][0])[piece];
      }
    }
  }
  if (!ok) {
    // a wait gave up: let the copies in flight land before the CTA exits
    if (tid == 0)
      for (int x = ch; x < nchunk && x < ch + 2; ++x) mbar_wait_bounded(&sm.full[x & 1], (x >> 1) & 1, err);
    return;
  }
  if (final_state) {
    float* base = final_state + (int64_t)bh * kK7 * kK7 + 4 * g;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      *reinterpret_cast<float4*>(base + (8 * q + 2 * m) * kK7) = make_float4(S[0][m].x, S[1][m].x, S[2][m].x, S[3][m].x);
      *reinterpret_cast<float4*>(base + (8 * q + 2 * m + 1) * kK7) =
          make_float4(S[0][m].y, S[1][m].y, S[2][m].y, S[3][m].y);
    }
  }
}

wkv_status launch_wkv7_forward(const Wkv7FwdArgs& a, cudaStream_t stream, unsigned* err, const char** why) {
  CUtensorMap maps[kIn7];
  memset(maps, 0, sizeof(maps));
  const uint64_t HK = (uint64_t)a.H * kK7;
  if (a.T > 0) {
    const void* src[kIn7] = {a.r, a.w, a.k, a.v, a.a, a.b};
    for (int m = 0; m < kIn7; ++m)
      if (!encode_tmap_3d(&maps[m], src[m], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, HK, (uint64_t)a.T, (uint64_t)a.B,
                          kK7, kL7, 1, why))
        return WKV_ERR_INVALID_ARG;
  }
  const size_t smem = sizeof(Wkv7Smem);
  auto kern = a.ckpt ? wkv7_fwd_kernel<true> : wkv7_fwd_kernel<false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
    *why = "wkv7_forward: shared memory configuration failed";
    return WKV_ERR_CUDA;
  }
  kern<<<(unsigned)(a.B * a.H), kT7, smem, stream>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], (int)a.T,
                                                    (int)a.H, a.init_state, a.final_state,
                                                    static_cast<__nv_bfloat16*>(a.o), a.ckpt, err);
  if (cudaGetLastError() != cudaSuccess) {
    *why = "wkv7_forward kernel launch failed";
    return WKV_ERR_CUDA;
  }
  return WKV_OK;
}

}  // namespace wkv
