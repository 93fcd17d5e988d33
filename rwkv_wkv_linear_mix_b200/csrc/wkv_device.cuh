// wkv_device.cuh -- device-side building blocks shared by the WKV kernels:
// storage-type traits, hardware exp2 / reciprocal, mbarrier and TMA wrappers
// (sm_100a inline PTX), bounded waits, and the RWKV-4 running-max step.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "wkv.h"
#include "wkv_internal.h"

namespace wkv {

// log2(e): the RWKV-4 kernels run the recurrence in base 2, so every
// exponential is a single ex2 instruction.
constexpr float kLog2e = 1.4426950408889634f;
// pp of the empty past: a finite "minus infinity" (no inf - inf under ftz).
constexpr float kEmptyPP = -1.0e38f;
// Give up a wait on a copy after this many nanoseconds (then record an error).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// ----------------------------------------------------------------------------
// storage types
// ----------------------------------------------------------------------------
template <class E> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f32(float x) { return x; }
  static __device__ __forceinline__ float from_f32(float x) { return x; }
  static constexpr CUtensorMapDataType tma_type = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f32(float x) { return __float2bfloat16_rn(x); }
  static constexpr CUtensorMapDataType tma_type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
};

// ----------------------------------------------------------------------------
// hardware transcendental instructions (PTX ex2.approx / rcp.approx)
// ----------------------------------------------------------------------------
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_error(unsigned* err, unsigned code) {
  if (err) atomicOr(err, code);
}

// ----------------------------------------------------------------------------
// mbarrier (shared::cta) and TMA
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that may suspend the thread for up to `hint_ns` nanoseconds while
// the phase is incomplete (a suspended thread issues no instructions; it is
// woken when the phase completes).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, for at most kWaitLimitNs.
// Returns false (and records WKV_DEVERR_WAIT_TIMEOUT) if it never does.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, unsigned* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      record_error(err, WKV_DEVERR_WAIT_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled bulk tensor load global -> shared (no multicast), completion
// signalled on `bar` as transaction bytes. x is the innermost coordinate.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// 3-D tiled bulk tensor store shared -> global (rows outside the tensor are
// not written; coordinates must not be negative), tracked as a bulk group of
// the issuing thread.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void tma_store_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the issuing thread's stores have finished reading shared memory.
__device__ __forceinline__ void tma_store_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// ----------------------------------------------------------------------------
// thread-block clusters and distributed shared memory
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// All threads of every CTA of the cluster arrive (release: this CTA's shared
// memory writes become visible to the cluster) / wait (acquire).
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory object in the CTA of cluster rank `rank`.
__device__ __forceinline__ uint32_t map_shared_rank(const void* p, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
  return a;
}
__device__ __forceinline__ float ld_shared_cluster(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float2 ld_shared_cluster_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
  return v;
}

// ----------------------------------------------------------------------------
// tcgen05 (5th-generation tensor cores, accumulators in tensor memory)
//
// Operand tiles are 64 x 64 matrices stored as rows of 128 bytes in the
// 128-byte-swizzled layout (the 16-byte chunk index of row r is XORed with
// r % 8; tiles are 1024-byte aligned), which is also the layout a TMA load
// with CU_TENSOR_MAP_SWIZZLE_128B writes. A bf16 tile is 64 rows of 64
// elements; an fp32 (tf32) tile is two 8 KB panels of 64 rows x 32 columns.
//  * K-major (rows M or N, columns K): the K step kk (16 bf16 / 8 tf32
//    elements = 32 bytes) starts 32 * (kk % 4) bytes into its panel.
//  * MN-major bf16 (rows K, columns M or N): the K step kk starts 2048 * kk
//    bytes (16 rows) into the tile.
//  * MN-major tf32 uses another swizzle (umma_desc_sw128_32b): 32-byte
//    chunks XORed with row % 4; the K step kk (8 rows) starts 1024 * kk
//    bytes into the panel and the second 32-column panel is LBO away.
// An M = 64 accumulator holds row m in TMEM lane (m % 16) + 32 * (m / 16),
// so warp q of a warpgroup reads rows 16q .. 16q + 15 in its lanes 0 .. 15.
// ----------------------------------------------------------------------------
__device__ __forceinline__ int sw128_offset(int row, int col_bf16) {
  return row * 128 + ((((col_bf16 >> 3) ^ (row & 7)) & 7) << 4) + (col_bf16 & 7) * 2;
}

// Shared-memory matrix descriptor (sm_100 format, 128-byte swizzle).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Descriptor of an MN-major tf32 operand in the 32-byte-granular 128-byte
// swizzle (layout type 1: the 32-byte chunk index of row r is XORed with
// r % 4; 4-row K groups SBO bytes apart, 32-column MN atoms LBO bytes apart).
// This is the only swizzled layout the tensor cores take for MN-major tf32.
__device__ __forceinline__ uint64_t umma_desc_sw128_32b(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (1ull << 61);
}
__device__ __forceinline__ uint64_t umma_kmajor(uint32_t tile, int kk) { return umma_desc_sw128(tile + 32u * kk, 16u, 1024u); }
__device__ __forceinline__ uint64_t umma_mnmajor(uint32_t tile, int kk) {
  return umma_desc_sw128(tile + 2048u * kk, 8192u, 1024u);
}

// Instruction descriptor of kind::f16: bf16 A and B, f32 accumulator, M x N,
// a_mn / b_mn = 1 when that operand is MN-major.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A * B for one 16-deep K step; issued by a single thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}
// Instruction descriptor of kind::tf32: tf32 A and B (fp32 storage, low 13
// mantissa bits ignored), f32 accumulator, M x N.
__host__ __device__ constexpr uint32_t umma_idesc_tf32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// D[tmem] (+)= A * B for one 8-deep K step of tf32 operands.
__device__ __forceinline__ void umma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}
// Arrive once on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor-core operand reads, TMA).
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 32 consecutive 32-bit TMEM columns of this thread's lane (32x32b shape).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]),
        "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15]),
        "=f"(v[16]), "=f"(v[17]), "=f"(v[18]), "=f"(v[19]), "=f"(v[20]), "=f"(v[21]), "=f"(v[22]), "=f"(v[23]),
        "=f"(v[24]), "=f"(v[25]), "=f"(v[26]), "=f"(v[27]), "=f"(v[28]), "=f"(v[29]), "=f"(v[30]), "=f"(v[31])
      : "r"(taddr)
      : "memory");
}
// 16 consecutive 32-bit TMEM columns of this thread's lane (32x32b shape).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]),
        "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15])
      : "r"(taddr)
      : "memory");
}
// 16 TMEM lanes x 32 columns (16x256b shape, 4 repetitions): relative to the
// lane base, thread t receives for q = 0..3 the columns c = 8q + 2 (t % 4)
// and c + 1 of row t / 4 (v[4q], v[4q + 1]) and of row t / 4 + 8
// (v[4q + 2], v[4q + 3]) -- all 32 threads busy for an M = 64 accumulator.
__device__ __forceinline__ void tmem_ld16x256b_x4(uint32_t taddr, float (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]),
        "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// bf16 pair <-> two floats (low half = first element).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}
__device__ __forceinline__ float bf16lo(uint32_t p) { return __uint_as_float(p << 16); }
__device__ __forceinline__ float bf16hi(uint32_t p) { return __uint_as_float(p & 0xFFFF0000u); }

// ----------------------------------------------------------------------------
// RWKV-4 step, running-max form in base 2.
//
// State of one lane: the past sums a = aa * 2^(P + ref), b = bb * 2^(P + ref)
// with P = base - n * w2. Three choices keep every exponent accurate to one
// rounding, however long the sequence and however large the keys:
//  * ref = fl(k_first * log2e) is a per-lane reference fixed by the first key
//    the lane absorbs; a key enters as kk = fl(k * log2e - ref) (one fused
//    multiply-add), so exponents have the size of the key range.
//  * the decay is counted, not accumulated: while the past keeps the maximum
//    only the step count n grows, and P is formed with one fused
//    multiply-add whenever it is needed (repeated P -= w2 would drift by up to
//    half an ulp per step, always in the same direction).
//  * each max-pair costs one ex2 and a select (one of its exponents is 0).
// u2 = u * log2e, w2 = w * log2e. For token t with kk:
//   absorb  z1 = kk - (P - w2), f = 2^{-|z1|}, (f1, f2) = (1, f) if z1 <= 0
//           else (f, 1);  aa <- f2 v + fl(f1 aa),  bb <- f1 bb + f2 (each
//           one fused multiply-add), and
//           (base, n) <- (base, n + 1) if z1 <= 0 else (kk, 0). The choices
//           are made with a 0/1 float mask (keep_mask) in exact fused
//           multiply-adds rather than selects.
//   output  the weight of the current token against the past is
//           e = 2^{zo}, zo = (u2 + kk) - P, and y = (aa + e v) / (bb + e).
//           It is formed in one of two ways, chosen per channel pair from
//           u2 - w2 alone (so every kernel makes the same choice):
//    * scaled (|u2 - w2| <= kScaledSpan): zo = z1 + (u2 - w2), so
//      e = 2^{z1} E with the channel constant E = 2^{u2 - w2}; numerator and
//      denominator multiplied by f1 give
//          y = (f1 aa + f2 E v) / (f1 bb + f2 E),
//      which reuses f1 aa and f1 bb of the absorb and needs no second ex2.
//      The denominator is >= bb >= 1 (z1 <= 0, a token absorbed before) or
//      >= E >= 2^-kScaledSpan (z1 > 0), so it never vanishes; a term that
//      underflows to zero (f below 2^-126) is below 2^-68 of the other.
//    * exact (any u2 - w2): e = 2^{min(zo, 64)} from a second ex2 (bb >= 1
//      once a token is absorbed and bb <= number of tokens, so beyond 2^64
//      the past is far below float32 resolution of the sum; the empty past,
//      aa = bb = 0, gives y = v).
// All roundings are explicit (_rn intrinsics) so that every kernel that runs
// this step produces bit-identical results from the same state and inputs;
// a sum of a product is always written as one fused multiply-add (the packed
// pair forms of a separate multiply and add were measured to come out fused
// in some places and not in others).
// ----------------------------------------------------------------------------
struct Wkv4State {
  float aa, bb, base, n;
};

// 1.0f when z <= 0 (the decayed past keeps the maximum), else 0.0f: the PTX
// set instruction writes the float mask directly, and the step's selects
// become exact fused multiply-adds with it (one of the two products is an
// exact zero, the other an exact copy), which run on the FMA pipe instead of
// the select unit.
__device__ __forceinline__ float keep_mask(float z) {
  float r;
  asm("set.le.f32.f32 %0, %1, 0f00000000;" : "=f"(r) : "f"(z));
  return r;
}

// |u2 - w2| (base 2) up to which the scaled output form is used: E and 1/E
// stay within 2^57, far from float32 overflow and underflow.
constexpr float kScaledSpan = 57.f;

__device__ __forceinline__ Wkv4State wkv4_empty_state() { return {0.f, 0.f, kEmptyPP, 0.f}; }

// Reference exponent of a lane whose first absorbed key is k_first.
__device__ __forceinline__ float wkv4_ref(float k_first) { return __fmul_rn(k_first, kLog2e); }

// Key in base-2 units relative to the lane reference.
__device__ __forceinline__ float wkv4_key(float k, float ref) { return __fmaf_rn(k, kLog2e, -ref); }

// Exponent P of the past sums (one rounding).
__device__ __forceinline__ float wkv4_exponent(const Wkv4State& s, float w2) {
  return __fmaf_rn(-s.n, w2, s.base);
}

// Output form of the channel pair (c, c + 1) with base-2 rates (u2, w2) of
// each: scaled iff both channels are within kScaledSpan. Every kernel decides
// per pair, so a channel's results do not depend on how a kernel groups them.
__device__ __forceinline__ bool wkv4_scaled_pair(float u2a, float w2a, float u2b, float w2b) {
  return fabsf(__fsub_rn(u2a, w2a)) <= kScaledSpan && fabsf(__fsub_rn(u2b, w2b)) <= kScaledSpan;
}
// The channel constant E = 2^{u2 - w2} of the scaled form.
__device__ __forceinline__ float wkv4_out_scale(float u2, float w2) { return ex2(__fsub_rn(u2, w2)); }

// Output of the token, then absorb it. Returns y. scaled: the pair's output
// form (wkv4_scaled_pair), E its channel constant.
__device__ __forceinline__ float wkv4_token(Wkv4State& s, float kk, float v, float u2, float w2, bool scaled,
                                            float E) {
  const float y0 = __fsub_rn(kk, s.base);
  const float n1 = __fadd_rn(s.n, 1.f);
  const float z1 = __fmaf_rn(n1, w2, y0);
  const float ea = ex2(-fabsf(z1));
  const float pk = keep_mask(z1), nk = __fmaf_rn(pk, -1.f, 1.f);
  const float f1 = __fmaf_rn(nk, ea, pk);  // 1 if the past keeps the maximum, else ea
  const float f2 = __fmaf_rn(pk, ea, nk);  // ea if it does, else 1
  const float t1 = __fmul_rn(f1, s.aa);
  float num, den;
  if (scaled) {
    const float g = __fmul_rn(f2, E);
    num = __fmaf_rn(g, v, t1);
    den = __fmaf_rn(f1, s.bb, g);
  } else {
    const float zo = __fmaf_rn(s.n, w2, __fadd_rn(y0, u2));
    const float e = ex2(fminf(zo, 64.f));
    num = __fmaf_rn(e, v, s.aa);
    den = __fadd_rn(s.bb, e);
  }
  s.aa = __fmaf_rn(f2, v, t1);
  s.bb = __fmaf_rn(f1, s.bb, f2);
  s.base = __fmaf_rn(nk, kk, __fmul_rn(pk, s.base));  // base if kept, else kk
  s.n = __fmul_rn(pk, n1);                            // n + 1 if kept, else 0
  return __fmul_rn(num, rcp(den));
}

// Merge two states of the same lane given in the same reference: the result
// represents the sum of both (max-combine of their exponents P1, P2).
struct Wkv4Sum {
  float aa, bb, P;
};
__device__ __forceinline__ Wkv4Sum wkv4_merge(const Wkv4Sum& x, const Wkv4Sum& y) {
  const float d = __fsub_rn(x.P, y.P);
  const float e = ex2(-fabsf(d));
  const bool xm = d >= 0.f;
  const float fx = xm ? 1.f : e;
  const float fy = xm ? e : 1.f;
  return {__fmaf_rn(fx, x.aa, __fmul_rn(fy, y.aa)), __fmaf_rn(fx, x.bb, __fmul_rn(fy, y.bb)), xm ? x.P : y.P};
}

// Absorb only (no output): the same state update as wkv4_token.
__device__ __forceinline__ void wkv4_absorb(Wkv4State& s, float kk, float v, float w2) {
  const float y0 = __fsub_rn(kk, s.base);
  const float n1 = __fadd_rn(s.n, 1.f);
  const float z1 = __fmaf_rn(n1, w2, y0);
  const float ea = ex2(-fabsf(z1));
  const float pk = keep_mask(z1), nk = __fmaf_rn(pk, -1.f, 1.f);
  const float f1 = __fmaf_rn(nk, ea, pk);
  const float f2 = __fmaf_rn(pk, ea, nk);
  s.aa = __fmaf_rn(f2, v, __fmul_rn(f1, s.aa));
  s.bb = __fmaf_rn(f1, s.bb, f2);
  s.base = __fmaf_rn(nk, kk, __fmul_rn(pk, s.base));
  s.n = __fmul_rn(pk, n1);
}

// ----------------------------------------------------------------------------
// Two channels per lane. The RWKV-4 kernels give each lane an adjacent pair
// of channels and run the step above on float2 with the packed fp32 pair
// instructions of sm_100 (FFMA2 / FADD2 / FMUL2 behind __ffma2_rn and
// friends): one issue slot does the arithmetic of both channels, and every
// component is rounded exactly as its scalar counterpart, so a pair step is
// bit for bit two scalar steps. k, v and y move as 4-byte (bf16) or 8-byte
// (float32) pairs. C is even (see the ABI), so a pair never straddles C.
// ----------------------------------------------------------------------------
__device__ __forceinline__ float2 splat2(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
// a - b with one rounding: fma(b, -1, a) is exact before it rounds, so it
// equals the scalar __fsub_rn(a, b)
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.f, -1.f), a); }
__device__ __forceinline__ float2 ex2_2(float2 a) { return make_float2(ex2(a.x), ex2(a.y)); }
__device__ __forceinline__ float2 rcp2(float2 a) { return make_float2(rcp(a.x), rcp(a.y)); }

// sigmoid(x) = 1 / (1 + 2^{-x log2 e}) of a pair
__device__ __forceinline__ float2 sigmoid2(float2 x) {
  const float2 e = make_float2(ex2(__fmul_rn(-x.x, kLog2e)), ex2(__fmul_rn(-x.y, kLog2e)));
  return rcp2(add2(e, splat2(1.f)));
}

__device__ __forceinline__ float2 ld_pair(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ float2 ld_pair(const __nv_bfloat16* p) {
  const uint32_t x = *reinterpret_cast<const uint32_t*>(p);  // channel c in the low half
  return make_float2(__uint_as_float(x << 16), __uint_as_float(x & 0xFFFF0000u));
}
__device__ __forceinline__ void st_pair(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }
__device__ __forceinline__ void st_pair(__nv_bfloat16* p, float2 v) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v.x, v.y);
}

// A compile-time bool as a value (for generic lambdas that instantiate a
// loop per flag).
template <bool V>
struct BoolConst {
  static constexpr bool value = V;
};

struct Wkv4State2 {
  float2 aa, bb, base, n;
};

__device__ __forceinline__ Wkv4State2 wkv4_empty_state2() {
  return {splat2(0.f), splat2(0.f), splat2(kEmptyPP), splat2(0.f)};
}
__device__ __forceinline__ float2 wkv4_key2(float2 k, float2 ref) {
  return fma2(k, splat2(kLog2e), make_float2(-ref.x, -ref.y));
}
__device__ __forceinline__ float2 wkv4_exponent2(const Wkv4State2& s, float2 w2) {
  return fma2(make_float2(-s.n.x, -s.n.y), w2, s.base);
}
__device__ __forceinline__ float2 keep_mask2(float2 z) { return make_float2(keep_mask(z.x), keep_mask(z.y)); }
__device__ __forceinline__ bool wkv4_scaled_pair2(float2 u2, float2 w2) {
  return wkv4_scaled_pair(u2.x, w2.x, u2.y, w2.y);
}
__device__ __forceinline__ float2 wkv4_out_scale2(float2 u2, float2 w2) {
  return make_float2(wkv4_out_scale(u2.x, w2.x), wkv4_out_scale(u2.y, w2.y));
}

// The step of a pair split in two halves, so that a kernel can run the
// exponent chain of a group of tokens ahead of their value updates (the
// chain is the only part whose latency carries from token to token that
// involves more than one instruction; the halves together are wkv4_token
// on each channel, operation for operation).
// First half: the absorb exponent z1 of the token (and, for the exact output
// form, zo), advancing (base, n).
// MASK: make the choices with the float mask (keep_mask) on the FMA pipe;
// otherwise with predicates and selects. Both give the same values (the
// masked forms are exact; at most the sign of a zero base differs, which no
// later operation can see): the forward, bound by its select unit, takes the
// masks, the backward's recompute, bound by the latency of this chain, the
// two-instruction select path.
template <bool SCALED, bool MASK = true>
__device__ __forceinline__ float2 wkv4_chain2(Wkv4State2& s, float2 kk, float2 u2, float2 w2, float2& zo) {
  const float2 y0 = sub2(kk, s.base);
  if constexpr (!SCALED) zo = fma2(s.n, w2, add2(y0, u2));
  const float2 n1 = add2(s.n, splat2(1.f));
  const float2 z1 = fma2(n1, w2, y0);
  if constexpr (MASK) {
    const float2 pk = keep_mask2(z1), nk = fma2(pk, splat2(-1.f), splat2(1.f));
    s.base = fma2(nk, kk, mul2(pk, s.base));
    s.n = mul2(pk, n1);
  } else {
    const bool px = z1.x <= 0.f, py = z1.y <= 0.f;
    s.base = make_float2(px ? s.base.x : kk.x, py ? s.base.y : kk.y);
    s.n = make_float2(px ? n1.x : 0.f, py ? n1.y : 0.f);
  }
  return z1;
}
// Absorb factors (f1, f2) of a token with exponent z1.
template <bool MASK = true>
__device__ __forceinline__ void wkv4_factors2(float2 z1, float2& f1, float2& f2) {
  const float2 ea = make_float2(ex2(-fabsf(z1.x)), ex2(-fabsf(z1.y)));
  if constexpr (MASK) {
    const float2 pk = keep_mask2(z1), nk = fma2(pk, splat2(-1.f), splat2(1.f));
    f1 = fma2(nk, ea, pk);
    f2 = fma2(pk, ea, nk);
  } else {
    const bool px = z1.x <= 0.f, py = z1.y <= 0.f;
    f1 = make_float2(px ? 1.f : ea.x, py ? 1.f : ea.y);
    f2 = make_float2(px ? ea.x : 1.f, py ? ea.y : 1.f);
  }
}
// Second half: output of the token and the update of (aa, bb). E: the
// pair's channel constants (scaled form); zo from the first half (exact).
template <bool SCALED>
__device__ __forceinline__ float2 wkv4_values2(Wkv4State2& s, float2 z1, float2 zo, float2 v, float2 E) {
  float2 f1, f2;
  wkv4_factors2(z1, f1, f2);
  const float2 t1 = mul2(f1, s.aa);
  float2 num, den;
  if constexpr (SCALED) {
    const float2 g = mul2(f2, E);
    num = fma2(g, v, t1);
    den = fma2(f1, s.bb, g);
  } else {
    const float2 e = make_float2(ex2(fminf(zo.x, 64.f)), ex2(fminf(zo.y, 64.f)));
    num = fma2(e, v, s.aa);
    den = add2(s.bb, e);
  }
  s.aa = fma2(f2, v, t1);
  s.bb = fma2(f1, s.bb, f2);
  return mul2(num, rcp2(den));
}

// Pair form of wkv4_token (same operations in the same order).
template <bool SCALED>
__device__ __forceinline__ float2 wkv4_token2(Wkv4State2& s, float2 kk, float2 v, float2 u2, float2 w2, float2 E) {
  float2 zo = splat2(0.f);
  const float2 z1 = wkv4_chain2<SCALED>(s, kk, u2, w2, zo);
  return wkv4_values2<SCALED>(s, z1, zo, v, E);
}
__device__ __forceinline__ float2 wkv4_token2(Wkv4State2& s, float2 kk, float2 v, float2 u2, float2 w2, bool scaled,
                                              float2 E) {
  return scaled ? wkv4_token2<true>(s, kk, v, u2, w2, E) : wkv4_token2<false>(s, kk, v, u2, w2, E);
}

// Pair form of wkv4_absorb. Returns z1, the exponent of the token against
// the decayed past (2^{-|z1|} is the absorb factor; z1 <= 0 keeps the past's
// maximum), and the factors f1, f2.
template <bool MASK = true>
__device__ __forceinline__ float2 wkv4_absorb2(Wkv4State2& s, float2 kk, float2 v, float2 w2, float2& f1,
                                               float2& f2) {
  float2 unused;
  const float2 z1 = wkv4_chain2<true, MASK>(s, kk, splat2(0.f), w2, unused);
  wkv4_factors2<MASK>(z1, f1, f2);
  s.aa = fma2(f2, v, mul2(f1, s.aa));
  s.bb = fma2(f1, s.bb, f2);
  return z1;
}
template <bool MASK = true>
__device__ __forceinline__ float2 wkv4_absorb2(Wkv4State2& s, float2 kk, float2 v, float2 w2) {
  float2 f1, f2;
  return wkv4_absorb2<MASK>(s, kk, v, w2, f1, f2);
}

}  // namespace wkv
