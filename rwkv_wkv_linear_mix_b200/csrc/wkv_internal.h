// wkv_internal.h -- host-side interface between the C ABI layer (capi.cu) and
// the kernel launchers of each .cu file. Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <algorithm>

#include "wkv.h"

namespace wkv {

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Channels of one RWKV-4 warp (32 lanes x a channel pair each).
#define WKV4_WARP_CH 64

// Launch-shape constants of the RWKV-4 kernels (build-time tunables).
#ifndef WKV4_TARGET_WARPS
#define WKV4_TARGET_WARPS (148 * 4)  // warps wanted in flight: 4 per SM of a B200 (8 channels each)
#endif
#ifndef WKV4_FWD_MAX_SEGMENTS
#define WKV4_FWD_MAX_SEGMENTS 8
#endif
#ifndef WKV4_BWD_MAX_SEGMENTS
#define WKV4_BWD_MAX_SEGMENTS 8
#endif
// 16 segments (a non-portable cluster size) are compiled in only when one of
// the caps above allows them.
#define WKV4_MAX_SEGMENTS_ANY (WKV4_FWD_MAX_SEGMENTS > WKV4_BWD_MAX_SEGMENTS ? WKV4_FWD_MAX_SEGMENTS : WKV4_BWD_MAX_SEGMENTS)

// Number of sequence segments each RWKV-4 lane is split into (the cluster
// size of a kernel): doubled while the launch has fewer warps than
// WKV4_TARGET_WARPS and every segment keeps at least WKV4_MIN_SEG_STEPS
// steps (splitting reruns each segment, so short ones do not pay); at most
// max_seg (<= 16; above 8 a non-portable cluster size).
#ifndef WKV4_MIN_SEG_STEPS
#define WKV4_MIN_SEG_STEPS 64
#endif
inline int wkv4_segments_capped(int64_t B, int64_t T, int64_t C, int max_seg) {
  const int64_t groups = B * ceil_div(C, WKV4_WARP_CH);
  const int64_t steps = ceil_div(T, WKV4_CKPT_LEN) * WKV4_CKPT_LEN;
  int nseg = 1;
  while (nseg < max_seg && groups * nseg < (int64_t)(WKV4_TARGET_WARPS) && steps >= 2 * WKV4_MIN_SEG_STEPS * nseg)
    nseg *= 2;
  return nseg;
}
// Warps (independent 64-channel lane groups) per CTA of a split launch: the
// GPU keeps only ~140 clusters resident at once, so a split launch packs
// several lane groups into each CTA to stay within one wave of clusters.
#ifndef WKV4_MAX_CLUSTERS
#define WKV4_MAX_CLUSTERS 128
#endif
inline int wkv4_warps_per_cta(int64_t B, int64_t C, int nseg) {
  if (nseg == 1) return 1;
  const int64_t groups = B * ceil_div(C, WKV4_WARP_CH);
  int nw = 1;
  while (nw < 4 && ceil_div(groups, nw) > WKV4_MAX_CLUSTERS) nw *= 2;
  return nw;
}

inline int wkv4_fwd_segments(int64_t B, int64_t T, int64_t C) {
  return wkv4_segments_capped(B, T, C, WKV4_FWD_MAX_SEGMENTS);
}
inline int wkv4_bwd_segments(int64_t B, int64_t T, int64_t C) {
  return wkv4_segments_capped(B, T, C, WKV4_BWD_MAX_SEGMENTS);
}

// Segment s of nseg covers checkpoint intervals [seg_begin(s), seg_begin(s+1)).
__host__ __device__ __forceinline__ int wkv4_seg_begin(int s, int nseg, int nck) {
  return (int)(((int64_t)s * nck) / nseg);
}

// Encode a 3-D tiled TMA descriptor over a dense row-major tensor with
// dims {d0 (innermost), d1, d2} of `elem_bytes`-byte elements, box
// {b0, b1, b2}, out-of-bounds elements filled with zero. swizzle128: write
// the tile in the 128-byte-swizzled shared-memory layout (b0 * elem_bytes
// must then be 128 and the destination 1024-byte aligned); else unswizzled.
// Returns false (with a message in *why) if the driver rejects it.
bool encode_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType type, size_t elem_bytes,
                    uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1, uint32_t b2,
                    const char** why, bool swizzle128 = false);

struct Wkv4FwdArgs {
  int64_t B, T, C;
  int dtype;
  const float* w;
  const float* u;
  const void* k;
  const void* v;
  void* y;      // may be null
  float* ckpt;  // may be null
  const void* r = nullptr;  // gate input: y = sigmoid(r) * WKV (may be null: ungated)
};

struct Wkv4BwdArgs {
  int64_t B, T, C;
  int dtype;
  const float* w;
  const float* u;
  const void* k;
  const void* v;
  const void* gy;
  const float* ckpt;  // never null here
  void* gk;
  void* gv;
  float* gw;
  float* gu;
  float* part;  // [2][B * wkv4_bwd_segments(B, T, C)][C] scratch
  const void* r = nullptr;  // gate input (gy is then dL/d(sigmoid(r) * WKV)); null: ungated
  void* gr = nullptr;       // dL/dr, written when r is given
};

struct Wkv4ChunkArgs {
  int64_t S, C;
  int dtype;
  const float* w;
  const float* u;
  const void* k;
  const void* v;
  void* y;
  int64_t n_tokens;
  const int32_t* cu_tokens;
  float* state;
};

struct Wkv6FwdArgs {
  int64_t B, T, H, K;
  const void* r;
  const void* k;
  const void* v;
  const void* w;
  const float* u;
  const float* init_state;
  const int32_t* state_map;
  int64_t n_state;
  float* final_state;
  void* o;                   // may be null (no output written)
  float* ck_state = nullptr;  // [B*H][ceil(T/64)][64][64]: state entering each chunk (may be null)
  bool reverse = false;       // run the recurrence from the last token to the first
};

struct Wkv6BwdArgs {
  int64_t B, T, H, K;
  const void* r;
  const void* k;
  const void* v;
  const void* w;
  const float* u;
  const float* init_state;
  const int32_t* state_map;
  int64_t n_state;
  const void* dout;
  const float* g_final;
  void* gr;
  void* gk;
  void* gv;
  void* glogw;
  float* gu;
  float* g_init;
  void* workspace;
};
size_t wkv6_bwd_workspace_bytes(int64_t B, int64_t T, int64_t H);

struct Wkv7FwdArgs {
  int64_t B, T, H, K;
  const void* r;
  const void* w;
  const void* k;
  const void* v;
  const void* a;
  const void* b;
  const float* init_state;
  float* final_state;
  void* o;
  float* ckpt = nullptr;  // backward sweep: write state checkpoints, no o
};
// Tokens per RWKV-7 state checkpoint of the backward.
#define WKV7_CKPT_LEN 4
struct Wkv7BwdArgs {
  int64_t B, T, H;
  const void *r, *w, *k, *v, *a, *b, *dout;
  const float* ckpt;     // [B*H][ceil(T/4)][64][64], from the checkpoint sweep
  const float* g_final;  // may be null
  void *dr, *dw, *dk, *dv, *da, *db;
  float* d_init;
};
wkv_status launch_wkv7_backward(const Wkv7BwdArgs& a, cudaStream_t stream, const char** why);

// Record `why` as the calling thread's wkv_last_error() message.
void set_last_error(const char* why);

// Each launcher enqueues its kernels on `stream` and returns WKV_OK or an
// error status with a static message in *why. `err` is the device error word.
wkv_status launch_wkv4_forward(const Wkv4FwdArgs& a, cudaStream_t stream, unsigned* err, const char** why);
wkv_status launch_wkv4_backward(const Wkv4BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why);
wkv_status launch_wkv4_state_init(int64_t S, int64_t C, float* state, cudaStream_t stream, const char** why);
wkv_status launch_wkv4_chunk_step(const Wkv4ChunkArgs& a, cudaStream_t stream, unsigned* err, const char** why);
// One token per slot: k, v, y [S][C], state [S][5][C].
wkv_status launch_wkv4_decode_step(int64_t S, int64_t C, int dtype, const float* w, const float* u, const void* k,
                                   const void* v, void* y, float* state, cudaStream_t stream, const char** why);
wkv_status launch_wkv6_forward(const Wkv6FwdArgs& a, cudaStream_t stream, unsigned* err, const char** why);
wkv_status launch_wkv6_backward(const Wkv6BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why);
wkv_status launch_wkv7_forward(const Wkv7FwdArgs& a, cudaStream_t stream, unsigned* err, const char** why);

// Time-shift mix (time-mix prologue). out / g: [n_mix][B][T][C]; mix, gmix:
// [n_mix][C] float32; x_prev, gx_prev: [B][C] (may be null); part: the
// backward's partial sums, [n_mix][B * nrun][C] float32.
struct TimeShiftArgs {
  int64_t B, T, C;
  int dtype;
  int n_mix;
  const void* x;
  const float* mix;
  const void* x_prev;
  void* out;
  const void* g;
  void* gx;
  float* gmix;
  void* gx_prev;
  float* part;
};
// Launch shape: channel blocks of 128 threads x `vec` channels, and each
// sequence cut into nrun runs of Lt tokens.
struct TsShape {
  int ncb, nrun, Lt;
};
TsShape time_shift_shape(int64_t B, int64_t T, int64_t C, int vec);
// Channels per thread of the backward kernel (bf16: 4 or 8; float32: 4) and
// tokens per batch of loads of each kernel (a batch is loaded, still packed,
// before any of it is used).
#ifndef TS_BWD_BF16_VEC
#define TS_BWD_BF16_VEC 4
#endif
#ifndef TS_BWD_U
#define TS_BWD_U 8
#endif
#ifndef TS_FWD_U
#define TS_FWD_U 4
#endif
inline int time_shift_bwd_vec(int dtype) { return dtype == WKV_BF16 ? TS_BWD_BF16_VEC : 4; }
wkv_status launch_time_shift_mix(const TimeShiftArgs& a, cudaStream_t stream, const char** why);
wkv_status launch_time_shift_mix_backward(const TimeShiftArgs& a, cudaStream_t stream, const char** why);
wkv_status launch_wait_selfcheck(int64_t limit_ns, cudaStream_t stream, unsigned* err, const char** why);

}  // namespace wkv
