// wkv_internal.h -- host-side interface between the C ABI layer (capi.cu) and
// the kernel launchers of each .cu file. Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "wkv.h"

namespace wkv {

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Encode a 3-D tiled TMA descriptor over a dense row-major tensor with
// dims {d0 (innermost), d1, d2} of `elem_bytes`-byte elements, box
// {b0, b1, b2}, no swizzle, out-of-bounds elements filled with zero.
// Returns false (with a message in *why) if the driver rejects it.
bool encode_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType type, size_t elem_bytes,
                    uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1, uint32_t b2,
                    const char** why);

struct Wkv4FwdArgs {
  int64_t B, T, C;
  int dtype;
  const float* w;
  const float* u;
  const void* k;
  const void* v;
  void* y;      // may be null
  float* ckpt;  // may be null
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
  float* part;  // [2][B][C] scratch
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
  void* o;
};

// Record `why` as the calling thread's wkv_last_error() message.
void set_last_error(const char* why);

// Each launcher enqueues its kernels on `stream` and returns WKV_OK or an
// error status with a static message in *why. `err` is the device error word.
wkv_status launch_wkv4_forward(const Wkv4FwdArgs& a, cudaStream_t stream, unsigned* err, const char** why);
wkv_status launch_wkv4_backward(const Wkv4BwdArgs& a, cudaStream_t stream, unsigned* err, const char** why);
wkv_status launch_wkv4_state_init(int64_t S, int64_t C, float* state, cudaStream_t stream, const char** why);
wkv_status launch_wkv4_chunk_step(const Wkv4ChunkArgs& a, cudaStream_t stream, unsigned* err, const char** why);
wkv_status launch_wkv6_forward(const Wkv6FwdArgs& a, cudaStream_t stream, unsigned* err, const char** why);

}  // namespace wkv
