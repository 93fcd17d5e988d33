// capi.cu -- the C ABI of libwkv_b200.so (declared in include/wkv.h).
//
// Every entry point validates its arguments on the host, encodes the TMA
// descriptors it needs and enqueues the kernels on the caller's stream. It
// never allocates, never synchronises (except wkv_device_error, which says
// so), and turns every failure into a wkv_status plus a per-thread message.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "wkv.h"
#include "wkv_internal.h"

#define WKV_EXPORT extern "C" __attribute__((visibility("default")))

namespace wkv {

// Device-side error word (WKV_DEVERR_* bits), one per device that loads the
// library. Kernels receive its address and OR codes into it.
__device__ unsigned int g_device_error;

namespace {

thread_local const char* t_last_error = "";

wkv_status fail(wkv_status s, const char* why) {
  t_last_error = why ? why : "";
  return s;
}

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned* g_err_ptr[kMaxDevices] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Address of g_device_error on the current device (looked up once per device).
wkv_status device_error_ptr(unsigned** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return fail(WKV_ERR_CUDA, "cudaGetDevice failed");
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess || !p)
      return fail(WKV_ERR_CUDA, "cudaGetSymbolAddress(g_device_error) failed");
    g_err_ptr[dev] = static_cast<unsigned*>(p);
  }
  *out = g_err_ptr[dev];
  return WKV_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  return g_encode;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shared checks of the activation shape and storage type.
wkv_status check_act(int64_t B, int64_t T, int64_t C, int dtype) {
  if (B < 0 || T < 0 || C < 0) return fail(WKV_ERR_INVALID_ARG, "negative size");
  if (dtype != WKV_F32 && dtype != WKV_BF16) return fail(WKV_ERR_INVALID_ARG, "unknown dtype");
  if ((dtype == WKV_F32 && C % 4) || (dtype == WKV_BF16 && C % 8))
    return fail(WKV_ERR_UNSUPPORTED, "C must be a multiple of 4 (f32) or 8 (bf16)");
  if (T > INT32_MAX || C > INT32_MAX || B > INT32_MAX) return fail(WKV_ERR_UNSUPPORTED, "size above 2^31-1");
  const int64_t ncb = (C + 31) / 32;
  if (B > 0 && ncb > 0 && ncb * B > INT32_MAX) return fail(WKV_ERR_UNSUPPORTED, "B * ceil(C/32) above 2^31-1");
  return WKV_OK;
}

#define WKV_REQUIRE_PTR(p, name)                                                         \
  do {                                                                                   \
    if (!(p)) return fail(WKV_ERR_INVALID_ARG, name " is NULL");                         \
    if (!aligned16(p)) return fail(WKV_ERR_INVALID_ARG, name " is not 16-byte aligned"); \
  } while (0)

#define WKV_OPTIONAL_PTR(p, name) \
  do {                            \
    if ((p) && !aligned16(p)) return fail(WKV_ERR_INVALID_ARG, name " is not 16-byte aligned"); \
  } while (0)

}  // namespace

void set_last_error(const char* why) { t_last_error = why ? why : ""; }

bool encode_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType type, size_t elem_bytes, uint64_t d0,
                    uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1, uint32_t b2, const char** why,
                    bool swizzle128) {
  auto fn = encode_fn();
  if (!fn) {
    *why = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * elem_bytes, d0 * d1 * elem_bytes};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, type, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *why = "cuTensorMapEncodeTiled rejected the tensor";
    return false;
  }
  return true;
}

}  // namespace wkv

using namespace wkv;

WKV_EXPORT int wkv_abi_version(void) { return WKV_ABI_VERSION; }

WKV_EXPORT const char* wkv_status_string(int status) {
  switch (status) {
    case WKV_OK: return "WKV_OK";
    case WKV_ERR_INVALID_ARG: return "WKV_ERR_INVALID_ARG";
    case WKV_ERR_UNSUPPORTED: return "WKV_ERR_UNSUPPORTED";
    case WKV_ERR_CUDA: return "WKV_ERR_CUDA";
    case WKV_ERR_DEVICE: return "WKV_ERR_DEVICE";
    default: return "WKV_ERR_UNKNOWN";
  }
}

WKV_EXPORT const char* wkv_last_error(void) { return t_last_error; }

WKV_EXPORT wkv_status wkv_device_error(uint32_t* code, int reset) {
  if (!code) return fail(WKV_ERR_INVALID_ARG, "code is NULL");
  unsigned* p = nullptr;
  if (wkv_status s = device_error_ptr(&p)) return s;
  unsigned h = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return fail(WKV_ERR_CUDA, "cudaDeviceSynchronize failed");
  if (cudaMemcpy(&h, p, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
    return fail(WKV_ERR_CUDA, "reading the device error word failed");
  if (reset) {
    const unsigned z = 0;
    if (cudaMemcpy(p, &z, sizeof(z), cudaMemcpyHostToDevice) != cudaSuccess)
      return fail(WKV_ERR_CUDA, "clearing the device error word failed");
  }
  *code = h;
  return WKV_OK;
}

WKV_EXPORT size_t wkv4_ckpt_floats(int64_t B, int64_t T, int64_t C) {
  if (B <= 0 || T <= 0 || C <= 0) return 0;
  return (size_t)B * (size_t)ceil_div(T, WKV4_CKPT_LEN) * 3u * (size_t)C;
}

// r: the gate input of the gated entry point, null for the plain one
static wkv_status wkv4_forward_any(int64_t B, int64_t T, int64_t C, int dtype, const float* w, const float* u,
                                   const void* k, const void* v, const void* r, void* y, float* ckpt, void* stream) {
  if (wkv_status s = check_act(B, T, C, dtype)) return s;
  if (B == 0 || T == 0 || C == 0) return WKV_OK;
  WKV_REQUIRE_PTR(w, "w");
  WKV_REQUIRE_PTR(u, "u");
  WKV_REQUIRE_PTR(k, "k");
  WKV_REQUIRE_PTR(v, "v");
  WKV_OPTIONAL_PTR(y, "y");
  WKV_OPTIONAL_PTR(ckpt, "ckpt");
  if (!y && !ckpt) return fail(WKV_ERR_INVALID_ARG, "y and ckpt are both NULL");
  unsigned* err = nullptr;
  if (wkv_status s = device_error_ptr(&err)) return s;
  const char* why = "";
  Wkv4FwdArgs a{B, T, C, dtype, w, u, k, v, y, ckpt};
  a.r = y ? r : nullptr;  // without y there is nothing to gate
  wkv_status s = launch_wkv4_forward(a, static_cast<cudaStream_t>(stream), err, &why);
  return s == WKV_OK ? s : fail(s, why);
}

WKV_EXPORT wkv_status wkv4_forward(int64_t B, int64_t T, int64_t C, int dtype, const float* w, const float* u,
                                   const void* k, const void* v, void* y, float* ckpt, void* stream) {
  return wkv4_forward_any(B, T, C, dtype, w, u, k, v, nullptr, y, ckpt, stream);
}

WKV_EXPORT wkv_status wkv4_forward_gated(int64_t B, int64_t T, int64_t C, int dtype, const float* w,
                                         const float* u, const void* k, const void* v, const void* r, void* y,
                                         float* ckpt, void* stream) {
  if (wkv_status s = check_act(B, T, C, dtype)) return s;
  if (B > 0 && T > 0 && C > 0) {
    WKV_REQUIRE_PTR(r, "r");
    WKV_REQUIRE_PTR(y, "y");
  }
  return wkv4_forward_any(B, T, C, dtype, w, u, k, v, r, y, ckpt, stream);
}

WKV_EXPORT size_t wkv4_backward_workspace_bytes(int64_t B, int64_t T, int64_t C, int has_ckpt) {
  if (B <= 0 || T <= 0 || C <= 0) return 0;
  // gw/gu partial sums per (sample, sequence segment, channel)
  size_t bytes = 2u * (size_t)B * (size_t)wkv4_bwd_segments(B, T, C) * (size_t)C * sizeof(float);
  bytes = (bytes + 255) & ~(size_t)255;
  if (!has_ckpt) bytes += wkv4_ckpt_floats(B, T, C) * sizeof(float);
  return bytes;
}

// r, gr: the gate input and its gradient (gated entry point), null otherwise
static wkv_status wkv4_backward_any(int64_t B, int64_t T, int64_t C, int dtype, const float* w, const float* u,
                                    const void* k, const void* v, const void* r, const void* gy, const float* ckpt,
                                    void* gk, void* gv, void* gr, float* gw, float* gu, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (wkv_status s = check_act(B, T, C, dtype)) return s;
  if (C == 0) return WKV_OK;
  WKV_REQUIRE_PTR(gw, "gw");
  WKV_REQUIRE_PTR(gu, "gu");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (B == 0 || T == 0) {
    // nothing flows back: the parameter gradients are zero
    if (cudaMemsetAsync(gw, 0, C * sizeof(float), st) != cudaSuccess ||
        cudaMemsetAsync(gu, 0, C * sizeof(float), st) != cudaSuccess)
      return fail(WKV_ERR_CUDA, "cudaMemsetAsync failed");
    return WKV_OK;
  }
  WKV_REQUIRE_PTR(w, "w");
  WKV_REQUIRE_PTR(u, "u");
  WKV_REQUIRE_PTR(k, "k");
  WKV_REQUIRE_PTR(v, "v");
  WKV_REQUIRE_PTR(gy, "gy");
  WKV_OPTIONAL_PTR(ckpt, "ckpt");
  WKV_REQUIRE_PTR(gk, "gk");
  WKV_REQUIRE_PTR(gv, "gv");
  WKV_REQUIRE_PTR(workspace, "workspace");
  if (workspace_bytes < wkv4_backward_workspace_bytes(B, T, C, ckpt != nullptr))
    return fail(WKV_ERR_INVALID_ARG, "workspace_bytes below wkv4_backward_workspace_bytes()");
  unsigned* err = nullptr;
  if (wkv_status s = device_error_ptr(&err)) return s;
  const char* why = "";
  float* part = static_cast<float*>(workspace);
  const float* ck = ckpt;
  if (!ck) {
    size_t off = (2u * (size_t)B * (size_t)wkv4_bwd_segments(B, T, C) * (size_t)C * sizeof(float) + 255) & ~(size_t)255;
    float* regen = reinterpret_cast<float*>(static_cast<char*>(workspace) + off);
    Wkv4FwdArgs fa{B, T, C, dtype, w, u, k, v, nullptr, regen};
    if (wkv_status s = launch_wkv4_forward(fa, st, err, &why)) return fail(s, why);
    ck = regen;
  }
  Wkv4BwdArgs a{B, T, C, dtype, w, u, k, v, gy, ck, gk, gv, gw, gu, part};
  a.r = r;
  a.gr = gr;
  wkv_status s = launch_wkv4_backward(a, st, err, &why);
  return s == WKV_OK ? s : fail(s, why);
}

WKV_EXPORT wkv_status wkv4_backward(int64_t B, int64_t T, int64_t C, int dtype, const float* w, const float* u,
                                    const void* k, const void* v, const void* gy, const float* ckpt, void* gk,
                                    void* gv, float* gw, float* gu, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  return wkv4_backward_any(B, T, C, dtype, w, u, k, v, nullptr, gy, ckpt, gk, gv, nullptr, gw, gu, workspace,
                           workspace_bytes, stream);
}

WKV_EXPORT wkv_status wkv4_backward_gated(int64_t B, int64_t T, int64_t C, int dtype, const float* w,
                                          const float* u, const void* k, const void* v, const void* r,
                                          const void* gy, const float* ckpt, void* gk, void* gv, void* gr,
                                          float* gw, float* gu, void* workspace, size_t workspace_bytes,
                                          void* stream) {
  if (wkv_status s = check_act(B, T, C, dtype)) return s;
  if (B > 0 && T > 0 && C > 0) {
    WKV_REQUIRE_PTR(r, "r");
    WKV_REQUIRE_PTR(gr, "gr");
  }
  return wkv4_backward_any(B, T, C, dtype, w, u, k, v, r, gy, ckpt, gk, gv, gr, gw, gu, workspace, workspace_bytes,
                           stream);
}

WKV_EXPORT wkv_status wkv4_state_init(int64_t S, int64_t C, float* state, void* stream) {
  if (S < 0 || C < 0) return fail(WKV_ERR_INVALID_ARG, "negative size");
  if (S == 0 || C == 0) return WKV_OK;
  if (C > INT32_MAX) return fail(WKV_ERR_UNSUPPORTED, "C above 2^31-1");
  WKV_REQUIRE_PTR(state, "state");
  const char* why = "";
  wkv_status s = launch_wkv4_state_init(S, C, state, static_cast<cudaStream_t>(stream), &why);
  return s == WKV_OK ? s : fail(s, why);
}

WKV_EXPORT wkv_status wkv4_chunk_step(int64_t S, int64_t C, int dtype, const float* w, const float* u, const void* k,
                                      const void* v, void* y, int64_t n_tokens, const int32_t* cu_tokens,
                                      float* state, void* stream) {
  if (n_tokens < 0) return fail(WKV_ERR_INVALID_ARG, "negative n_tokens");
  if (wkv_status s = check_act(S, 1, C, dtype)) return s;
  if (S == 0 || C == 0) return WKV_OK;
  WKV_REQUIRE_PTR(w, "w");
  WKV_REQUIRE_PTR(u, "u");
  WKV_REQUIRE_PTR(cu_tokens, "cu_tokens");
  WKV_REQUIRE_PTR(state, "state");
  if (n_tokens > 0) {
    WKV_REQUIRE_PTR(k, "k");
    WKV_REQUIRE_PTR(v, "v");
    WKV_REQUIRE_PTR(y, "y");
  }
  unsigned* err = nullptr;
  if (wkv_status s = device_error_ptr(&err)) return s;
  const char* why = "";
  Wkv4ChunkArgs a{S, C, dtype, w, u, k, v, y, n_tokens, cu_tokens, state};
  wkv_status s = launch_wkv4_chunk_step(a, static_cast<cudaStream_t>(stream), err, &why);
  return s == WKV_OK ? s : fail(s, why);
}

WKV_EXPORT wkv_status wkv4_decode_step(int64_t S, int64_t C, int dtype, const float* w, const float* u,
                                       const void* k, const void* v, void* y, float* state, void* stream) {
  if (wkv_status s = check_act(S, 1, C, dtype)) return s;
  if (S == 0 || C == 0) return WKV_OK;
  WKV_REQUIRE_PTR(w, "w");
  WKV_REQUIRE_PTR(u, "u");
  WKV_REQUIRE_PTR(k, "k");
  WKV_REQUIRE_PTR(v, "v");
  WKV_REQUIRE_PTR(y, "y");
  WKV_REQUIRE_PTR(state, "state");
  const char* why = "";
  wkv_status s = launch_wkv4_decode_step(S, C, dtype, w, u, k, v, y, state, static_cast<cudaStream_t>(stream), &why);
  return s == WKV_OK ? s : fail(s, why);
}

WKV_EXPORT wkv_status wkv6_forward(int64_t B, int64_t T, int64_t H, int64_t K, int dtype, const void* r,
                                   const void* k, const void* v, const void* w, const float* u,
                                   const float* init_state, const int32_t* state_map, int64_t n_state,
                                   float* final_state, void* o, void* stream) {
  if (B < 0 || T < 0 || H < 0 || K < 0 || n_state < 0) return fail(WKV_ERR_INVALID_ARG, "negative size");
  if (dtype != WKV_F32 && dtype != WKV_BF16) return fail(WKV_ERR_INVALID_ARG, "unknown dtype");
  if (dtype != WKV_BF16) return fail(WKV_ERR_UNSUPPORTED, "wkv6_forward supports bf16 only");
  if (K != 64) return fail(WKV_ERR_UNSUPPORTED, "wkv6_forward supports head size 64 only");
  if (B == 0 || H == 0) return WKV_OK;
  if (T > INT32_MAX || H > 65535 || B * H > INT32_MAX) return fail(WKV_ERR_UNSUPPORTED, "size out of range");
  WKV_REQUIRE_PTR(u, "u");
  WKV_OPTIONAL_PTR(final_state, "final_state");
  WKV_OPTIONAL_PTR(init_state, "init_state");
  WKV_OPTIONAL_PTR(state_map, "state_map");
  if (init_state) {
    if (n_state < 1) return fail(WKV_ERR_INVALID_ARG, "init_state given with n_state < 1");
    if (!state_map && n_state != 1 && n_state != B)
      return fail(WKV_ERR_INVALID_ARG, "without state_map, n_state must be 1 or B");
  }
  if (T > 0) {
    WKV_REQUIRE_PTR(r, "r");
    WKV_REQUIRE_PTR(k, "k");
    WKV_REQUIRE_PTR(v, "v");
    WKV_REQUIRE_PTR(w, "w");
    WKV_REQUIRE_PTR(o, "o");
  }
  unsigned* err = nullptr;
  if (wkv_status s = device_error_ptr(&err)) return s;
  const char* why = "";
  Wkv6FwdArgs a{B, T, H, K, r, k, v, w, u, init_state, state_map, init_state ? n_state : 0, final_state, o};
  wkv_status s = launch_wkv6_forward(a, static_cast<cudaStream_t>(stream), err, &why);
  return s == WKV_OK ? s : fail(s, why);
}

WKV_EXPORT wkv_status wkv7_forward(int64_t B, int64_t T, int64_t H, int64_t K, int dtype, const void* r,
                                   const void* w, const void* k, const void* v, const void* a, const void* b,
                                   const float* init_state, float* final_state, void* o, void* stream) {
  if (B < 0 || T < 0 || H < 0 || K < 0) return fail(WKV_ERR_INVALID_ARG, "negative size");
  if (dtype != WKV_F32 && dtype != WKV_BF16) return fail(WKV_ERR_INVALID_ARG, "unknown dtype");
  if (dtype != WKV_BF16) return fail(WKV_ERR_UNSUPPORTED, "wkv7_forward supports bf16 only");
  if (K != 64) return fail(WKV_ERR_UNSUPPORTED, "wkv7_forward supports head size 64 only");
  if (B == 0 || H == 0) return WKV_OK;
  if (T > INT32_MAX || H > 65535 || B * H > INT32_MAX) return fail(WKV_ERR_UNSUPPORTED, "size out of range");
  WKV_OPTIONAL_PTR(init_state, "init_state");
  WKV_OPTIONAL_PTR(final_state, "final_state");
  if (T > 0) {
    WKV_REQUIRE_PTR(r, "r");
    WKV_REQUIRE_PTR(w, "w");
    WKV_REQUIRE_PTR(k, "k");
    WKV_REQUIRE_PTR(v, "v");
    WKV_REQUIRE_PTR(a, "a");
    WKV_REQUIRE_PTR(b, "b");
    WKV_REQUIRE_PTR(o, "o");
  }
  unsigned* err = nullptr;
  if (wkv_status s = device_error_ptr(&err)) return s;
  const char* why = "";
  Wkv7FwdArgs args{B, T, H, K, r, w, k, v, a, b, init_state, final_state, o};
  wkv_status s = launch_wkv7_forward(args, static_cast<cudaStream_t>(stream), err, &why);
  return s == WKV_OK ? s : fail(s, why);
}

WKV_EXPORT size_t wkv7_backward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t K) {
  if (B <= 0 || T <= 0 || H <= 0 || K != 64) return 0;
  return (size_t)B * (size_t)H * (size_t)ceil_div(T, WKV7_CKPT_LEN) * 64u * 64u * sizeof(float);
}

WKV_EXPORT wkv_status wkv7_backward(int64_t B, int64_t T, int64_t H, int64_t K, int dtype, const void* r,
                                    const void* w, const void* k, const void* v, const void* a, const void* b,
                                    const float* init_state, const void* dout, const float* g_final, void* dr,
                                    void* dw, void* dk, void* dv, void* da, void* db, float* d_init,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  if (B < 0 || T < 0 || H < 0 || K < 0) return fail(WKV_ERR_INVALID_ARG, "negative size");
  if (dtype != WKV_F32 && dtype != WKV_BF16) return fail(WKV_ERR_INVALID_ARG, "unknown dtype");
  if (dtype != WKV_BF16) return fail(WKV_ERR_UNSUPPORTED, "wkv7_backward supports bf16 only");
  if (K != 64) return fail(WKV_ERR_UNSUPPORTED, "wkv7_backward supports head size 64 only");
  if (B == 0 || H == 0) return WKV_OK;
  if (T > INT32_MAX || H > 65535 || B * H > INT32_MAX) return fail(WKV_ERR_UNSUPPORTED, "size out of range");
  WKV_OPTIONAL_PTR(init_state, "init_state");
  WKV_OPTIONAL_PTR(g_final, "g_final");
  WKV_REQUIRE_PTR(d_init, "d_init");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t state_bytes = (size_t)B * (size_t)H * 64u * 64u * sizeof(float);
  if (T == 0) {
    // nothing flows through time: d_init = g_final (or 0)
    const cudaError_t e = g_final ? cudaMemcpyAsync(d_init, g_final, state_bytes, cudaMemcpyDeviceToDevice, st)
                                  : cudaMemsetAsync(d_init, 0, state_bytes, st);
    return e == cudaSuccess ? WKV_OK : fail(WKV_ERR_CUDA, "copy of g_final failed");
  }
  WKV_REQUIRE_PTR(r, "r");
  WKV_REQUIRE_PTR(w, "w");
  WKV_REQUIRE_PTR(k, "k");
  WKV_REQUIRE_PTR(v, "v");
  WKV_REQUIRE_PTR(a, "a");
  WKV_REQUIRE_PTR(b, "b");
  WKV_REQUIRE_PTR(dout, "dout");
  WKV_REQUIRE_PTR(dr, "dr");
  WKV_REQUIRE_PTR(dw, "dw");
  WKV_REQUIRE_PTR(dk, "dk");
  WKV_REQUIRE_PTR(dv, "dv");
  WKV_REQUIRE_PTR(da, "da");
  WKV_REQUIRE_PTR(db, "db");
  WKV_REQUIRE_PTR(workspace, "workspace");
  if (workspace_bytes < wkv7_backward_workspace_bytes(B, T, H, K))
    return fail(WKV_ERR_INVALID_ARG, "workspace_bytes below wkv7_backward_workspace_bytes()");
  unsigned* err = nullptr;
  if (wkv_status s = device_error_ptr(&err)) return s;
  const char* why = "";
  float* ck = static_cast<float*>(workspace);
  Wkv7FwdArgs fa{B, T, H, K, r, w, k, v, a, b, init_state, nullptr, nullptr};
  fa.ckpt = ck;
  if (wkv_status s = launch_wkv7_forward(fa, st, err, &why)) return fail(s, why);
  Wkv7BwdArgs ba{B, T, H, r, w, k, v, a, b, dout, ck, g_final, dr, dw, dk, dv, da, db, d_init};
  wkv_status s = launch_wkv7_backward(ba, st, &why);
  return s == WKV_OK ? s : fail(s, why);
}

WKV_EXPORT wkv_status wkv_wait_selfcheck(int64_t limit_ns, void* stream) {
  if (limit_ns < 1000 || limit_ns > 10000000000ll) return fail(WKV_ERR_INVALID_ARG, "limit_ns outside 1 us .. 10 s");
  unsigned* err = nullptr;
  if (wkv_status s = device_error_ptr(&err)) return s;
  const char* why = "";
  wkv_status s = launch_wait_selfcheck(limit_ns, static_cast<cudaStream_t>(stream), err, &why);
  return s == WKV_OK ? s : fail(s, why);
}

WKV_EXPORT size_t wkv6_backward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t K) {
  if (B < 0 || T < 0 || H < 0 || K != 64) return 0;
  return wkv6_bwd_workspace_bytes(B, T, H);
}

WKV_EXPORT wkv_status wkv6_backward(int64_t B, int64_t T, int64_t H, int64_t K, int dtype, const void* r,
                                    const void* k, const void* v, const void* w, const float* u,
                                    const float* init_state, const int32_t* state_map, int64_t n_state,
                                    const void* dout, const float* g_final, void* gr, void* gk, void* gv,
                                    void* glogw, float* gu, float* g_init, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (B < 0 || T < 0 || H < 0 || K < 0 || n_state < 0) return fail(WKV_ERR_INVALID_ARG, "negative size");
  if (dtype != WKV_F32 && dtype != WKV_BF16) return fail(WKV_ERR_INVALID_ARG, "unknown dtype");
  if (dtype != WKV_BF16) return fail(WKV_ERR_UNSUPPORTED, "wkv6_backward supports bf16 only");
  if (K != 64) return fail(WKV_ERR_UNSUPPORTED, "wkv6_backward supports head size 64 only");
  if (B == 0 || H == 0) return WKV_OK;
  if (T > INT32_MAX || H > 65535 || B * H > INT32_MAX) return fail(WKV_ERR_UNSUPPORTED, "size out of range");
  WKV_REQUIRE_PTR(u, "u");
  WKV_REQUIRE_PTR(gu, "gu");
  WKV_REQUIRE_PTR(workspace, "workspace");
  WKV_OPTIONAL_PTR(init_state, "init_state");
  WKV_OPTIONAL_PTR(state_map, "state_map");
  WKV_OPTIONAL_PTR(g_final, "g_final");
  WKV_OPTIONAL_PTR(g_init, "g_init");
  if (init_state) {
    if (n_state < 1) return fail(WKV_ERR_INVALID_ARG, "init_state given with n_state < 1");
    if (!state_map && n_state != 1 && n_state != B)
      return fail(WKV_ERR_INVALID_ARG, "without state_map, n_state must be 1 or B");
  }
  if (T > 0) {
    WKV_REQUIRE_PTR(r, "r");
    WKV_REQUIRE_PTR(k, "k");
    WKV_REQUIRE_PTR(v, "v");
    WKV_REQUIRE_PTR(w, "w");
    WKV_REQUIRE_PTR(dout, "dout");
    WKV_REQUIRE_PTR(gr, "gr");
    WKV_REQUIRE_PTR(gk, "gk");
    WKV_REQUIRE_PTR(gv, "gv");
    WKV_REQUIRE_PTR(glogw, "glogw");
  }
  if (workspace_bytes < wkv6_bwd_workspace_bytes(B, T, H)) return fail(WKV_ERR_INVALID_ARG, "workspace too small");
  unsigned* err = nullptr;
  if (wkv_status s = device_error_ptr(&err)) return s;
  const char* why = "";
  Wkv6BwdArgs a{B, T, H, K, r, k, v, w, u, init_state, state_map, init_state ? n_state : 0, dout, g_final,
                gr, gk, gv, glogw, gu, g_init, workspace};
  wkv_status s = launch_wkv6_backward(a, static_cast<cudaStream_t>(stream), err, &why);
  return s == WKV_OK ? s : fail(s, why);
}

// ---------------------------------------------------------------------------
// Time-shift mix (time-mix prologue)
// ---------------------------------------------------------------------------

WKV_EXPORT wkv_status wkv4_time_shift_mix(int64_t B, int64_t T, int64_t C, int dtype, int64_t n_mix, const void* x,
                                          const float* mix, const void* x_prev, void* out, void* stream) {
  if (wkv_status s = check_act(B, T, C, dtype)) return s;
  if (n_mix < 1 || n_mix > 3) return fail(WKV_ERR_INVALID_ARG, "n_mix must be 1, 2 or 3");
  if (B == 0 || T == 0 || C == 0) return WKV_OK;
  if (B * T * C * n_mix > ((int64_t)1 << 40)) return fail(WKV_ERR_UNSUPPORTED, "problem above 2^40 elements");
  WKV_REQUIRE_PTR(x, "x");
  WKV_REQUIRE_PTR(mix, "mix");
  WKV_OPTIONAL_PTR(x_prev, "x_prev");
  WKV_REQUIRE_PTR(out, "out");
  TimeShiftArgs a{B, T, C, dtype, (int)n_mix, x, mix, x_prev, out, nullptr, nullptr, nullptr, nullptr, nullptr};
  const char* why = "";
  wkv_status s = launch_time_shift_mix(a, static_cast<cudaStream_t>(stream), &why);
  return s == WKV_OK ? s : fail(s, why);
}

WKV_EXPORT size_t wkv4_time_shift_mix_backward_workspace_bytes(int64_t B, int64_t T, int64_t C, int dtype,
                                                               int64_t n_mix) {
  if (B <= 0 || T <= 0 || C <= 0 || n_mix < 1 || n_mix > 3 || (dtype != WKV_F32 && dtype != WKV_BF16)) return 0;
  const TsShape sh = time_shift_shape(B, T, C, time_shift_bwd_vec(dtype));
  return (size_t)n_mix * (size_t)B * (size_t)sh.nrun * (size_t)C * sizeof(float);
}

WKV_EXPORT wkv_status wkv4_time_shift_mix_backward(int64_t B, int64_t T, int64_t C, int dtype, int64_t n_mix,
                                                   const void* x, const float* mix, const void* x_prev,
                                                   const void* g, void* gx, float* gmix, void* gx_prev,
                                                   void* workspace, size_t workspace_bytes, void* stream) {
  if (wkv_status s = check_act(B, T, C, dtype)) return s;
  if (n_mix < 1 || n_mix > 3) return fail(WKV_ERR_INVALID_ARG, "n_mix must be 1, 2 or 3");
  if (C == 0) return WKV_OK;
  WKV_REQUIRE_PTR(gmix, "gmix");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (B == 0 || T == 0) {
    // nothing flows back: the mix gradients (and gx_prev) are zero
    WKV_OPTIONAL_PTR(gx_prev, "gx_prev");
    const size_t esz = dtype == WKV_BF16 ? 2 : 4;
    if (cudaMemsetAsync(gmix, 0, (size_t)n_mix * C * sizeof(float), st) != cudaSuccess ||
        (gx_prev && B > 0 && cudaMemsetAsync(gx_prev, 0, (size_t)B * C * esz, st) != cudaSuccess))
      return fail(WKV_ERR_CUDA, "cudaMemsetAsync failed");
    return WKV_OK;
  }
  if (B * T * C * n_mix > ((int64_t)1 << 40)) return fail(WKV_ERR_UNSUPPORTED, "problem above 2^40 elements");
  WKV_REQUIRE_PTR(x, "x");
  WKV_REQUIRE_PTR(mix, "mix");
  WKV_OPTIONAL_PTR(x_prev, "x_prev");
  WKV_REQUIRE_PTR(g, "g");
  WKV_REQUIRE_PTR(gx, "gx");
  WKV_OPTIONAL_PTR(gx_prev, "gx_prev");
  WKV_REQUIRE_PTR(workspace, "workspace");
  if (workspace_bytes < wkv4_time_shift_mix_backward_workspace_bytes(B, T, C, dtype, n_mix))
    return fail(WKV_ERR_INVALID_ARG, "workspace_bytes below wkv4_time_shift_mix_backward_workspace_bytes()");
  TimeShiftArgs a{B, T, C, dtype, (int)n_mix, x, mix, x_prev, nullptr, g, gx, gmix, gx_prev,
                  static_cast<float*>(workspace)};
  const char* why = "";
  wkv_status s = launch_time_shift_mix_backward(a, st, &why);
  return s == WKV_OK ? s : fail(s, why);
}
