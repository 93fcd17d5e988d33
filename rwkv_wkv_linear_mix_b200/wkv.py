"""Thin Python binding over the C ABI of libwkv_b200.so (include/wkv.h).

Argument marshalling only: every function checks tensor dtypes, shapes,
devices and contiguity, allocates outputs with torch (device memory is the
only thing torch provides here), and calls the C entry point of the same name
on the current CUDA stream. All arithmetic runs in the library's sm_100a
kernels; if the library is missing, importing this module raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwkv_b200.so")

WKV_OK, WKV_ERR_INVALID_ARG, WKV_ERR_UNSUPPORTED, WKV_ERR_CUDA, WKV_ERR_DEVICE = range(5)
WKV_F32, WKV_BF16 = 0, 1
WKV_DEVERR_WAIT_TIMEOUT, WKV_DEVERR_BAD_SLOT, WKV_DEVERR_BAD_STATE = 1, 2, 4
CKPT_LEN = 16  # WKV4_CKPT_LEN

# Every symbol include/wkv.h declares, with its ctypes signature.
_i64, _i32, _int, _vp, _sz = ctypes.c_int64, ctypes.c_int32, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
SIGNATURES = {
    "wkv_abi_version": (_int, []),
    "wkv_status_string": (ctypes.c_char_p, [_int]),
    "wkv_last_error": (ctypes.c_char_p, []),
    "wkv_device_error": (_int, [ctypes.POINTER(ctypes.c_uint32), _int]),
    "wkv4_ckpt_floats": (_sz, [_i64, _i64, _i64]),
    "wkv4_forward": (_int, [_i64, _i64, _i64, _int, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "wkv4_backward_workspace_bytes": (_sz, [_i64, _i64, _i64, _int]),
    "wkv4_backward": (_int, [_i64, _i64, _i64, _int] + [_vp] * 11 + [_sz, _vp]),
    "wkv4_state_init": (_int, [_i64, _i64, _vp, _vp]),
    "wkv4_chunk_step": (_int, [_i64, _i64, _int, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp]),
    "wkv6_forward": (_int, [_i64, _i64, _i64, _i64, _int] + [_vp] * 7 + [_i64, _vp, _vp, _vp]),
    "wkv4_backward_noalloc": (_int, [_i64, _i64, _i64, _int] + [_vp] * 11),
    "wkv6_backward_workspace_bytes": (_sz, [_i64, _i64, _i64, _i64]),
    "wkv_wait_selfcheck": (_int, [_i64, _vp]),
    "wkv7_forward": (_int, [_i64, _i64, _i64, _i64, _int] + [_vp] * 10),
    "wkv6_backward": (_int, [_i64, _i64, _i64, _i64, _int] + [_vp] * 7 + [_i64] + [_vp] * 9 + [_sz, _vp]),
    "wkv4_forward_gated": (_int, [_i64, _i64, _i64, _int] + [_vp] * 8),
    "wkv4_backward_gated": (_int, [_i64, _i64, _i64, _int] + [_vp] * 13 + [_sz, _vp]),
    "wkv4_time_shift_mix": (_int, [_i64, _i64, _i64, _int, _i64] + [_vp] * 5),
    "wkv4_decode_step": (_int, [_i64, _i64, _int] + [_vp] * 7),
    "wkv7_backward_workspace_bytes": (_sz, [_i64, _i64, _i64, _i64]),
    "wkv7_backward": (_int, [_i64, _i64, _i64, _i64, _int] + [_vp] * 17 + [_sz, _vp]),
    "wkv4_time_shift_mix_backward_workspace_bytes": (_sz, [_i64, _i64, _i64, _int, _i64]),
    "wkv4_time_shift_mix_backward": (_int, [_i64, _i64, _i64, _int, _i64] + [_vp] * 8 + [_sz, _vp]),
}


class WkvError(RuntimeError):
    def __init__(self, status: int, fn: str, msg: str):
        self.status = status
        super().__init__(f"{fn}: {_status_name(status)}: {msg}")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m rwkv_wkv_linear_mix_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = load_library()


def lib() -> ctypes.CDLL:
    """The loaded ctypes library (raw C entry points)."""
    return _lib


def _status_name(s: int) -> str:
    return _lib.wkv_status_string(int(s)).decode()


def _check(status: int, fn: str):
    if status != WKV_OK:
        raise WkvError(status, fn, _lib.wkv_last_error().decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return WKV_F32
    if t.dtype == torch.bfloat16:
        return WKV_BF16
    raise TypeError(f"unsupported activation dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _want(t: torch.Tensor, name: str, dtype=None, shape=None, device=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _want_wkv4_grads(k, gk, gv, gw, gu):
    """Caller-provided RWKV-4 gradient buffers must match what the kernels
    write: gk, gv like k; gw, gu float32 [C] (a smaller or mistyped buffer
    would be written past its end)."""
    C = k.shape[-1]
    _want(gk, "gk", dtype=k.dtype, shape=k.shape, device=k.device)
    _want(gv, "gv", dtype=k.dtype, shape=k.shape, device=k.device)
    _want(gw, "gw", dtype=torch.float32, shape=(C,), device=k.device)
    _want(gu, "gu", dtype=torch.float32, shape=(C,), device=k.device)


def abi_version() -> int:
    return int(_lib.wkv_abi_version())


def device_error(reset: bool = True) -> int:
    """Device-side error bits of the current device (synchronises)."""
    code = ctypes.c_uint32(0)
    _check(_lib.wkv_device_error(ctypes.byref(code), int(reset)), "wkv_device_error")
    return int(code.value)


# ----------------------------------------------------------------------------
# RWKV-4
# ----------------------------------------------------------------------------

def ckpt_shape(B: int, T: int, C: int):
    return (B, (T + CKPT_LEN - 1) // CKPT_LEN, 3, C)


def wkv4_forward(w: torch.Tensor, u: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *,
                 y: Optional[torch.Tensor] = None, ckpt: Optional[torch.Tensor] = None,
                 want_ckpt: bool = False, want_y: bool = True):
    """RWKV-4 WKV forward. w (decay rate > 0), u: [C] float32; k, v: [B, T, C].

    Returns y, or (y, ckpt) when ``want_ckpt`` (or a ckpt buffer is passed).
    """
    B, T, C = k.shape
    dev = k.device
    _want(k, "k")
    _want(v, "v", dtype=k.dtype, shape=k.shape, device=dev)
    _want(w, "w", dtype=torch.float32, shape=(C,), device=dev)
    _want(u, "u", dtype=torch.float32, shape=(C,), device=dev)
    if want_y and y is None:
        y = torch.empty_like(k)
    if y is not None:
        _want(y, "y", dtype=k.dtype, shape=k.shape, device=dev)
    if ckpt is None and want_ckpt:
        ckpt = torch.empty(ckpt_shape(B, T, C), dtype=torch.float32, device=dev)
    if ckpt is not None:
        _want(ckpt, "ckpt", dtype=torch.float32, shape=ckpt_shape(B, T, C), device=dev)
    _check(_lib.wkv4_forward(B, T, C, _dtype_code(k), _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(y),
                             _ptr(ckpt), _stream(k)), "wkv4_forward")
    return (y, ckpt) if (want_ckpt or ckpt is not None) else y


def wkv4_backward_workspace_bytes(B: int, T: int, C: int, has_ckpt: bool) -> int:
    return int(_lib.wkv4_backward_workspace_bytes(B, T, C, int(has_ckpt)))


def wkv4_backward(w, u, k, v, gy, ckpt: Optional[torch.Tensor] = None, *, gk=None, gv=None, gw=None, gu=None,
                  workspace: Optional[torch.Tensor] = None):
    """RWKV-4 WKV backward. Returns (gk, gv, gw, gu); gw = dL/dw, gu = dL/du
    (float32 [C], summed over batch and time)."""
    B, T, C = k.shape
    dev = k.device
    for name, t in (("k", k), ("v", v), ("gy", gy)):
        _want(t, name, dtype=k.dtype, shape=k.shape, device=dev)
    _want(w, "w", dtype=torch.float32, shape=(C,), device=dev)
    _want(u, "u", dtype=torch.float32, shape=(C,), device=dev)
    if ckpt is not None:
        _want(ckpt, "ckpt", dtype=torch.float32, shape=ckpt_shape(B, T, C), device=dev)
    gk = torch.empty_like(k) if gk is None else gk
    gv = torch.empty_like(k) if gv is None else gv
    gw = torch.empty(C, dtype=torch.float32, device=dev) if gw is None else gw
    gu = torch.empty(C, dtype=torch.float32, device=dev) if gu is None else gu
    _want_wkv4_grads(k, gk, gv, gw, gu)
    nbytes = wkv4_backward_workspace_bytes(B, T, C, ckpt is not None)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    _want(workspace, "workspace", device=dev)
    _check(_lib.wkv4_backward(B, T, C, _dtype_code(k), _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(gy), _ptr(ckpt),
                              _ptr(gk), _ptr(gv), _ptr(gw), _ptr(gu), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(k)), "wkv4_backward")
    return gk, gv, gw, gu


def wkv4_backward_noalloc(w, u, k, v, gy, ckpt: Optional[torch.Tensor] = None, *, gk=None, gv=None, gw=None,
                          gu=None):
    """wkv4_backward with the library's static device scratch instead of a
    workspace (for callers that cannot allocate per call; see wkv.h).
    Outputs may be passed in preallocated. Returns (gk, gv, gw, gu)."""
    B, T, C = k.shape
    dev = k.device
    for name, t in (("k", k), ("v", v), ("gy", gy)):
        _want(t, name, dtype=k.dtype, shape=k.shape, device=dev)
    _want(w, "w", dtype=torch.float32, shape=(C,), device=dev)
    _want(u, "u", dtype=torch.float32, shape=(C,), device=dev)
    if ckpt is not None:
        _want(ckpt, "ckpt", dtype=torch.float32, shape=ckpt_shape(B, T, C), device=dev)
    gk = torch.empty_like(k) if gk is None else gk
    gv = torch.empty_like(k) if gv is None else gv
    gw = torch.empty(C, dtype=torch.float32, device=dev) if gw is None else gw
    gu = torch.empty(C, dtype=torch.float32, device=dev) if gu is None else gu
    _want_wkv4_grads(k, gk, gv, gw, gu)
    # the library finds the static array of the current device: make it k's
    with torch.cuda.device(dev):
        _check(_lib.wkv4_backward_noalloc(B, T, C, _dtype_code(k), _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(gy),
                                          _ptr(ckpt), _ptr(gk), _ptr(gv), _ptr(gw), _ptr(gu), _stream(k)),
               "wkv4_backward_noalloc")
    return gk, gv, gw, gu


def wkv4_forward_gated(w, u, k, v, r, *, y: Optional[torch.Tensor] = None, ckpt: Optional[torch.Tensor] = None,
                       want_ckpt: bool = False):
    """sigmoid(r) * WKV in one kernel (the time-mix gate fused into the RWKV-4
    forward). r: [B, T, C] like k. Returns y, or (y, ckpt)."""
    B, T, C = k.shape
    dev = k.device
    for name, t in (("k", k), ("v", v), ("r", r)):
        _want(t, name, dtype=k.dtype, shape=k.shape, device=dev)
    _want(w, "w", dtype=torch.float32, shape=(C,), device=dev)
    _want(u, "u", dtype=torch.float32, shape=(C,), device=dev)
    y = torch.empty_like(k) if y is None else y
    _want(y, "y", dtype=k.dtype, shape=k.shape, device=dev)
    if ckpt is None and want_ckpt:
        ckpt = torch.empty(ckpt_shape(B, T, C), dtype=torch.float32, device=dev)
    if ckpt is not None:
        _want(ckpt, "ckpt", dtype=torch.float32, shape=ckpt_shape(B, T, C), device=dev)
    _check(_lib.wkv4_forward_gated(B, T, C, _dtype_code(k), _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(y),
                                   _ptr(ckpt), _stream(k)), "wkv4_forward_gated")
    return (y, ckpt) if (want_ckpt or ckpt is not None) else y


def wkv4_backward_gated(w, u, k, v, r, gy, ckpt: Optional[torch.Tensor] = None, *, gk=None, gv=None, gr=None,
                        gw=None, gu=None, workspace: Optional[torch.Tensor] = None):
    """Gradients of the gated forward. Returns (gk, gv, gr, gw, gu)."""
    B, T, C = k.shape
    dev = k.device
    for name, t in (("k", k), ("v", v), ("r", r), ("gy", gy)):
        _want(t, name, dtype=k.dtype, shape=k.shape, device=dev)
    _want(w, "w", dtype=torch.float32, shape=(C,), device=dev)
    _want(u, "u", dtype=torch.float32, shape=(C,), device=dev)
    if ckpt is not None:
        _want(ckpt, "ckpt", dtype=torch.float32, shape=ckpt_shape(B, T, C), device=dev)
    gk = torch.empty_like(k) if gk is None else gk
    gv = torch.empty_like(k) if gv is None else gv
    gr = torch.empty_like(k) if gr is None else gr
    gw = torch.empty(C, dtype=torch.float32, device=dev) if gw is None else gw
    gu = torch.empty(C, dtype=torch.float32, device=dev) if gu is None else gu
    _want_wkv4_grads(k, gk, gv, gw, gu)
    _want(gr, "gr", dtype=k.dtype, shape=k.shape, device=dev)
    nbytes = wkv4_backward_workspace_bytes(B, T, C, ckpt is not None)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    _want(workspace, "workspace", device=dev)
    _check(_lib.wkv4_backward_gated(B, T, C, _dtype_code(k), _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r), _ptr(gy),
                                    _ptr(ckpt), _ptr(gk), _ptr(gv), _ptr(gr), _ptr(gw), _ptr(gu), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(k)), "wkv4_backward_gated")
    return gk, gv, gr, gw, gu


def wkv4_time_shift_mix(x, mix, x_prev: Optional[torch.Tensor] = None, *, out: Optional[torch.Tensor] = None):
    """The time-mix prologue: n_mix blends of each token with the one before.
    x: [B, T, C]; mix: [n_mix, C] float32 (n_mix 1..3); x_prev: [B, C] like x
    or None (zeros). Returns out [n_mix, B, T, C] (out[0], out[1], out[2] are
    the k, v, r inputs)."""
    B, T, C = x.shape
    dev = x.device
    _want(x, "x")
    n = mix.shape[0] if mix.dim() == 2 else -1
    _want(mix, "mix", dtype=torch.float32, shape=(n, C), device=dev)
    if x_prev is not None:
        _want(x_prev, "x_prev", dtype=x.dtype, shape=(B, C), device=dev)
    out = torch.empty((n, B, T, C), dtype=x.dtype, device=dev) if out is None else out
    _want(out, "out", dtype=x.dtype, shape=(n, B, T, C), device=dev)
    _check(_lib.wkv4_time_shift_mix(B, T, C, _dtype_code(x), n, _ptr(x), _ptr(mix), _ptr(x_prev), _ptr(out),
                                    _stream(x)), "wkv4_time_shift_mix")
    return out


def wkv4_time_shift_mix_backward_workspace_bytes(B: int, T: int, C: int, dtype: torch.dtype, n_mix: int) -> int:
    code = WKV_BF16 if dtype == torch.bfloat16 else WKV_F32
    return int(_lib.wkv4_time_shift_mix_backward_workspace_bytes(B, T, C, code, n_mix))


def wkv4_time_shift_mix_backward(x, mix, g, x_prev: Optional[torch.Tensor] = None, *, want_gx_prev: bool = False,
                                 gx=None, gmix=None, gx_prev=None, workspace: Optional[torch.Tensor] = None):
    """Gradients of sum(g * wkv4_time_shift_mix(x, mix, x_prev)). g: [n_mix, B,
    T, C]. Returns (gx, gmix, gx_prev); gx_prev is None unless wanted (or a
    buffer is passed)."""
    B, T, C = x.shape
    dev = x.device
    _want(x, "x")
    n = mix.shape[0] if mix.dim() == 2 else -1
    _want(mix, "mix", dtype=torch.float32, shape=(n, C), device=dev)
    _want(g, "g", dtype=x.dtype, shape=(n, B, T, C), device=dev)
    if x_prev is not None:
        _want(x_prev, "x_prev", dtype=x.dtype, shape=(B, C), device=dev)
    gx = torch.empty_like(x) if gx is None else gx
    gmix = torch.empty((n, C), dtype=torch.float32, device=dev) if gmix is None else gmix
    if gx_prev is None and want_gx_prev:
        gx_prev = torch.empty((B, C), dtype=x.dtype, device=dev)
    _want(gx, "gx", dtype=x.dtype, shape=x.shape, device=dev)
    _want(gmix, "gmix", dtype=torch.float32, shape=(n, C), device=dev)
    if gx_prev is not None:
        _want(gx_prev, "gx_prev", dtype=x.dtype, shape=(B, C), device=dev)
    nbytes = wkv4_time_shift_mix_backward_workspace_bytes(B, T, C, x.dtype, n)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    _want(workspace, "workspace", device=dev)
    _check(_lib.wkv4_time_shift_mix_backward(B, T, C, _dtype_code(x), n, _ptr(x), _ptr(mix), _ptr(x_prev), _ptr(g),
                                             _ptr(gx), _ptr(gmix), _ptr(gx_prev), _ptr(workspace),
                                             workspace.numel() * workspace.element_size(), _stream(x)),
           "wkv4_time_shift_mix_backward")
    return gx, gmix, gx_prev


STATE_ROWS = 5  # aa, bb, base, n, ref


def wkv4_state_init(S: int, C: int, device, state: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Slot states [S, 5, C] float32 (aa, bb, base, n, ref) set to the empty past."""
    if state is None:
        state = torch.empty((S, STATE_ROWS, C), dtype=torch.float32, device=device)
    _want(state, "state", dtype=torch.float32, shape=(S, STATE_ROWS, C))
    _check(_lib.wkv4_state_init(S, C, _ptr(state), _stream(state)), "wkv4_state_init")
    return state


def wkv4_chunk_step(w, u, k, v, cu_tokens: torch.Tensor, state: torch.Tensor, *, y=None) -> torch.Tensor:
    """One batched inference call. k, v: [N, C] packed tokens of all slots;
    cu_tokens: int32 [S+1] on the device; state: [S, 5, C] float32 (in/out)."""
    N, C = k.shape
    S = state.shape[0]
    dev = k.device
    _want(k, "k")
    _want(v, "v", dtype=k.dtype, shape=k.shape, device=dev)
    _want(w, "w", dtype=torch.float32, shape=(C,), device=dev)
    _want(u, "u", dtype=torch.float32, shape=(C,), device=dev)
    _want(cu_tokens, "cu_tokens", dtype=torch.int32, shape=(S + 1,), device=dev)
    _want(state, "state", dtype=torch.float32, shape=(S, STATE_ROWS, C), device=dev)
    y = torch.empty_like(k) if y is None else y
    _want(y, "y", dtype=k.dtype, shape=k.shape, device=dev)
    _check(_lib.wkv4_chunk_step(S, C, _dtype_code(k), _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(y), N,
                                _ptr(cu_tokens), _ptr(state), _stream(k)), "wkv4_chunk_step")
    return y


def wkv4_decode_step(w, u, k, v, state: torch.Tensor, *, y=None) -> torch.Tensor:
    """One decode call: slot s takes token k[s], v[s] (k, v: [S, C]); state
    [S, 5, C] float32 (in/out). Same results as wkv4_chunk_step with one
    token per slot, in one streaming kernel."""
    S, C = k.shape
    dev = k.device
    _want(k, "k")
    _want(v, "v", dtype=k.dtype, shape=k.shape, device=dev)
    _want(w, "w", dtype=torch.float32, shape=(C,), device=dev)
    _want(u, "u", dtype=torch.float32, shape=(C,), device=dev)
    _want(state, "state", dtype=torch.float32, shape=(S, STATE_ROWS, C), device=dev)
    y = torch.empty_like(k) if y is None else y
    _want(y, "y", dtype=k.dtype, shape=k.shape, device=dev)
    _check(_lib.wkv4_decode_step(S, C, _dtype_code(k), _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(y), _ptr(state),
                                 _stream(k)), "wkv4_decode_step")
    return y


# ----------------------------------------------------------------------------
# RWKV-6
# ----------------------------------------------------------------------------

def wkv6_forward(r, k, v, w, u, init_state: Optional[torch.Tensor] = None,
                 state_map: Optional[torch.Tensor] = None, *, head_size: int = 64,
                 want_final_state: bool = True, o=None, final_state=None):
    """RWKV-6 head-state forward. r, k, v, w: [B, T, H*K] bf16; u: [H*K] float32.
    Returns (o, final_state or None)."""
    B, T, HK = r.shape
    K = head_size
    if HK % K:
        raise ValueError("hidden size must be a multiple of head_size")
    H = HK // K
    dev = r.device
    for name, t in (("r", r), ("k", k), ("v", v), ("w", w)):
        _want(t, name, dtype=r.dtype, shape=r.shape, device=dev)
    _want(u, "u", dtype=torch.float32, device=dev)
    if u.numel() != HK:
        raise ValueError("u must hold H*K values")
    n_state = 0
    if init_state is not None:
        _want(init_state, "init_state", dtype=torch.float32, device=dev)
        n_state = init_state.shape[0]
        if tuple(init_state.shape[1:]) != (H, K, K):
            raise ValueError("init_state must be [n_state, H, K, K]")
    if state_map is not None:
        _want(state_map, "state_map", dtype=torch.int32, shape=(B,), device=dev)
    o = torch.empty_like(r) if o is None else o
    _want(o, "o", dtype=r.dtype, shape=r.shape, device=dev)
    if want_final_state and final_state is None:
        final_state = torch.empty((B, H, K, K), dtype=torch.float32, device=dev)
    if final_state is not None:
        _want(final_state, "final_state", dtype=torch.float32, shape=(B, H, K, K), device=dev)
    _check(_lib.wkv6_forward(B, T, H, K, _dtype_code(r), _ptr(r), _ptr(k), _ptr(v), _ptr(w), _ptr(u),
                             _ptr(init_state), _ptr(state_map), n_state, _ptr(final_state), _ptr(o),
                             _stream(r)), "wkv6_forward")
    return o, final_state


def wait_selfcheck(limit_ns: int = 2_000_000, device=None) -> None:
    """Run the bounded-wait failure path once (see wkv_wait_selfcheck)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _check(_lib.wkv_wait_selfcheck(int(limit_ns), ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)),
               "wkv_wait_selfcheck")


def wkv6_backward_workspace_bytes(B: int, T: int, H: int, K: int = 64) -> int:
    return int(_lib.wkv6_backward_workspace_bytes(B, T, H, K))


def wkv6_backward(r, k, v, w, u, dout, init_state: Optional[torch.Tensor] = None,
                  state_map: Optional[torch.Tensor] = None, g_final: Optional[torch.Tensor] = None, *,
                  head_size: int = 64, want_g_init: bool = True, workspace: Optional[torch.Tensor] = None,
                  gr=None, gk=None, gv=None, glogw=None, gu=None, g_init=None):
    """RWKV-6 head-state backward of wkv6_forward(r, k, v, w, u, init_state,
    state_map). dout: [B, T, H*K] bf16; g_final: [B, H, K, K] float32 or None.
    Returns (gr, gk, gv, glogw, gu, g_init or None); glogw = w * dL/dw."""
    B, T, HK = r.shape
    K = head_size
    if HK % K:
        raise ValueError("hidden size must be a multiple of head_size")
    H = HK // K
    dev = r.device
    for name, t in (("r", r), ("k", k), ("v", v), ("w", w), ("dout", dout)):
        _want(t, name, dtype=r.dtype, shape=r.shape, device=dev)
    _want(u, "u", dtype=torch.float32, device=dev)
    if u.numel() != HK:
        raise ValueError("u must hold H*K values")
    n_state = 0
    if init_state is not None:
        _want(init_state, "init_state", dtype=torch.float32, device=dev)
        n_state = init_state.shape[0]
        if tuple(init_state.shape[1:]) != (H, K, K):
            raise ValueError("init_state must be [n_state, H, K, K]")
    if state_map is not None:
        _want(state_map, "state_map", dtype=torch.int32, shape=(B,), device=dev)
    if g_final is not None:
        _want(g_final, "g_final", dtype=torch.float32, shape=(B, H, K, K), device=dev)
    gr = torch.empty_like(r) if gr is None else gr
    gk = torch.empty_like(r) if gk is None else gk
    gv = torch.empty_like(r) if gv is None else gv
    glogw = torch.empty_like(r) if glogw is None else glogw
    gu = torch.empty(HK, dtype=torch.float32, device=dev) if gu is None else gu
    if want_g_init and g_init is None:
        g_init = torch.empty((B, H, K, K), dtype=torch.float32, device=dev)
    for name, t in (("gr", gr), ("gk", gk), ("gv", gv), ("glogw", glogw)):
        _want(t, name, dtype=r.dtype, shape=r.shape, device=dev)
    _want(gu, "gu", dtype=torch.float32, shape=(HK,), device=dev)
    if g_init is not None:
        _want(g_init, "g_init", dtype=torch.float32, shape=(B, H, K, K), device=dev)
    need = wkv6_backward_workspace_bytes(B, T, H, K)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _want(workspace, "workspace", device=dev)
    _check(_lib.wkv6_backward(B, T, H, K, _dtype_code(r), _ptr(r), _ptr(k), _ptr(v), _ptr(w), _ptr(u),
                              _ptr(init_state), _ptr(state_map), n_state, _ptr(dout), _ptr(g_final),
                              _ptr(gr), _ptr(gk), _ptr(gv), _ptr(glogw), _ptr(gu), _ptr(g_init),
                              _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(r)),
           "wkv6_backward")
    return gr, gk, gv, glogw, gu, g_init


def wkv7_forward(r, w, k, v, a, b, init_state: Optional[torch.Tensor] = None, *, head_size: int = 64,
                 want_final_state: bool = True, o=None, final_state=None):
    """RWKV-7 generalized delta rule forward. r, w, k, v, a, b: [B, T, H*K]
    bf16 (w the decay in log space); init_state: [B, H, K, K] float32
    (indexed [b][h][key][value]) or None. Returns (o, final_state or None)."""
    B, T, HK = r.shape
    K = head_size
    if HK % K:
        raise ValueError("hidden size must be a multiple of head_size")
    H = HK // K
    dev = r.device
    for name, t in (("r", r), ("w", w), ("k", k), ("v", v), ("a", a), ("b", b)):
        _want(t, name, dtype=r.dtype, shape=r.shape, device=dev)
    if init_state is not None:
        _want(init_state, "init_state", dtype=torch.float32, shape=(B, H, K, K), device=dev)
    o = torch.empty_like(r) if o is None else o
    _want(o, "o", dtype=r.dtype, shape=r.shape, device=dev)
    if want_final_state and final_state is None:
        final_state = torch.empty((B, H, K, K), dtype=torch.float32, device=dev)
    if final_state is not None:
        _want(final_state, "final_state", dtype=torch.float32, shape=(B, H, K, K), device=dev)
    _check(_lib.wkv7_forward(B, T, H, K, _dtype_code(r), _ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
                             _ptr(init_state), _ptr(final_state), _ptr(o), _stream(r)), "wkv7_forward")
    return o, final_state


def wkv7_backward_workspace_bytes(B: int, T: int, H: int, head_size: int = 64) -> int:
    return int(_lib.wkv7_backward_workspace_bytes(B, T, H, head_size))


def wkv7_backward(r, w, k, v, a, b, dout, init_state: Optional[torch.Tensor] = None,
                  g_final: Optional[torch.Tensor] = None, *, head_size: int = 64,
                  workspace: Optional[torch.Tensor] = None):
    """Gradients of sum(dout * o) (+ sum(g_final * S_final)) for wkv7_forward on
    the same inputs. Returns (dr, dw, dk, dv, da, db, d_init); dw is with respect
    to the log decay w, d_init (float32 [B, H, K, K]) to the initial state."""
    B, T, HK = r.shape
    K = head_size
    if HK % K:
        raise ValueError("hidden size must be a multiple of head_size")
    H = HK // K
    dev = r.device
    for name, t in (("r", r), ("w", w), ("k", k), ("v", v), ("a", a), ("b", b), ("dout", dout)):
        _want(t, name, dtype=r.dtype, shape=r.shape, device=dev)
    for name, t in (("init_state", init_state), ("g_final", g_final)):
        if t is not None:
            _want(t, name, dtype=torch.float32, shape=(B, H, K, K), device=dev)
    grads = [torch.empty_like(r) for _ in range(6)]
    d_init = torch.empty((B, H, K, K), dtype=torch.float32, device=dev)
    nbytes = wkv7_backward_workspace_bytes(B, T, H, K)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    _want(workspace, "workspace", device=dev)
    _check(_lib.wkv7_backward(B, T, H, K, _dtype_code(r), _ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
                              _ptr(init_state), _ptr(dout), _ptr(g_final), *[_ptr(x) for x in grads], _ptr(d_init),
                              _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(r)),
           "wkv7_backward")
    return (*grads, d_init)
