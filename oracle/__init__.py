"""fp64 CPU oracle for the WKV recurrences (test infrastructure).

Only the tests, the smoke check and the bench's CPU-baseline leg use this
package. The CUDA library never imports, links or calls it, and it imports
nothing from the CUDA side. The arithmetic lives in ``wkv_oracle.c`` (plain C,
fp64, OpenMP over independent lanes); this module only widens inputs to fp64,
calls it through ctypes and returns numpy arrays.

Definitions followed:
  * RWKV-4 WKV: the operator behind RUN_CUDA(B, T, C, time_decay, time_first,
    k, v) in RWKV_TimeMix.forward ("代码连连看——RWKV", section RWKV_TimeMix),
    y_t = (sum_{i<t} e^{-(t-1-i)w+k_i} v_i + e^{u+k_t} v_t)
          / (sum_{i<t} e^{-(t-1-i)w+k_i} + e^{u+k_t}),  w = exp(time_decay).
  * RWKV-6 head-state WKV: RWKV6_OP (rwkv-ops package page, section
    "rwkv6op 使用方法"): o_t = r_t (S_{t-1} + diag(u) k_t^T v_t),
    S_t = diag(w_t) S_{t-1} + k_t^T v_t; the op is trainable (the page's
    backend table lists its PyTorch CUDA backward), so its gradients are the
    chain rule of this recurrence.
  * Time-shift mix: the prologue of RWKV_TimeMix.jit_func (same RWKV-4 page):
    x_m,t = x_t mix_m + x_{t-1} (1 - mix_m), x_{-1} = 0 (time_shift pads one
    zero row), for m in (k, v, r).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wkv_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle_wkv.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile wkv_oracle.c with gcc (-O2 -fopenmp, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    os.makedirs(_BUILD_DIR, exist_ok=True)
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off",
           "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _open(path):
    lib = ctypes.CDLL(path)
    i64, dp = ctypes.c_int64, ctypes.c_void_p
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
    lib.oracle_set_num_threads.restype = None
    lib.oracle_wkv4_forward.argtypes = [i64, i64, i64] + [dp] * 8
    lib.oracle_wkv4_forward.restype = ctypes.c_int
    lib.oracle_wkv4_backward.argtypes = [i64, i64, i64] + [dp] * 10
    lib.oracle_wkv4_backward.restype = ctypes.c_int
    lib.oracle_wkv6_forward.argtypes = [i64, i64, i64, i64] + [dp] * 7 + [i64, dp, dp]
    lib.oracle_wkv6_forward.restype = ctypes.c_int
    lib.oracle_wkv6_backward.argtypes = [i64, i64, i64, i64] + [dp] * 7 + [i64] + [dp] * 8
    lib.oracle_wkv7_forward.argtypes = [i64, i64, i64, i64] + [dp] * 9
    lib.oracle_wkv7_forward.restype = ctypes.c_int
    lib.oracle_wkv6_backward.restype = ctypes.c_int
    lib.oracle_wkv7_backward.argtypes = [i64, i64, i64, i64] + [dp] * 16
    lib.oracle_wkv7_backward.restype = ctypes.c_int
    lib.oracle_time_shift_mix.argtypes = [i64, i64, i64, i64] + [dp] * 4
    lib.oracle_time_shift_mix.restype = ctypes.c_int
    lib.oracle_time_shift_mix_backward.argtypes = [i64, i64, i64, i64] + [dp] * 7
    lib.oracle_time_shift_mix_backward.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _open(build())
    return _lib


class _Variant:
    """The same entry points bound to another build of wkv_oracle.c.

    Used by the tests that plant a mistake in a copy of the oracle source and
    check that the pins catch it.
    """

    def __init__(self, path):
        self._lib = _open(path)

    def __getattr__(self, name):
        fn = globals()[name]
        lib = self._lib

        def bound(*a, **kw):
            return fn(*a, _lib=lib, **kw)
        return bound


def build_variant(source_text: str, out_dir: str) -> "_Variant":
    """Compile ``source_text`` (an edited copy of wkv_oracle.c) into out_dir."""
    src = os.path.join(out_dir, "variant.c")
    with open(src, "w") as f:
        f.write(source_text)
    so = os.path.join(out_dir, "libvariant.so")
    subprocess.run(["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off",
                    "-fopenmp", "-fPIC", "-shared", src, "-o", so, "-lm"], check=True)
    return _Variant(so)


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS, else all cores)."""
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Use n OpenMP threads from now on (the bench times the oracle on one
    core and on all of them; results do not depend on the count)."""
    _load().oracle_set_num_threads(int(n))


def wkv4_forward(w, u, k, v, return_state: bool = False, _lib=None):
    """RWKV-4 WKV forward in fp64.

    w, u: [C] (w > 0 is the per-step decay rate), k, v: [B, T, C].
    Returns y [B, T, C]; with ``return_state`` also a dict holding the state
    after the last token as a_end, b_end (scaled by e^{-kmax}) and kmax, each
    [B, C], so that the true sums are a = a_end * e^{kmax}, b = b_end * e^{kmax}.
    """
    lib = _lib or _load()
    k, v, w, u = _f64(k), _f64(v), _f64(w), _f64(u)
    B, T, C = k.shape
    assert v.shape == k.shape and w.shape == (C,) and u.shape == (C,)
    y = np.empty_like(k)
    st = {n: np.empty((B, C)) for n in ("a_end", "b_end", "kmax")} if return_state else None
    rc = lib.oracle_wkv4_forward(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(y),
                                 _ptr(st and st["a_end"]), _ptr(st and st["b_end"]),
                                 _ptr(st and st["kmax"]))
    if rc != 0:
        raise FloatingPointError(f"oracle_wkv4_forward: non-finite result (rc={rc})")
    return (y, st) if return_state else y


def wkv4_backward(w, u, k, v, gy, return_reverse_gw: bool = False, _lib=None):
    """RWKV-4 WKV backward in fp64.

    Returns (gk, gv, gw, gu): gk, gv [B, T, C]; gw = dL/dw and gu = dL/du, [C],
    summed over batch and time, for L = sum(gy * y). With ``return_reverse_gw``
    a fifth item holds gw evaluated by the independent reverse-scan formula.
    """
    lib = _lib or _load()
    k, v, w, u, gy = _f64(k), _f64(v), _f64(w), _f64(u), _f64(gy)
    B, T, C = k.shape
    assert v.shape == k.shape == gy.shape and w.shape == (C,) and u.shape == (C,)
    gk, gv = np.empty_like(k), np.empty_like(k)
    gw, gu, gwr = np.empty(C), np.empty(C), np.empty(C)
    rc = lib.oracle_wkv4_backward(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(gy),
                                  _ptr(gk), _ptr(gv), _ptr(gw), _ptr(gu), _ptr(gwr))
    if rc != 0:
        raise FloatingPointError(f"oracle_wkv4_backward failed (rc={rc})")
    return (gk, gv, gw, gu, gwr) if return_reverse_gw else (gk, gv, gw, gu)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def wkv4_forward_gated(w, u, k, v, r, _lib=None):
    """The gated output of RWKV_TimeMix.forward ("代码连连看——RWKV", section
    RWKV_TimeMix: rwkv = sigmoid(r) * RUN_CUDA(...)): sigmoid(r) * y in fp64,
    y the WKV above. r: [B, T, C]."""
    return _sigmoid(_f64(r)) * wkv4_forward(w, u, k, v, _lib=_lib)


def wkv4_backward_gated(w, u, k, v, r, g, _lib=None):
    """Gradients of L = sum(g * sigmoid(r) * y) in fp64 by the chain rule:
    with s = sigmoid(r), the WKV sees gy = g * s, and dL/dr = g * y * s (1 - s).
    Returns (gk, gv, gr, gw, gu)."""
    r, g = _f64(r), _f64(g)
    s = _sigmoid(r)
    y = wkv4_forward(w, u, k, v, _lib=_lib)
    gk, gv, gw, gu = wkv4_backward(w, u, k, v, g * s, _lib=_lib)
    return gk, gv, g * y * s * (1.0 - s), gw, gu


def wkv6_forward(r, k, v, w, u, init_state=None, state_map=None, _lib=None):
    """RWKV-6 head-state WKV forward in fp64.

    r, k, v, w: [B, T, H*K]; u: [H*K] or [H, K]; K is inferred from
    init_state when given, else must be passed through ``u`` shaped [H, K].
    init_state: [n_state, H, K, K] or None; state_map: [B] int or None.
    Returns (o [B, T, H*K], final_state [B, H, K, K]).
    """
    lib = _lib or _load()
    u = np.asarray(u)
    if u.ndim == 2:
        H, K = u.shape
    elif init_state is not None:
        H, K = np.asarray(init_state).shape[1:3]
    else:
        raise ValueError("pass u as [H, K] or give init_state to fix the head size")
    r, k, v, w, u = _f64(r), _f64(k), _f64(v), _f64(w), _f64(u).reshape(-1)
    B, T, HK = r.shape
    assert HK == H * K and k.shape == v.shape == w.shape == r.shape
    n_state = 0
    s0 = None
    if init_state is not None:
        s0 = _f64(init_state)
        n_state = s0.shape[0]
        assert s0.shape == (n_state, H, K, K)
    sm = None
    if state_map is not None:
        sm = np.ascontiguousarray(state_map, dtype=np.int32)
        assert sm.shape == (B,)
    o = np.empty_like(r)
    fs = np.empty((B, H, K, K))
    rc = lib.oracle_wkv6_forward(B, T, H, K, _ptr(r), _ptr(k), _ptr(v), _ptr(w), _ptr(u),
                                 _ptr(s0), _ptr(sm), n_state, _ptr(o), _ptr(fs))
    if rc != 0:
        raise FloatingPointError(f"oracle_wkv6_forward failed (rc={rc})")
    return o, fs


def wkv6_backward(r, k, v, w, u, dout, init_state=None, state_map=None, g_final=None, _lib=None):
    """Gradients of sum(o * dout) + sum(final_state * g_final) for
    wkv6_forward(r, k, v, w, u, init_state, state_map), in fp64.

    u is [H, K] (or [H*K] with init_state fixing K). Returns
    (gr, gk, gv, gw [B, T, H*K], gu [H*K] summed over samples and tokens,
    g_init [B, H, K, K] = dL/dS_{-1} of each sample).
    """
    lib = _lib or _load()
    u = np.asarray(u)
    if u.ndim == 2:
        H, K = u.shape
    elif init_state is not None:
        H, K = np.asarray(init_state).shape[1:3]
    else:
        raise ValueError("pass u as [H, K] or give init_state to fix the head size")
    r, k, v, w, u, dout = _f64(r), _f64(k), _f64(v), _f64(w), _f64(u).reshape(-1), _f64(dout)
    B, T, HK = r.shape
    assert HK == H * K and k.shape == v.shape == w.shape == r.shape == dout.shape
    n_state, s0, sm, gf = 0, None, None, None
    if init_state is not None:
        s0 = _f64(init_state)
        n_state = s0.shape[0]
        assert s0.shape == (n_state, H, K, K)
    if state_map is not None:
        sm = np.ascontiguousarray(state_map, dtype=np.int32)
        assert sm.shape == (B,)
    if g_final is not None:
        gf = _f64(g_final)
        assert gf.shape == (B, H, K, K)
    gr, gk, gv, gw = (np.empty_like(r) for _ in range(4))
    gu = np.empty(HK)
    gi = np.empty((B, H, K, K))
    rc = lib.oracle_wkv6_backward(B, T, H, K, _ptr(r), _ptr(k), _ptr(v), _ptr(w), _ptr(u), _ptr(s0), _ptr(sm),
                                  n_state, _ptr(dout), _ptr(gf), _ptr(gr), _ptr(gk), _ptr(gv), _ptr(gw),
                                  _ptr(gu), _ptr(gi))
    if rc != 0:
        raise FloatingPointError(f"oracle_wkv6_backward failed (rc={rc})")
    return gr, gk, gv, gw, gu, gi


def wkv7_forward(r, w, k, v, a, b, init_state=None, head_size: int = 64, _lib=None):
    """RWKV-7 generalized delta rule forward in fp64 (see oracle_wkv7_forward).

    r, w, k, v, a, b: [B, T, H*K] (w the decay in log space); init_state:
    [B, H, K, K] indexed [b][h][key][value] or None. Returns (o [B, T, H*K],
    final_state [B, H, K, K]).
    """
    lib = _lib or _load()
    r, w, k, v, a, b = (_f64(x) for x in (r, w, k, v, a, b))
    B, T, HK = r.shape
    K = head_size
    assert HK % K == 0 and all(x.shape == r.shape for x in (w, k, v, a, b))
    H = HK // K
    s0 = None
    if init_state is not None:
        s0 = _f64(init_state)
        assert s0.shape == (B, H, K, K)
    o = np.empty_like(r)
    fs = np.empty((B, H, K, K))
    rc = lib.oracle_wkv7_forward(B, T, H, K, _ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(s0),
                                 _ptr(o), _ptr(fs))
    if rc != 0:
        raise FloatingPointError(f"oracle_wkv7_forward failed (rc={rc})")
    return o, fs


def wkv7_backward(r, w, k, v, a, b, dout, init_state=None, g_final=None, head_size: int = 64, _lib=None):
    """Gradients of sum(dout * o) + sum(g_final * S_final) for wkv7_forward
    (see oracle_wkv7_backward), in fp64. Returns (dr, dw, dk, dv, da, db,
    d_init); dw is with respect to the log decay w."""
    lib = _lib or _load()
    r, w, k, v, a, b, dout = (_f64(x) for x in (r, w, k, v, a, b, dout))
    B, T, HK = r.shape
    K = head_size
    assert HK % K == 0 and all(x.shape == r.shape for x in (w, k, v, a, b, dout))
    H = HK // K
    s0 = None if init_state is None else _f64(init_state)
    gf = None if g_final is None else _f64(g_final)
    for x in (s0, gf):
        assert x is None or x.shape == (B, H, K, K)
    outs = [np.empty_like(r) for _ in range(6)]
    d_init = np.empty((B, H, K, K))
    rc = lib.oracle_wkv7_backward(B, T, H, K, _ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(s0),
                                  _ptr(dout), _ptr(gf), *[_ptr(o) for o in outs], _ptr(d_init))
    if rc != 0:
        raise FloatingPointError(f"oracle_wkv7_backward failed (rc={rc})")
    return (*outs, d_init)


def time_shift_mix(x, mix, x_prev=None, _lib=None):
    """The time-shift mix in fp64 (see oracle_time_shift_mix). x: [B, T, C];
    mix: [n_mix, C]; x_prev: [B, C] or None (zeros). Returns [n_mix, B, T, C]."""
    lib = _lib or _load()
    x, mix = _f64(x), _f64(mix)
    B, T, C = x.shape
    n = mix.shape[0]
    assert mix.shape == (n, C)
    xp = None if x_prev is None else _f64(x_prev)
    assert xp is None or xp.shape == (B, C)
    out = np.empty((n, B, T, C))
    if lib.oracle_time_shift_mix(B, T, C, n, _ptr(x), _ptr(mix), _ptr(xp), _ptr(out)) != 0:
        raise FloatingPointError("oracle_time_shift_mix: non-finite output")
    return out


def time_shift_mix_backward(x, mix, g, x_prev=None, _lib=None):
    """Gradients of sum(g * time_shift_mix(x, mix, x_prev)) in fp64.
    g: [n_mix, B, T, C]. Returns (gx [B, T, C], gmix [n_mix, C],
    gx_prev [B, C] or None when x_prev is None)."""
    lib = _lib or _load()
    x, mix, g = _f64(x), _f64(mix), _f64(g)
    B, T, C = x.shape
    n = mix.shape[0]
    assert g.shape == (n, B, T, C)
    xp = None if x_prev is None else _f64(x_prev)
    gx = np.empty((B, T, C))
    gmix = np.empty((n, C))
    gxp = None if xp is None else np.empty((B, C))
    if lib.oracle_time_shift_mix_backward(B, T, C, n, _ptr(x), _ptr(mix), _ptr(xp), _ptr(g), _ptr(gx),
                                          _ptr(gmix), _ptr(gxp)) != 0:
        raise FloatingPointError("oracle_time_shift_mix_backward: non-finite output")
    return gx, gmix, gxp
