"""Host-side checks of the C ABI that need no GPU.

The library must load on a machine without a GPU, export every function that
include/wkv.h declares, and reject malformed arguments before it touches the
CUDA runtime.
"""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wkv.h")


@pytest.fixture(scope="module")
def W():
    from rwkv_wkv_linear_mix_b200 import build
    build.build()
    from rwkv_wkv_linear_mix_b200 import wkv
    return wkv


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                       src, flags=re.M)
    return sorted(set(n for n in names if n.startswith("wkv")))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("wkv4_forward", "wkv4_backward", "wkv4_chunk_step", "wkv4_state_init", "wkv6_forward",
              "wkv4_backward_workspace_bytes", "wkv4_ckpt_floats", "wkv_status_string", "wkv_last_error",
              "wkv_device_error", "wkv_abi_version", "wkv6_backward", "wkv6_backward_workspace_bytes",
              "wkv4_forward_gated", "wkv4_backward_gated", "wkv7_forward", "wkv4_time_shift_mix",
              "wkv4_time_shift_mix_backward", "wkv4_time_shift_mix_backward_workspace_bytes",
              "wkv4_decode_step", "wkv7_backward", "wkv7_backward_workspace_bytes"):
        assert n in names


def test_every_declared_symbol_is_exported(W):
    lib = ctypes.CDLL(W.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in wkv.h but not exported"
    assert set(declared_functions()) == set(W.SIGNATURES), "binding signatures out of sync with wkv.h"


def declared_arity():
    """Number of parameters of every function wkv.h declares."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(wkv[A-Za-z0-9_]*)\s*\(([^;{]*?)\)\s*;", src, flags=re.S):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_the_header(W):
    """Every ctypes signature has as many arguments as the C declaration."""
    arity = declared_arity()
    for name, (_, args) in W.SIGNATURES.items():
        assert arity[name] == len(args), f"{name}: header {arity[name]} vs binding {len(args)}"


def test_version_and_strings(W):
    L = W.lib()
    assert L.wkv_abi_version() == 1
    assert L.wkv_status_string(0) == b"WKV_OK"
    assert L.wkv_status_string(2) == b"WKV_ERR_UNSUPPORTED"
    assert L.wkv_status_string(99) == b"WKV_ERR_UNKNOWN"


def test_size_helpers(W):
    L = W.lib()
    n = lambda T: -(-T // W.CKPT_LEN)  # checkpoints of a T-token sequence
    assert L.wkv4_ckpt_floats(2, 64, 128) == 2 * n(64) * 3 * 128
    assert L.wkv4_ckpt_floats(1, 33, 8) == 1 * n(33) * 3 * 8
    assert L.wkv4_ckpt_floats(0, 10, 8) == 0
    ws = L.wkv4_backward_workspace_bytes(2, 64, 128, 1)
    assert ws >= 2 * 2 * 128 * 4
    assert L.wkv4_backward_workspace_bytes(2, 64, 128, 0) >= ws + 2 * n(64) * 3 * 128 * 4


FAKE = 1 << 20  # 16-byte aligned, never dereferenced: every call below fails validation first


def _fwd(L, B, T, C, dt, w=FAKE, u=FAKE, k=FAKE, v=FAKE, y=FAKE, ck=None):
    return L.wkv4_forward(B, T, C, dt, w, u, k, v, y, ck, None)


def test_forward_argument_errors(W):
    L = W.lib()
    assert _fwd(L, -1, 4, 8, 0) == W.WKV_ERR_INVALID_ARG
    assert _fwd(L, 1, 4, 8, 7) == W.WKV_ERR_INVALID_ARG          # unknown dtype
    assert _fwd(L, 1, 4, 6, 0) == W.WKV_ERR_UNSUPPORTED          # C % 4
    assert _fwd(L, 1, 4, 12, 1) == W.WKV_ERR_UNSUPPORTED         # C % 8 for bf16
    assert _fwd(L, 1, 4, 8, 0, k=None) == W.WKV_ERR_INVALID_ARG
    assert b"k is NULL" in L.wkv_last_error()
    assert _fwd(L, 1, 4, 8, 0, v=FAKE + 4) == W.WKV_ERR_INVALID_ARG
    assert b"aligned" in L.wkv_last_error()
    assert _fwd(L, 1, 4, 8, 0, y=None, ck=None) == W.WKV_ERR_INVALID_ARG
    assert _fwd(L, 1, 1 << 31, 8, 0) == W.WKV_ERR_UNSUPPORTED
    # empty problems are valid no-ops and launch nothing
    assert _fwd(L, 0, 4, 8, 0) == W.WKV_OK
    assert _fwd(L, 3, 0, 8, 0) == W.WKV_OK


def test_backward_argument_errors(W):
    L = W.lib()
    args = [FAKE] * 11
    # workspace too small
    rc = L.wkv4_backward(2, 8, 8, 0, *args[:10], FAKE, 0, None)
    assert rc == W.WKV_ERR_INVALID_ARG and b"workspace" in L.wkv_last_error()
    rc = L.wkv4_backward(2, 8, 8, 0, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None)
    assert rc == W.WKV_ERR_INVALID_ARG and b"gy" in L.wkv_last_error()
    assert L.wkv4_backward(2, 8, 10, 0, *args[:10], FAKE, 1 << 30, None) == W.WKV_ERR_UNSUPPORTED


def test_gated_argument_errors(W):
    L = W.lib()
    fg = lambda B=1, T=4, C=8, dt=0, r=FAKE, y=FAKE: L.wkv4_forward_gated(B, T, C, dt, FAKE, FAKE, FAKE, FAKE, r,
                                                                          y, None, None)
    assert fg(r=None) == W.WKV_ERR_INVALID_ARG and b"r is NULL" in L.wkv_last_error()
    assert fg(y=None) == W.WKV_ERR_INVALID_ARG and b"y is NULL" in L.wkv_last_error()
    assert fg(r=FAKE + 8) == W.WKV_ERR_INVALID_ARG and b"aligned" in L.wkv_last_error()
    assert fg(C=6) == W.WKV_ERR_UNSUPPORTED
    assert fg(B=0, r=None, y=None) == W.WKV_OK
    bg = lambda T=8, r=FAKE, gr=FAKE, ws=1 << 30: L.wkv4_backward_gated(
        2, T, 8, 0, FAKE, FAKE, FAKE, FAKE, r, FAKE, None, FAKE, FAKE, gr, FAKE, FAKE, FAKE, ws, None)
    assert bg(r=None) == W.WKV_ERR_INVALID_ARG and b"r is NULL" in L.wkv_last_error()
    assert bg(gr=None) == W.WKV_ERR_INVALID_ARG and b"gr is NULL" in L.wkv_last_error()
    assert bg(ws=0) == W.WKV_ERR_INVALID_ARG and b"workspace" in L.wkv_last_error()


def test_time_shift_argument_errors(W):
    L = W.lib()
    f = lambda B=2, T=4, C=8, dt=0, n=3, x=FAKE, mix=FAKE, xp=None, out=FAKE: L.wkv4_time_shift_mix(
        B, T, C, dt, n, x, mix, xp, out, None)
    assert f(n=0) == W.WKV_ERR_INVALID_ARG and b"n_mix" in L.wkv_last_error()
    assert f(n=4) == W.WKV_ERR_INVALID_ARG
    assert f(x=None) == W.WKV_ERR_INVALID_ARG and b"x is NULL" in L.wkv_last_error()
    assert f(out=None) == W.WKV_ERR_INVALID_ARG and b"out is NULL" in L.wkv_last_error()
    assert f(xp=FAKE + 4) == W.WKV_ERR_INVALID_ARG and b"x_prev" in L.wkv_last_error()
    assert f(C=12, dt=1) == W.WKV_ERR_UNSUPPORTED
    assert f(T=0, x=None, out=None) == W.WKV_OK
    ws = L.wkv4_time_shift_mix_backward_workspace_bytes
    assert ws(2, 64, 128, 0, 3) >= 3 * 2 * 128 * 4
    assert ws(2, 64, 128, 0, 4) == 0 and ws(0, 64, 128, 0, 3) == 0
    b = lambda n=3, g=FAKE, gx=FAKE, gmix=FAKE, wsb=1 << 30: L.wkv4_time_shift_mix_backward(
        2, 64, 128, 0, n, FAKE, FAKE, None, g, gx, gmix, None, FAKE, wsb, None)
    assert b(g=None) == W.WKV_ERR_INVALID_ARG and b"g is NULL" in L.wkv_last_error()
    assert b(gmix=None) == W.WKV_ERR_INVALID_ARG and b"gmix" in L.wkv_last_error()
    assert b(wsb=16) == W.WKV_ERR_INVALID_ARG and b"workspace" in L.wkv_last_error()


def test_wkv7_backward_argument_errors(W):
    L = W.lib()
    wb = lambda K=64, dt=1, dout=FAKE, ws=1 << 30, d_init=FAKE: L.wkv7_backward(
        1, 8, 1, K, dt, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, dout, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
        d_init, FAKE, ws, None)
    assert wb(K=32) == W.WKV_ERR_UNSUPPORTED
    assert wb(dt=0) == W.WKV_ERR_UNSUPPORTED
    assert wb(dout=None) == W.WKV_ERR_INVALID_ARG and b"dout is NULL" in L.wkv_last_error()
    assert wb(d_init=None) == W.WKV_ERR_INVALID_ARG and b"d_init" in L.wkv_last_error()
    assert wb(ws=16) == W.WKV_ERR_INVALID_ARG and b"workspace" in L.wkv_last_error()
    assert L.wkv7_backward_workspace_bytes(2, 9, 3, 64) == 2 * 3 * 3 * 64 * 64 * 4
    assert L.wkv7_backward_workspace_bytes(2, 9, 3, 32) == 0


def test_time_shift_workspace_follows_the_run_split(W):
    """The backward's partial mix gradients are [n_mix][B * runs][C] floats,
    each sequence cut into runs of at least 16 tokens, about 16 CTAs of 128
    threads per SM (4 channels each) over 148 SMs."""
    L = W.lib()
    cdiv = lambda a, b: -(-a // b)
    for B, T, C, n in ((16, 4096, 4096, 3), (8, 1024, 768, 2), (1, 5, 8, 1), (2, 100000, 64, 3)):
        ncb = cdiv(C, 128 * 4)
        nrun = max(1, min(cdiv(148 * 16, B * ncb), max(1, cdiv(T, 16))))
        lt = cdiv(T, nrun)
        nrun = cdiv(T, lt)
        for dt in (0, 1):
            assert L.wkv4_time_shift_mix_backward_workspace_bytes(B, T, C, dt, n) == n * B * nrun * C * 4


def test_chunk_and_wkv6_argument_errors(W):
    L = W.lib()
    dec = lambda S=4, C=8, dt=0, k=FAKE, state=FAKE: L.wkv4_decode_step(S, C, dt, FAKE, FAKE, k, FAKE, FAKE, state,
                                                                       None)
    assert dec(k=None) == W.WKV_ERR_INVALID_ARG and b"k is NULL" in L.wkv_last_error()
    assert dec(state=FAKE + 4) == W.WKV_ERR_INVALID_ARG and b"state" in L.wkv_last_error()
    assert dec(C=6) == W.WKV_ERR_UNSUPPORTED
    assert dec(S=-1) == W.WKV_ERR_INVALID_ARG
    assert dec(S=0, k=None, state=None) == W.WKV_OK
    assert L.wkv4_chunk_step(4, 8, 0, FAKE, FAKE, FAKE, FAKE, FAKE, -1, FAKE, FAKE, None) == W.WKV_ERR_INVALID_ARG
    assert L.wkv4_chunk_step(4, 8, 0, FAKE, FAKE, FAKE, FAKE, FAKE, 10, None, FAKE, None) == W.WKV_ERR_INVALID_ARG
    assert L.wkv4_chunk_step(0, 8, 0, FAKE, FAKE, FAKE, FAKE, FAKE, 0, FAKE, FAKE, None) == W.WKV_OK
    wk6 = lambda B=1, T=4, H=2, K=64, dt=1, init=None, smap=None, ns=0: L.wkv6_forward(
        B, T, H, K, dt, FAKE, FAKE, FAKE, FAKE, FAKE, init, smap, ns, None, FAKE, None)
    assert wk6(K=32) == W.WKV_ERR_UNSUPPORTED
    assert wk6(dt=0) == W.WKV_ERR_UNSUPPORTED
    assert wk6(B=-1) == W.WKV_ERR_INVALID_ARG
    assert wk6(B=3, init=FAKE, ns=2) == W.WKV_ERR_INVALID_ARG     # n_state neither 1 nor B
    assert wk6(B=3, init=FAKE, ns=0) == W.WKV_ERR_INVALID_ARG
    assert wk6(B=0) == W.WKV_OK
    need = L.wkv6_backward_workspace_bytes(2, 40, 3, 64)
    r256 = lambda n: (n + 255) // 256 * 256
    nch = 1  # ceil(40 / 64) chunks
    assert need == 2 * r256(4 * 2 * 3 * nch * 64 * 64) + r256(4 * 2 * 3 * nch * 64)
    assert L.wkv6_backward_workspace_bytes(2, 40, 3, 32) == 0
    wb6 = lambda B=2, T=40, H=3, K=64, dt=1, init=None, ns=0, ws=need, wsp=FAKE: L.wkv6_backward(
        B, T, H, K, dt, FAKE, FAKE, FAKE, FAKE, FAKE, init, None, ns, FAKE, None,
        FAKE, FAKE, FAKE, FAKE, FAKE, None, wsp, ws, None)
    assert wb6(K=32) == W.WKV_ERR_UNSUPPORTED
    assert wb6(dt=0) == W.WKV_ERR_UNSUPPORTED
    assert wb6(T=-1) == W.WKV_ERR_INVALID_ARG
    assert wb6(ws=need - 1) == W.WKV_ERR_INVALID_ARG
    assert wb6(wsp=None) == W.WKV_ERR_INVALID_ARG
    assert wb6(init=FAKE, ns=3) == W.WKV_ERR_INVALID_ARG      # n_state neither 1 nor B
    assert wb6(H=0) == W.WKV_OK
    wk7 = lambda B=1, T=4, H=2, K=64, dt=1: L.wkv7_forward(B, T, H, K, dt, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                                           None, None, FAKE, None)
    assert wk7(K=32) == W.WKV_ERR_UNSUPPORTED
    assert wk7(dt=0) == W.WKV_ERR_UNSUPPORTED
    assert wk7(T=-1) == W.WKV_ERR_INVALID_ARG
    assert wk7(B=0) == W.WKV_OK
    assert L.wkv_wait_selfcheck(0, None) == W.WKV_ERR_INVALID_ARG
    assert L.wkv_wait_selfcheck(20_000_000_000, None) == W.WKV_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors(W):
    import torch
    k = torch.zeros(1, 4, 8)
    with pytest.raises(ValueError):
        W.wkv4_forward(torch.zeros(8), torch.zeros(8), k, k)
