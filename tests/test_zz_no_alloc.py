"""wkv4_backward_noalloc: the backward for callers that cannot allocate.

Some callers of this library cannot hand it a workspace: code reached through a
plain C interface that only receives the tensors it reads and writes, or
latency-critical loops that must not call cudaMalloc/cudaFree. For them
wkv4_backward_noalloc runs the same kernels with the workspace in a static
4 MiB device array. These tests check, through the C ABI, that it returns
exactly what wkv4_backward returns (the same deterministic kernels on the same
launch shape, so every bit must agree), on two calls in a row (so the second
call also runs on whatever the first left in the shared array), after a call
that filled the array's partial sums with NaN (so a read of a scratch element
the call did not write would show), and that it refuses problems too large for
the array. This file is collected last on purpose.
"""

import ctypes

import numpy as np
import pytest
import torch

from _dev import dev, host64, need_gpu, rel_err
from rwkv_wkv_linear_mix_b200 import synth


def _lib():
    from rwkv_wkv_linear_mix_b200 import build
    build.build()
    from rwkv_wkv_linear_mix_b200 import wkv
    return wkv


def test_refuses_problems_above_the_static_scratch():
    W = _lib()
    L = W.lib()
    FAKE = 1 << 20
    # B*C so large that the 2*B*C partial sums alone exceed the array: refused
    # on the host before any CUDA call
    rc = L.wkv4_backward_noalloc(1024, 64, 1024, 0, *([FAKE] * 11))
    assert rc == W.WKV_ERR_UNSUPPORTED
    assert b"4 MiB" in L.wkv_last_error()


@pytest.mark.gpu
def test_matches_workspace_entry_point_twice():
    need_gpu()
    W = _lib()
    W.device_error(reset=True)
    # leave NaN partial sums in the shared array: the comparisons below must
    # not see any of them
    rec0 = synth.WKV4_RECIPES["wkv4_fb_f32_169m"].with_shape(4, 64, 1024)
    inp0 = synth.wkv4_inputs(rec0, seed=99)
    w0, u0, k0, gy0 = (dev(inp0[n]) for n in ("w", "u", "k", "gy"))
    v0 = torch.full_like(k0, float("nan"))
    gw0 = W.wkv4_backward_noalloc(w0, u0, k0, v0, gy0)[2]
    torch.cuda.synchronize()
    assert torch.isnan(gw0).all()
    cases = [
        # (B, T, C, dtype, with_ckpt): first call regenerates the checkpoints
        # inside the static array, second passes them in
        (3, 100, 72, "f32", False),
        (2, 257, 264, "bf16", True),
    ]
    for i, (B, T, C, dtype, with_ckpt) in enumerate(cases):
        rec = synth.WKV4_RECIPES["wkv4_fb_f32_169m"].with_shape(B, T, C)
        rec = synth.Wkv4Recipe(**{**rec.__dict__, "dtype": dtype})
        inp = synth.wkv4_inputs(rec, seed=100 + i)
        w, u, k, v, gy = (dev(inp[n]) for n in ("w", "u", "k", "v", "gy"))
        ck = W.wkv4_forward(w, u, k, v, want_ckpt=True)[1] if with_ckpt else None
        ref = W.wkv4_backward(w, u, k, v, gy, ck)
        got = W.wkv4_backward_noalloc(w, u, k, v, gy, ck)
        torch.cuda.synchronize()
        for name, a, b in zip(("gk", "gv", "gw", "gu"), got, ref):
            assert torch.equal(a, b), (i, name, rel_err(host64(a), host64(b)))
    assert W.device_error(reset=True) == 0
