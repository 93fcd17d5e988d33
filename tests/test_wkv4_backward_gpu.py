"""GPU parity of wkv4_backward against the fp64 oracle's backward."""

import dataclasses

import numpy as np
import pytest
import torch

from _dev import TOL, assert_no_device_error, dev, host64, need_gpu, rel_err
from rwkv_wkv_linear_mix_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def W():
    need_gpu()
    from rwkv_wkv_linear_mix_b200 import wkv
    wkv.device_error(reset=True)
    return wkv


def run_bwd(W, inp, with_ckpt=True):
    w, u, k, v, gy = (dev(inp[n]) for n in ("w", "u", "k", "v", "gy"))
    ck = None
    if with_ckpt:
        _, ck = W.wkv4_forward(w, u, k, v, want_ckpt=True)
    return W.wkv4_backward(w, u, k, v, gy, ck)


def check(grads, ref, dtype, tol_param=None):
    gk, gv, gw, gu = (host64(g) for g in grads)
    rgk, rgv, rgw, rgu = ref
    tol = TOL[dtype]
    assert rel_err(gk, rgk) < tol, "gk"
    assert rel_err(gv, rgv) < tol, "gv"
    tp = tol_param or tol
    assert rel_err(gw, rgw) < tp, "gw"
    assert rel_err(gu, rgu) < tp, "gu"


SHAPES = [(2, 64, 128), (3, 100, 72), (1, 1, 8), (2, 33, 40), (1, 257, 264), (2, 500, 32),
          # 257 lane groups split 4 ways: 4 warps per CTA, the last CTA with one active warp
          (1, 300, 8200)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,T,C", SHAPES)
def test_backward_matches_oracle(W, oracle, dtype, B, T, C):
    rec = dataclasses.replace(synth.WKV4_RECIPES["wkv4_fb_f32_169m"].with_shape(B, T, C), dtype=dtype)
    inp = synth.wkv4_inputs(rec, seed=B * 7 + T * 3 + C)
    grads = run_bwd(W, inp)
    ref = oracle.wkv4_backward(inp["w"], inp["u"], inp["k32"], inp["v32"], inp["gy32"])
    check(grads, ref, dtype)
    assert_no_device_error()


def test_169m_config_full(W, oracle):
    rec = synth.WKV4_RECIPES["wkv4_fb_f32_169m"]
    inp = synth.wkv4_inputs(rec, seed=0)
    grads = run_bwd(W, inp)
    ref = oracle.wkv4_backward(inp["w"], inp["u"], inp["k32"], inp["v32"], inp["gy32"])
    check(grads, ref, "f32")
    assert_no_device_error()


def test_3b_config_every_channel(W, oracle):
    """The 3B-width workload (B=16, T=4096, C=2560, bf16): every gradient
    element against the oracle (run on blocks of channels to bound its
    memory; each channel's gw, gu depend on that channel only)."""
    rec = synth.WKV4_RECIPES["wkv4_fb_bf16_3b"]
    inp = synth.wkv4_inputs(rec, seed=0)
    got = [host64(x).astype(np.float32) for x in run_bwd(W, inp)]
    ref = [np.empty(g.shape, np.float32) for g in got]
    for c0 in range(0, rec.C, 512):
        cs = slice(c0, min(rec.C, c0 + 512))
        part = oracle.wkv4_backward(inp["w"][cs], inp["u"][cs], inp["k32"][:, :, cs], inp["v32"][:, :, cs],
                                    inp["gy32"][:, :, cs])
        ref[0][:, :, cs], ref[1][:, :, cs], ref[2][cs], ref[3][cs] = part
    for name, g, r in zip(("gk", "gv", "gw", "gu"), got, ref):
        assert rel_err(g.astype(np.float64), r.astype(np.float64)) < TOL["bf16"], name
    assert_no_device_error()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_without_checkpoints_is_identical(W, dtype):
    rec = dataclasses.replace(synth.WKV4_RECIPES["wkv4_fb_f32_169m"].with_shape(2, 150, 96), dtype=dtype)
    inp = synth.wkv4_inputs(rec, seed=3)
    a = run_bwd(W, inp, with_ckpt=True)
    b = run_bwd(W, inp, with_ckpt=False)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    c = run_bwd(W, inp, with_ckpt=True)
    for x, y in zip(a, c):
        assert torch.equal(x, y)  # deterministic, including the batch sums


def test_special_cases(W, oracle):
    rec = synth.WKV4_RECIPES["wkv4_fb_f32_169m"].with_shape(2, 80, 32)
    inp = synth.wkv4_inputs(rec, seed=4)
    C = rec.C
    cases = {
        "shift_k_1000": dict(k=inp["k32"] + 1000.0),
        "huge_bonus": dict(u=np.full(C, 30.0, np.float32)),
        "huge_decay": dict(w=np.full(C, np.exp(6.0), np.float32)),
        "no_decay": dict(w=np.full(C, np.exp(-30.0), np.float32)),
    }
    for name, over in cases.items():
        w = over.get("w", inp["w"])
        u = over.get("u", inp["u"])
        k = np.ascontiguousarray(over.get("k", inp["k32"]), dtype=np.float32)
        v, gy = inp["v32"], inp["gy32"]
        _, ck = W.wkv4_forward(dev(w), dev(u), dev(k), dev(v), want_ckpt=True)
        grads = W.wkv4_backward(dev(w), dev(u), dev(k), dev(v), dev(gy), ck)
        ref = oracle.wkv4_backward(w, u, k, v, gy)
        check(grads, ref, "f32")
    # constant v: only gv is non-zero, and it sums to sum(gy) per lane
    v = np.ascontiguousarray(np.broadcast_to(inp["v32"][:, :1], inp["v32"].shape))
    gk, gv, gw, gu = (host64(g) for g in W.wkv4_backward(dev(inp["w"]), dev(inp["u"]), dev(inp["k32"]), dev(v),
                                                         dev(inp["gy32"])))
    assert np.max(np.abs(gk)) < 1e-4 and np.max(np.abs(gu)) < 1e-3 and np.max(np.abs(gw)) < 1e-2
    np.testing.assert_allclose(gv.sum(axis=1), inp["gy32"].sum(axis=1), rtol=1e-4, atol=1e-3)
    assert_no_device_error()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_extreme_bonus_and_decay_groups(W, oracle, dtype):
    from test_wkv4_forward_gpu import extreme_channels
    rec = dataclasses.replace(synth.WKV4_RECIPES["wkv4_fb_f32_169m"].with_shape(2, 300, 200), dtype=dtype)
    inp = extreme_channels(synth.wkv4_inputs(rec, seed=5))
    grads = run_bwd(W, inp)
    ref = oracle.wkv4_backward(inp["w"], inp["u"], inp["k32"], inp["v32"], inp["gy32"])
    check(grads, ref, dtype)
    assert_no_device_error()
