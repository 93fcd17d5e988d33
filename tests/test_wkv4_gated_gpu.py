"""GPU parity of the fused time-mix gate, y = sigmoid(r) * WKV ("代码连连看——
RWKV", section RWKV_TimeMix), forward and backward, against the fp64 oracle's
gated forward and its chain-rule gradients."""

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


def draw(B, T, C, dtype, seed, recipe="wkv4_fb_f32_169m"):
    rec = dataclasses.replace(synth.WKV4_RECIPES[recipe].with_shape(B, T, C), dtype=dtype)
    inp = synth.wkv4_inputs(rec, seed=seed)
    inp["r"], inp["r32"] = synth.gate_input((B, T, C), dtype, seed=seed)
    return inp


def on_dev(inp):
    return [dev(inp[n]) for n in ("w", "u", "k", "v", "r")]


SHAPES = [(2, 64, 128), (3, 100, 72), (1, 1, 8), (2, 33, 40), (1, 257, 264), (2, 500, 32),
          (1, 300, 8200)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,T,C", SHAPES)
def test_forward_matches_oracle(W, oracle, dtype, B, T, C):
    inp = draw(B, T, C, dtype, seed=B * 5 + T + C)
    w, u, k, v, r = on_dev(inp)
    y = W.wkv4_forward_gated(w, u, k, v, r)
    want = oracle.wkv4_forward_gated(inp["w"], inp["u"], inp["k32"], inp["v32"], inp["r32"])
    assert rel_err(host64(y), want) < TOL[dtype]
    assert_no_device_error()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,T,C", SHAPES)
def test_backward_matches_oracle(W, oracle, dtype, B, T, C):
    inp = draw(B, T, C, dtype, seed=B * 11 + T + 3 * C)
    w, u, k, v, r = on_dev(inp)
    gy = dev(inp["gy"])
    _, ck = W.wkv4_forward_gated(w, u, k, v, r, want_ckpt=True)
    got = W.wkv4_backward_gated(w, u, k, v, r, gy, ck)
    want = oracle.wkv4_backward_gated(inp["w"], inp["u"], inp["k32"], inp["v32"], inp["r32"], inp["gy32"])
    for name, g, ref in zip(("gk", "gv", "gr", "gw", "gu"), got, want):
        assert rel_err(host64(g), ref) < TOL[dtype], name
    assert_no_device_error()


def test_169m_config_full(W, oracle):
    """The RWKV-4 169M shape (B=8, T=1024, C=768, float32), every element."""
    rec = synth.WKV4_RECIPES["wkv4_fb_f32_169m"]
    inp = draw(rec.B, rec.T, rec.C, "f32", seed=0)
    w, u, k, v, r = on_dev(inp)
    gy = dev(inp["gy"])
    y, ck = W.wkv4_forward_gated(w, u, k, v, r, want_ckpt=True)
    got = W.wkv4_backward_gated(w, u, k, v, r, gy, ck)
    assert rel_err(host64(y), oracle.wkv4_forward_gated(inp["w"], inp["u"], inp["k32"], inp["v32"],
                                                        inp["r32"])) < TOL["f32"]
    want = oracle.wkv4_backward_gated(inp["w"], inp["u"], inp["k32"], inp["v32"], inp["r32"], inp["gy32"])
    for name, g, ref in zip(("gk", "gv", "gr", "gw", "gu"), got, want):
        assert rel_err(host64(g), ref) < TOL["f32"], name
    assert_no_device_error()


def test_c4096_bf16_sampled_channels(W, oracle):
    """The bf16 C = 4096 roofline shape: the whole problem runs on the GPU;
    18 channels are checked against the oracle on their slices (channels
    are independent)."""
    rec = synth.WKV4_RECIPES["wkv4_fb_bf16_c4096"]
    inp = draw(rec.B, rec.T, rec.C, "bf16", seed=1, recipe="wkv4_fb_bf16_c4096")
    w, u, k, v, r = on_dev(inp)
    gy = dev(inp["gy"])
    y, ck = W.wkv4_forward_gated(w, u, k, v, r, want_ckpt=True)
    gk, gv, gr, gw, gu = W.wkv4_backward_gated(w, u, k, v, r, gy, ck)
    torch.cuda.synchronize()
    rng = np.random.default_rng(4)
    cs = np.unique(np.concatenate([rng.choice(rec.C, size=16, replace=False), [0, rec.C - 1]]))
    ci = torch.from_numpy(cs).cuda()
    sl = lambda a: np.ascontiguousarray(a[:, :, cs])
    args = (inp["w"][cs], inp["u"][cs], sl(inp["k32"]), sl(inp["v32"]), sl(inp["r32"]))
    assert rel_err(host64(y[:, :, ci]), oracle.wkv4_forward_gated(*args)) < TOL["bf16"]
    want = oracle.wkv4_backward_gated(*args, sl(inp["gy32"]))
    for name, g, ref in zip(("gk", "gv", "gr", "gw", "gu"), (gk[:, :, ci], gv[:, :, ci], gr[:, :, ci], gw[ci],
                                                             gu[ci]), want):
        assert rel_err(host64(g), ref) < TOL["bf16"], name
    assert_no_device_error()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_open_gate_is_the_plain_wkv(W, dtype):
    """r = 40: sigmoid(r) rounds to exactly 1 in float32, so the gated kernels
    must give the ungated results bit for bit and dL/dr = 0."""
    B, T, C = 2, 200, 136
    inp = draw(B, T, C, dtype, seed=8)
    w, u, k, v, _ = on_dev(inp)
    r = torch.full_like(k, 40.0)
    gy = dev(inp["gy"])
    y0, ck = W.wkv4_forward(w, u, k, v, want_ckpt=True)
    y1 = W.wkv4_forward_gated(w, u, k, v, r)
    assert torch.equal(y0, y1)
    gk0, gv0, gw0, gu0 = W.wkv4_backward(w, u, k, v, gy, ck)
    gk1, gv1, gr1, gw1, gu1 = W.wkv4_backward_gated(w, u, k, v, r, gy, ck)
    for a, b in ((gk0, gk1), (gv0, gv1), (gw0, gw1), (gu0, gu1)):
        assert torch.equal(a, b)
    assert torch.count_nonzero(gr1).item() == 0
    assert_no_device_error()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_regenerated_checkpoints_match(W, dtype):
    """ckpt = NULL regenerates the checkpoints in the workspace: same bits."""
    B, T, C = 2, 170, 200
    inp = draw(B, T, C, dtype, seed=9)
    w, u, k, v, r = on_dev(inp)
    gy = dev(inp["gy"])
    _, ck = W.wkv4_forward_gated(w, u, k, v, r, want_ckpt=True)
    a = W.wkv4_backward_gated(w, u, k, v, r, gy, ck)
    b = W.wkv4_backward_gated(w, u, k, v, r, gy, None)
    for x, z in zip(a, b):
        assert torch.equal(x, z)
    assert_no_device_error()


def test_gated_checkpoints_are_the_plain_ones(W):
    """The state does not see the gate: the gated forward writes the same
    checkpoints as the plain forward."""
    inp = draw(2, 123, 96, "bf16", seed=10)
    w, u, k, v, r = on_dev(inp)
    _, c0 = W.wkv4_forward(w, u, k, v, want_ckpt=True)
    _, c1 = W.wkv4_forward_gated(w, u, k, v, r, want_ckpt=True)
    assert torch.equal(c0, c1)


def test_empty_sequence(W):
    z = torch.zeros((2, 0, 64), device="cuda")
    w = torch.ones(64, device="cuda")
    gk, gv, gr, gw, gu = W.wkv4_backward_gated(w, w, z, z, z, z)
    torch.cuda.synchronize()
    assert gr.shape == (2, 0, 64)
    assert torch.count_nonzero(gw).item() == 0 and torch.count_nonzero(gu).item() == 0
    y = W.wkv4_forward_gated(w, w, z, z, z)
    assert y.shape == (2, 0, 64)
