"""GPU parity of wkv4_forward against the fp64 oracle (RWKV-4 WKV of
RWKV_TimeMix.forward, "代码连连看——RWKV", section RWKV_TimeMix)."""

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


def run_fwd(W, inp, **kw):
    return W.wkv4_forward(dev(inp["w"]), dev(inp["u"]), dev(inp["k"]), dev(inp["v"]), **kw)


SHAPES = [
    # (B, T, C): several tiles, ragged T and C tails, one-token and one-warp cases
    (2, 64, 128), (3, 100, 72), (1, 1, 8), (2, 33, 40), (1, 257, 264), (4, 31, 96), (1, 1000, 32),
    # 257 lane groups split 4 ways: 4 warps per CTA, the last CTA with one active warp
    (1, 300, 8200),
    # few lane groups, long ragged sequence: 8-CTA clusters, two sub-segments per CTA
    (2, 1500, 96),
    # 780 lane groups, too short to split: bf16 takes the general one-segment
    # kernel (above the one-warp sequential kernel's group limit), float32 the
    # sequential kernel; the last channel block is ragged
    (12, 100, 4104),
]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,T,C", SHAPES)
def test_forward_matches_oracle(W, oracle, dtype, B, T, C):
    rec = synth.WKV4_RECIPES["wkv4_fwd_f32_small"].with_shape(B, T, C)
    rec = dataclasses.replace(rec, dtype=dtype, k_std=2.0)
    inp = synth.wkv4_inputs(rec, seed=B * 1000 + T + C)
    y = host64(run_fwd(W, inp))
    ref = oracle.wkv4_forward(inp["w"], inp["u"], inp["k32"], inp["v32"])
    assert rel_err(y, ref) < TOL[dtype]
    assert_no_device_error()


def test_small_config_exact_recipe(W, oracle):
    inp = synth.wkv4_inputs(synth.WKV4_RECIPES["wkv4_fwd_f32_small"], seed=0)
    y = host64(run_fwd(W, inp))
    ref = oracle.wkv4_forward(inp["w"], inp["u"], inp["k32"], inp["v32"])
    assert rel_err(y, ref) < TOL["f32"]


def test_169m_config_full(W, oracle):
    rec = synth.WKV4_RECIPES["wkv4_fb_f32_169m"]
    inp = synth.wkv4_inputs(rec, seed=0)
    y, ckpt = run_fwd(W, inp, want_ckpt=True)
    ref = oracle.wkv4_forward(inp["w"], inp["u"], inp["k32"], inp["v32"])
    assert rel_err(host64(y), ref) < TOL["f32"]
    assert_no_device_error()


def test_3b_config_every_channel(W, oracle):
    """The 3B-width workload (B=16, T=4096, C=2560, bf16): every output
    element against the oracle (run on blocks of channels to bound its
    memory). The error metric's RMS floor is taken over the whole tensor."""
    rec = synth.WKV4_RECIPES["wkv4_fb_bf16_3b"]
    inp = synth.wkv4_inputs(rec, seed=0)
    y = host64(run_fwd(W, inp)).astype(np.float32)
    ref = np.empty(y.shape, np.float32)
    for c0 in range(0, rec.C, 512):
        cs = slice(c0, min(rec.C, c0 + 512))
        ref[:, :, cs] = oracle.wkv4_forward(inp["w"][cs], inp["u"][cs], inp["k32"][:, :, cs], inp["v32"][:, :, cs])
    assert rel_err(y.astype(np.float64), ref.astype(np.float64)) < TOL["bf16"]
    assert_no_device_error()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_special_cases(W, oracle, dtype):
    rec = synth.WKV4_RECIPES["wkv4_fwd_f32_small"].with_shape(2, 70, 64)
    rec = dataclasses.replace(rec, dtype=dtype)
    inp = synth.wkv4_inputs(rec, seed=5)
    C = rec.C
    cases = {
        "shift_k_1000": dict(k=inp["k32"] + 1000.0),
        "shift_k_-1000": dict(k=inp["k32"] - 1000.0),
        "huge_bonus": dict(u=np.full(C, 60.0, np.float32)),
        "huge_decay": dict(w=np.full(C, np.exp(6.0), np.float32)),
        "no_decay": dict(w=np.full(C, np.exp(-30.0), np.float32), u=np.zeros(C, np.float32)),
        "constant_v": dict(v=np.broadcast_to(inp["v32"][:, :1, :], inp["v32"].shape)),
        "wide_keys": dict(k=inp["k32"] * 20.0),
    }
    for name, over in cases.items():
        w = over.get("w", inp["w"])
        u = over.get("u", inp["u"])
        k = np.ascontiguousarray(over.get("k", inp["k32"]), dtype=np.float32)
        v = np.ascontiguousarray(over.get("v", inp["v32"]), dtype=np.float32)
        if dtype == "bf16":
            kb, vb = synth.f32_to_bf16_bits(k), synth.f32_to_bf16_bits(v)
            k32, v32 = synth.bf16_bits_to_f32(kb), synth.bf16_bits_to_f32(vb)
        else:
            kb, vb, k32, v32 = k, v, k, v
        y = host64(W.wkv4_forward(dev(w), dev(u), dev(kb), dev(vb)))
        ref = oracle.wkv4_forward(w, u, k32, v32)
        assert rel_err(y, ref) < TOL[dtype], name
        if name == "constant_v":
            assert rel_err(y, v32) < TOL[dtype]
    assert_no_device_error()


def test_single_token_returns_v(W):
    rec = synth.WKV4_RECIPES["wkv4_fwd_f32_small"].with_shape(3, 1, 64)
    inp = synth.wkv4_inputs(rec, seed=7)
    y = host64(run_fwd(W, inp))
    np.testing.assert_allclose(y, inp["v32"], rtol=1e-6, atol=1e-7)


def test_deterministic_and_ckpt_only(W):
    rec = synth.WKV4_RECIPES["wkv4_fwd_f32_small"].with_shape(2, 200, 96)
    inp = synth.wkv4_inputs(rec, seed=8)
    y1, c1 = run_fwd(W, inp, want_ckpt=True)
    y2, c2 = run_fwd(W, inp, want_ckpt=True)
    assert torch.equal(y1, y2) and torch.equal(c1, c2)
    _, c3 = run_fwd(W, inp, want_ckpt=True, want_y=False)
    assert torch.equal(c1, c3)
    # entry 0 is the empty past
    assert torch.all(c1[:, 0, 0] == 0) and torch.all(c1[:, 0, 1] == 0) and torch.all(c1[:, 0, 2] == -1e38)


def test_checkpoint_state_matches_oracle(W, oracle):
    # the state before token CKPT_LEN * n, as exact sums a = aa 2^pp, b = bb 2^pp
    rec = synth.WKV4_RECIPES["wkv4_fwd_f32_small"].with_shape(2, 96, 32)
    inp = synth.wkv4_inputs(rec, seed=9)
    _, ck = run_fwd(W, inp, want_ckpt=True)
    ck = host64(ck)
    # lane reference: fl(k[b, 0, c] * log2 e) in float32
    ref_exp = (inp["k32"][:, 0, :] * np.float32(1.4426950408889634)).astype(np.float32).astype(np.float64)
    for n in (1, 2, 96 // W.CKPT_LEN - 1):
        t = W.CKPT_LEN * n
        _, st = oracle.wkv4_forward(inp["w"], inp["u"], inp["k32"][:, :t], inp["v32"][:, :t], return_state=True)
        log_b = np.log(st["b_end"]) + st["kmax"]
        ratio = st["a_end"] / st["b_end"]
        aa, bb, pp = ck[:, n, 0], ck[:, n, 1], ck[:, n, 2]
        np.testing.assert_allclose(np.log(bb) + (pp + ref_exp) * np.log(2.0), log_b, rtol=0, atol=1e-4)
        assert rel_err(aa / bb, ratio) < 1e-4


def extreme_channels(inp):
    """Give channel group 1 (channels 64..127) a bonus u far above the decay
    and group 2 a decay w far above the bonus (|u - w| beyond 44 nats, where
    the kernels switch that 64-channel group to the capped-weight output
    evaluation); group 0 keeps the recipe's values (the fast evaluation)."""
    inp = dict(inp)
    inp["u"], inp["w"] = inp["u"].copy(), inp["w"].copy()
    inp["u"][64 + 5] = 60.0
    inp["u"][64 + 40] = 35.0
    inp["w"][128 + 7] = 90.0
    inp["u"][128 + 8] = -50.0
    return inp


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,T", [(2, 150), (1, 700)])
def test_extreme_bonus_and_decay_groups(W, oracle, dtype, B, T):
    rec = synth.WKV4_RECIPES["wkv4_fwd_f32_small"].with_shape(B, T, 200)
    rec = dataclasses.replace(rec, dtype=dtype, k_std=2.0)
    inp = extreme_channels(synth.wkv4_inputs(rec, seed=11 + T))
    y = host64(run_fwd(W, inp))
    ref = oracle.wkv4_forward(inp["w"], inp["u"], inp["k32"], inp["v32"])
    assert rel_err(y, ref) < TOL[dtype]
    # the big-bonus channel follows v closely; the fast-decay channel too
    assert rel_err(y[..., 64 + 5], ref[..., 64 + 5]) < TOL[dtype]
    assert rel_err(y[..., 128 + 7], ref[..., 128 + 7]) < TOL[dtype]
    assert_no_device_error()
