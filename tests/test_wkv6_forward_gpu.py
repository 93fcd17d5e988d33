"""GPU parity of wkv6_forward against the fp64 oracle (RWKV6_OP of the
rwkv-ops package page, section "rwkv6op 使用方法")."""

import numpy as np
import pytest
import torch

from _dev import TOL, dev, host64, need_gpu, rel_err
from rwkv_wkv_linear_mix_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def W():
    need_gpu()
    from rwkv_wkv_linear_mix_b200 import wkv
    wkv.device_error(reset=True)
    return wkv


def run(W, inp, **kw):
    return W.wkv6_forward(dev(inp["r"]), dev(inp["k"]), dev(inp["v"]), dev(inp["w"]), dev(inp["u"]), **kw)


def ref(oracle, inp, H, **kw):
    return oracle.wkv6_forward(inp["r32"], inp["k32"], inp["v32"], inp["w32"], inp["u"].reshape(H, 64), **kw)


@pytest.mark.parametrize("B,T,H", [(1, 64, 1), (2, 100, 2), (1, 1, 3), (2, 257, 2), (1, 130, 1)])
def test_matches_oracle(W, oracle, B, T, H):
    inp = synth.wkv6_inputs(synth.Wkv6Recipe("t", B, T, H), seed=B + T + H)
    o, fs = run(W, inp)
    ro, rfs = ref(oracle, inp, H)
    assert rel_err(host64(o), ro) < TOL["bf16"]
    assert rel_err(host64(fs), rfs) < TOL["bf16"]
    assert W.device_error(reset=True) == 0


@pytest.mark.parametrize("d_mean,d_std,seed", [(1.0, 1.5, 5), (3.0, 1.0, 6), (-0.5, 2.0, 7)])
def test_strong_decay_subchunks(W, oracle, d_mean, d_std, seed):
    """Decays strong enough that a 64-token chunk's cumulative decay falls
    below 2^-96 (and some w round to 0 in bf16): those chunks are processed as
    16-, 4- and 1-token sub-chunks, which must agree with the plain loop."""
    B, T, H = 2, 300, 2
    rec = synth.Wkv6Recipe("t", B, T, H, d_mean=d_mean, d_std=d_std)
    inp = synth.wkv6_inputs(rec, seed=seed)
    rng = np.random.default_rng(seed)
    init = rng.normal(size=(B, H, 64, 64)).astype(np.float32)
    o, fs = run(W, inp, init_state=dev(init))
    ro, rfs = ref(oracle, inp, H, init_state=init)
    assert rel_err(host64(o), ro) < TOL["bf16"]
    assert rel_err(host64(fs), rfs) < TOL["bf16"]
    assert W.device_error(reset=True) == 0


def test_no_decay_is_linear_attention(W, oracle):
    """w = 1 (d = -30): the state only accumulates k^T v."""
    B, T, H = 1, 192, 1
    inp = synth.wkv6_inputs(synth.Wkv6Recipe("t", B, T, H, d_mean=-30.0, d_std=0.1), seed=9)
    assert np.all(inp["w32"] == 1.0)
    o, fs = run(W, inp)
    ro, rfs = ref(oracle, inp, H)
    assert rel_err(host64(o), ro) < TOL["bf16"]
    assert rel_err(host64(fs), rfs) < TOL["bf16"]


def test_init_state_and_map(W, oracle):
    B, T, H = 3, 70, 2
    inp = synth.wkv6_inputs(synth.Wkv6Recipe("t", B, T, H), seed=11)
    rng = np.random.default_rng(2)
    init = rng.normal(size=(2, H, 64, 64)).astype(np.float32)
    smap = np.array([1, 0, 1], np.int32)
    o, fs = run(W, inp, init_state=dev(init), state_map=dev(smap))
    ro, rfs = ref(oracle, inp, H, init_state=init, state_map=smap)
    assert rel_err(host64(o), ro) < TOL["bf16"]
    assert rel_err(host64(fs), rfs) < TOL["bf16"]
    o1, _ = run(W, inp, init_state=dev(init[:1]))
    ro1, _ = ref(oracle, inp, H, init_state=init[:1])
    assert rel_err(host64(o1), ro1) < TOL["bf16"]
    # out-of-range map entry: that sample starts from zero, error recorded
    bad = np.array([0, 5, 1], np.int32)
    ob, _ = run(W, inp, init_state=dev(init), state_map=dev(bad))
    assert W.device_error(reset=True) & W.WKV_DEVERR_BAD_STATE
    rz, _ = ref(oracle, {n: x[1:2] if n != "u" else x for n, x in inp.items()}, H)
    assert rel_err(host64(ob[1:2]), rz) < TOL["bf16"]


# 32 of the 256 (sample, head) pairs of the 8x4096x32 workload: four heads of
# every sample, spread over the head index
HEADS32 = [(b, (b + 8 * m + 3 * b * m) % 32) for b in range(8) for m in range(4)]


def gather_heads(inp, pairs, names):
    """The (b, h) slices of [B, T, H*64] arrays side by side as the heads of
    one [1, T, len(pairs)*64] sample (the oracle runs them in parallel), and
    their bonus vectors as u [len(pairs), 64]."""
    out = {n: np.concatenate([inp[n][b:b + 1, :, h * 64:(h + 1) * 64] for b, h in pairs], axis=2) for n in names}
    out["u"] = np.stack([inp["u"][h * 64:(h + 1) * 64] for _, h in pairs])
    return out


def test_c2048_config_32_heads(W, oracle):
    rec = synth.WKV6_RECIPES["wkv6_fwd_bf16_c2048"]
    inp = synth.wkv6_inputs(rec, seed=0)
    o, fs = run(W, inp)
    assert len(set(HEADS32)) == 32 and {b for b, _ in HEADS32} == set(range(8))
    sub = gather_heads(inp, HEADS32, ("r32", "k32", "v32", "w32"))
    ro, rfs = oracle.wkv6_forward(sub["r32"], sub["k32"], sub["v32"], sub["w32"], sub["u"])
    for m, (b, h) in enumerate(HEADS32):
        sl = slice(h * 64, (h + 1) * 64)
        assert rel_err(host64(o[b:b + 1, :, sl]), ro[:, :, m * 64:(m + 1) * 64]) < TOL["bf16"], (b, h)
        assert rel_err(host64(fs[b, h]), rfs[0, m]) < TOL["bf16"], (b, h)
    assert W.device_error(reset=True) == 0
