"""GPU parity of wkv7_forward (RWKV-7 generalized delta rule, rwkv-ops
package page: generalized_delta_rule / rwkv7_op, and rwkv7_op_rnn for the
one-token decode step) against the fp64 oracle."""

import numpy as np
import pytest
import torch

from _dev import TOL, dev, host64, need_gpu, rel_err
from rwkv_wkv_linear_mix_b200 import synth

pytestmark = pytest.mark.gpu

NAMES = ("r", "w", "k", "v", "a", "b")


@pytest.fixture(scope="module")
def W():
    need_gpu()
    from rwkv_wkv_linear_mix_b200 import wkv
    wkv.device_error(reset=True)
    return wkv


def run(W, inp, **kw):
    return W.wkv7_forward(*(dev(inp[n]) for n in NAMES), **kw)


def ref(oracle, inp, **kw):
    return oracle.wkv7_forward(*(inp[n + "32"] for n in NAMES), **kw)


@pytest.mark.parametrize("B,T,H", [(1, 64, 1), (2, 100, 2), (1, 1, 3), (2, 257, 2), (1, 33, 1), (3, 96, 1)])
def test_matches_oracle(W, oracle, B, T, H):
    inp = synth.wkv7_inputs(synth.Wkv7Recipe("t", B, T, H), seed=B * 13 + T + H)
    init = np.random.default_rng(T).normal(size=(B, H, 64, 64)).astype(np.float32)
    o, fs = run(W, inp, init_state=dev(init))
    ro, rfs = ref(oracle, inp, init_state=init)
    assert rel_err(host64(o), ro) < TOL["bf16"]
    assert rel_err(host64(fs), rfs) < TOL["bf16"]
    assert W.device_error(reset=True) == 0


def test_zero_initial_state(W, oracle):
    inp = synth.wkv7_inputs(synth.Wkv7Recipe("t", 2, 130, 2), seed=5)
    o, fs = run(W, inp)
    ro, rfs = ref(oracle, inp)
    assert rel_err(host64(o), ro) < TOL["bf16"]
    assert rel_err(host64(fs), rfs) < TOL["bf16"]


def test_delta_rule_reads_back_what_it_wrote(W):
    """w = 0, a = -kappa, b = k = r = kappa: o_t = v_t (up to the bf16
    rounding of kappa), whatever the state before."""
    B, T, H = 1, 50, 2
    rng = np.random.default_rng(7)
    kap = rng.normal(size=(B, T, H, 64))
    kap /= np.linalg.norm(kap, axis=-1, keepdims=True)
    kap = kap.reshape(B, T, H * 64).astype(np.float32)
    v = rng.normal(size=(B, T, H * 64)).astype(np.float32)
    bf = lambda x: torch.from_numpy(x).cuda().to(torch.bfloat16)
    z = torch.zeros(B, T, H * 64, dtype=torch.bfloat16, device="cuda")
    init = torch.randn(B, H, 64, 64, device="cuda")
    o, _ = W.wkv7_forward(bf(kap), z, bf(kap), bf(v), bf(-kap), bf(kap), init_state=init)
    assert rel_err(host64(o), v.astype(np.float64)) < TOL["bf16"]


def test_fed_one_token_at_a_time_is_bitwise_the_whole_sequence(W):
    """The decode step (T = 1 per call, state carried in fp32) gives the same
    bits as one call over the whole sequence."""
    inp = synth.wkv7_inputs(synth.Wkv7Recipe("t", 2, 40, 2), seed=8)
    t = {n: dev(inp[n]) for n in NAMES}
    o_all, fs_all = W.wkv7_forward(*(t[n] for n in NAMES))
    state = None
    outs = []
    for s in range(40):
        step = [t[n][:, s:s + 1].contiguous() for n in NAMES]
        o1, state = W.wkv7_forward(*step, init_state=state)
        outs.append(o1)
    assert torch.equal(torch.cat(outs, dim=1), o_all)
    assert torch.equal(state, fs_all)


def test_full_size_sampled_heads(W, oracle):
    rec = synth.WKV7_RECIPES["wkv7_fwd_bf16_c2048"]
    inp = synth.wkv7_inputs(rec, seed=0)
    o, fs = run(W, inp)
    torch.cuda.synchronize()
    for b, h in ((0, 0), (5, 21)):
        cols = slice(h * 64, (h + 1) * 64)
        sl = {n + "32": inp[n + "32"][b:b + 1, :, cols] for n in NAMES}
        ro, rfs = ref(oracle, sl)
        assert rel_err(host64(o[b:b + 1, :, cols]), ro) < TOL["bf16"], (b, h)
        assert rel_err(host64(fs[b:b + 1, h:h + 1]), rfs) < TOL["bf16"], (b, h)
    assert W.device_error(reset=True) == 0
