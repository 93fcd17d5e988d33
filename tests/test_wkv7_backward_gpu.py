"""GPU parity of wkv7_backward (gradients of the RWKV-7 generalized delta
rule; generalized_delta_rule of the rwkv-ops package page carries gradients)
against the fp64 oracle's backward, which is pinned by finite differences."""

import numpy as np
import pytest
import torch

from _dev import TOL, dev, host64, need_gpu, rel_err
from rwkv_wkv_linear_mix_b200 import synth

pytestmark = pytest.mark.gpu

NAMES = ("r", "w", "k", "v", "a", "b")
GRADS = ("dr", "dw", "dk", "dv", "da", "db", "d_init")


@pytest.fixture(scope="module")
def W():
    need_gpu()
    from rwkv_wkv_linear_mix_b200 import wkv
    wkv.device_error(reset=True)
    return wkv


def draw(B, T, H, seed):
    inp = synth.wkv7_inputs(synth.Wkv7Recipe("t", B, T, H), seed=seed)
    rng = np.random.Generator(np.random.PCG64(seed + 101))
    inp["do"], inp["do32"] = synth._store(rng.standard_normal((B, T, H * 64), dtype=np.float32), "bf16")
    return inp


def check(got, want, skip=()):
    for name, g, r in zip(GRADS, got, want):
        if name in skip:
            continue
        e = rel_err(host64(g), r)
        assert e < TOL["bf16"], f"{name}: {e:.3g}"


@pytest.mark.parametrize("B,T,H", [(1, 8, 1), (2, 37, 2), (1, 1, 3), (2, 130, 1), (1, 6, 2)])
def test_matches_oracle(W, oracle, B, T, H):
    inp = draw(B, T, H, seed=B * 7 + T + H)
    rng = np.random.default_rng(T + H)
    init = rng.normal(size=(B, H, 64, 64)).astype(np.float32)
    gfin = rng.normal(size=(B, H, 64, 64)).astype(np.float32)
    got = W.wkv7_backward(*(dev(inp[n]) for n in NAMES), dev(inp["do"]), init_state=dev(init), g_final=dev(gfin))
    want = oracle.wkv7_backward(*(inp[n + "32"] for n in NAMES), inp["do32"], init_state=init, g_final=gfin)
    check(got, want)
    assert W.device_error(reset=True) == 0


def test_zero_initial_state_no_final_gradient(W, oracle):
    B, T, H = 2, 65, 2
    inp = draw(B, T, H, seed=3)
    got = W.wkv7_backward(*(dev(inp[n]) for n in NAMES), dev(inp["do"]))
    want = oracle.wkv7_backward(*(inp[n + "32"] for n in NAMES), inp["do32"])
    check(got, want)


def test_empty_sequence(W):
    """T = 0: nothing flows through time, d_init = g_final."""
    B, H = 2, 1
    z = torch.zeros((B, 0, 64), dtype=torch.bfloat16, device="cuda")
    gfin = torch.randn(B, H, 64, 64, device="cuda")
    *_, d_init = W.wkv7_backward(z, z, z, z, z, z, z, g_final=gfin)
    torch.cuda.synchronize()
    assert torch.equal(d_init, gfin)


def test_full_size_sampled_heads(W, oracle):
    """The bench shape (B=8, T=4096, H=32): every head runs on the GPU; two
    (sample, head) pairs are checked against the oracle on their slices."""
    rec = synth.WKV7_RECIPES["wkv7_fwd_bf16_c2048"]
    B, T, H = rec.B, rec.T, rec.H
    inp = draw(B, T, H, seed=0)
    got = W.wkv7_backward(*(dev(inp[n]) for n in NAMES), dev(inp["do"]))
    torch.cuda.synchronize()
    for bb, hh in ((0, 0), (6, 29)):
        cols = slice(hh * 64, (hh + 1) * 64)
        sl = [np.ascontiguousarray(inp[n + "32"][bb:bb + 1, :, cols]) for n in NAMES]
        want = oracle.wkv7_backward(*sl, np.ascontiguousarray(inp["do32"][bb:bb + 1, :, cols]))
        for name, g, r in zip(GRADS[:6], got[:6], want[:6]):
            e = rel_err(host64(g[bb:bb + 1, :, cols]), r)
            assert e < TOL["bf16"], f"{name} (b={bb}, h={hh}): {e:.3g}"
        e = rel_err(host64(got[6][bb:bb + 1, hh:hh + 1]), want[6])
        assert e < TOL["bf16"], f"d_init (b={bb}, h={hh}): {e:.3g}"
    assert W.device_error(reset=True) == 0
