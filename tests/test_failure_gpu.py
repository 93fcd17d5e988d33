"""Failure detection without a GPU fault: a bounded wait that runs out
records WKV_DEVERR_WAIT_TIMEOUT, the host reads it through wkv_device_error,
and the context stays usable for the next call."""

import dataclasses

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


def test_wait_that_runs_out_is_reported(W, oracle):
    assert W.device_error(reset=True) == 0
    W.wait_selfcheck(limit_ns=2_000_000)  # 2 ms on a barrier nothing completes
    assert W.device_error(reset=True) == W.WKV_DEVERR_WAIT_TIMEOUT
    assert W.device_error(reset=True) == 0  # cleared by the read
    # the context is intact: a forward right after it is still exact
    rec = dataclasses.replace(synth.WKV4_RECIPES["wkv4_fwd_f32_small"].with_shape(2, 80, 128), k_std=2.0)
    inp = synth.wkv4_inputs(rec, seed=1)
    y = W.wkv4_forward(dev(inp["w"]), dev(inp["u"]), dev(inp["k"]), dev(inp["v"]))
    ref = oracle.wkv4_forward(inp["w"], inp["u"], inp["k32"], inp["v32"])
    assert rel_err(host64(y), ref) < TOL["f32"]
    assert W.device_error(reset=True) == 0


def test_bad_state_map_entry_is_reported(W):
    """An out-of-range state_map entry starts that sample from zero and
    records WKV_DEVERR_BAD_STATE (forward and backward of RWKV-6)."""
    B, T, H = 2, 40, 1
    inp = synth.wkv6_inputs(synth.Wkv6Recipe("t", B, T, H), seed=4)
    r, k, v, w, u = (dev(inp[n]) for n in ("r", "k", "v", "w", "u"))
    init = torch.randn(1, H, 64, 64, device="cuda")
    smap = torch.tensor([0, 5], dtype=torch.int32, device="cuda")
    W.wkv6_forward(r, k, v, w, u, init_state=init, state_map=smap)
    assert W.device_error(reset=True) == W.WKV_DEVERR_BAD_STATE
    W.wkv6_backward(r, k, v, w, u, r, init_state=init, state_map=smap)
    assert W.device_error(reset=True) == W.WKV_DEVERR_BAD_STATE
