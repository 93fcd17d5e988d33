"""GPU checks of wkv4_decode_step, the T = 1 fast path of the slot step
(batched decode; web-rwkv crate page, section "批量推理" / batched
inference): bit-identical to wkv4_chunk_step fed one token per slot, and
equal to the whole-sequence oracle forward when a sequence is decoded token
by token after a chunked prefill."""

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


def draw(S, n, C, dtype, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    w = np.exp(rng.uniform(-6.0, 1.0, size=C)).astype(np.float32)
    u = rng.uniform(-1.0, 1.0, size=C).astype(np.float32)
    k, k32 = synth._store((rng.standard_normal((n, S, C), dtype=np.float32) * 2).astype(np.float32), dtype)
    v, v32 = synth._store(rng.standard_normal((n, S, C), dtype=np.float32), dtype)
    return w, u, k, k32, v, v32


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("S,C", [(256, 4096), (3, 8), (7, 264), (1, 1032)])
def test_equals_chunk_step_bitwise(W, dtype, S, C):
    """Several decode calls against the chunk step with cu_tokens = 0..S,
    starting from the empty past (so the first call sets each slot's
    reference exponent) and carrying the state."""
    n = 5
    w, u, k, _, v, _ = draw(S, n, C, dtype, seed=S + C)
    w, u, k, v = dev(w), dev(u), dev(k), dev(v)
    s_dec = W.wkv4_state_init(S, C, k.device)
    s_chk = W.wkv4_state_init(S, C, k.device)
    cu = torch.arange(S + 1, dtype=torch.int32, device="cuda")
    for t in range(n):
        yd = W.wkv4_decode_step(w, u, k[t], v[t], s_dec)
        yc = W.wkv4_chunk_step(w, u, k[t], v[t], cu, s_chk)
        assert torch.equal(yd, yc), f"y differs at step {t}"
        assert torch.equal(s_dec, s_chk), f"state differs at step {t}"
    assert W.device_error(reset=True) == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_prefill_then_decode_matches_oracle(W, oracle, dtype):
    """Prefill 100 tokens of each slot with the chunk step, decode 60 more
    one at a time: y equals the oracle's forward over all 160 tokens."""
    S, C, T0, T1 = 4, 136, 100, 60
    T = T0 + T1
    w, u, k, k32, v, v32 = draw(S, T, C, dtype, seed=11)
    wd, ud, kd, vd = dev(w), dev(u), dev(k), dev(v)
    state = W.wkv4_state_init(S, C, kd.device)
    # prefill: the slots' tokens packed slot by slot, one call
    kp = kd[:T0].transpose(0, 1).contiguous().reshape(S * T0, C)
    vp = vd[:T0].transpose(0, 1).contiguous().reshape(S * T0, C)
    cu = torch.arange(0, S * T0 + 1, T0, dtype=torch.int32, device="cuda")
    y0 = W.wkv4_chunk_step(wd, ud, kp, vp, cu, state).reshape(S, T0, C)
    ys = [W.wkv4_decode_step(wd, ud, kd[t], vd[t], state) for t in range(T0, T)]
    y = torch.cat([y0, torch.stack(ys, dim=1)], dim=1)
    want = oracle.wkv4_forward(w, u, k32.transpose(1, 0, 2), v32.transpose(1, 0, 2))
    assert rel_err(host64(y), want) < TOL[dtype]
    assert W.device_error(reset=True) == 0


def test_empty_batch(W):
    k = torch.zeros(0, 64, device="cuda")
    state = torch.zeros(0, 5, 64, device="cuda")
    w = torch.ones(64, device="cuda")
    assert W.wkv4_decode_step(w, w, k, k, state).shape == (0, 64)
