"""GPU checks of wkv4_chunk_step: web-rwkv-style batched inference slots
(web-rwkv crate page, section "批量推理" / batched inference)."""

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


def feed(W, inp, chunk, w, u, k, v):
    """Feed every slot's prompt in calls of at most `chunk` tokens; return
    y in the original packed order and the final state."""
    lengths, offs = inp["lengths"], inp["offsets"]
    S, C = len(lengths), k.shape[1]
    state = W.wkv4_state_init(S, C, k.device)
    y = torch.empty_like(k)
    done = np.zeros(S, np.int64)
    for take in synth.feed_schedule(lengths, chunk):
        idx = np.concatenate([np.arange(offs[s] + done[s], offs[s] + done[s] + take[s]) for s in range(S)])
        idx_t = torch.from_numpy(idx).cuda()
        cu = torch.from_numpy(np.concatenate([[0], np.cumsum(take)]).astype(np.int32)).cuda()
        yc = W.wkv4_chunk_step(w, u, k[idx_t].contiguous(), v[idx_t].contiguous(), cu, state)
        y[idx_t] = yc
        done += take
    return y, state


@pytest.fixture(scope="module")
def slots():
    return synth.wkv4_slot_inputs(S=32, C=4096, len_lo=1, len_hi=512, dtype="bf16", seed=0)


def test_chunked_equals_whole_bitwise(W, slots):
    w, u, k, v = dev(slots["w"]), dev(slots["u"]), dev(slots["k"]), dev(slots["v"])
    y32, s32 = feed(W, slots, 32, w, u, k, v)
    yall, sall = feed(W, slots, 1 << 30, w, u, k, v)
    y7, s7 = feed(W, slots, 7, w, u, k, v)
    assert torch.equal(y32, yall) and torch.equal(s32, sall)
    assert torch.equal(y7, yall) and torch.equal(s7, sall)
    # one token per slot per call: the decode path
    short = dict(slots)
    short["lengths"] = np.minimum(slots["lengths"], 40)
    short["offsets"] = np.concatenate([[0], np.cumsum(short["lengths"])])
    idx = np.concatenate([np.arange(slots["offsets"][s], slots["offsets"][s] + short["lengths"][s])
                          for s in range(len(short["lengths"]))])
    it = torch.from_numpy(idx).cuda()
    ks, vs = k[it].contiguous(), v[it].contiguous()
    y1, s1 = feed(W, short, 1, w, u, ks, vs)
    ya, sa = feed(W, short, 1 << 30, w, u, ks, vs)
    assert torch.equal(y1, ya) and torch.equal(s1, sa)
    assert W.device_error(reset=True) == 0


def test_equals_forward_and_oracle(W, oracle, slots):
    w, u, k, v = dev(slots["w"]), dev(slots["u"]), dev(slots["k"]), dev(slots["v"])
    y, state = feed(W, slots, 32, w, u, k, v)
    offs = slots["offsets"]
    n_exact = 0
    for s in range(len(slots["lengths"])):
        a, b = int(offs[s]), int(offs[s + 1])
        yf = W.wkv4_forward(w, u, k[a:b][None].contiguous(), v[a:b][None].contiguous())
        if b - a <= 64:
            # wkv4_forward runs one segment here (sequential schedule): the same
            # float32 steps in the same order, so y is bit-identical
            assert torch.equal(yf[0], y[a:b]), f"slot {s}"
            n_exact += 1
        else:
            # the forward splits the sequence across a cluster; merging the
            # segments reorders rounding, so compare within the tolerance
            assert rel_err(host64(yf[0]), host64(y[a:b])) < TOL["bf16"], f"slot {s}"
    short = {"w": slots["w"], "u": slots["u"], "lengths": np.array([1, 17, 33, 64])}
    short["offsets"] = np.concatenate([[0], np.cumsum(short["lengths"])])
    ks = k[: int(short["offsets"][-1])].contiguous()
    vs = v[: int(short["offsets"][-1])].contiguous()
    ys, _ = feed(W, short, 32, w, u, ks, vs)
    for s in range(4):
        a, b = int(short["offsets"][s]), int(short["offsets"][s + 1])
        yf = W.wkv4_forward(w, u, ks[a:b][None].contiguous(), vs[a:b][None].contiguous())
        assert torch.equal(yf[0], ys[a:b]), f"short slot {s}"
    for s in range(len(slots["lengths"])):  # every slot against the oracle
        a, b = int(offs[s]), int(offs[s + 1])
        ref, st = oracle.wkv4_forward(slots["w"], slots["u"], slots["k32"][None, a:b], slots["v32"][None, a:b],
                                      return_state=True)
        assert rel_err(host64(y[a:b]), ref[0]) < TOL["bf16"]
        aa, bb, base, n, ref = (host64(state[s, i]) for i in range(5))
        P = base - n * slots["w"].astype(np.float64) * np.log2(np.e)
        np.testing.assert_allclose(np.log(bb) + (P + ref) * np.log(2.0), np.log(st["b_end"][0]) + st["kmax"][0],
                                   rtol=0, atol=1e-3)
        assert rel_err(aa / bb, st["a_end"][0] / st["b_end"][0]) < 1e-3


def test_empty_slots_untouched_and_bad_ranges(W):
    S, C = 6, 64
    rng = np.random.default_rng(3)
    w = dev(np.exp(rng.uniform(-6, 1, C)).astype(np.float32))
    u = dev(rng.uniform(-1, 1, C).astype(np.float32))
    take = np.array([3, 0, 5, 0, 1, 2])
    n = int(take.sum())
    k = dev(rng.normal(size=(n, C)).astype(np.float32))
    v = dev(rng.normal(size=(n, C)).astype(np.float32))
    state = W.wkv4_state_init(S, C, k.device)
    state.normal_()
    before = state.clone()
    cu = torch.from_numpy(np.concatenate([[0], np.cumsum(take)]).astype(np.int32)).cuda()
    W.wkv4_chunk_step(w, u, k, v, cu, state)
    for s in range(S):
        assert torch.equal(state[s], before[s]) == (take[s] == 0)
    assert W.device_error(reset=True) == 0
    # decreasing or out-of-range slots are skipped and reported
    bad = torch.tensor([0, 3, 2, 100, 100, 101, n], dtype=torch.int32, device="cuda")
    before = state.clone()
    W.wkv4_chunk_step(w, u, k, v, bad, state)
    assert W.device_error(reset=True) & W.WKV_DEVERR_BAD_SLOT
    for s in (1, 2, 4):
        assert torch.equal(state[s], before[s])


def test_state_init_values(W):
    st = W.wkv4_state_init(3, 16, "cuda")
    assert torch.all(st[:, 0] == 0) and torch.all(st[:, 1] == 0) and torch.all(st[:, 2] == -1e38)
    assert torch.all(st[:, 3] == 0) and torch.all(st[:, 4] == 0)


def test_large_keys_keep_precision(W, oracle):
    # keys shifted by 1000: the per-slot reference keeps the exponents small
    S, C = 3, 64
    inp = synth.wkv4_slot_inputs(S=S, C=C, len_lo=40, len_hi=90, dtype="f32", seed=4)
    k = (inp["k32"] + np.float32(1000.0)).astype(np.float32)
    y, _ = feed(W, inp, 16, dev(inp["w"]), dev(inp["u"]), dev(k), dev(inp["v32"]))
    offs = inp["offsets"]
    for s in range(S):
        a, b = int(offs[s]), int(offs[s + 1])
        ref = oracle.wkv4_forward(inp["w"], inp["u"], k[None, a:b], inp["v32"][None, a:b])
        assert rel_err(host64(y[a:b]), ref[0]) < TOL["f32"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_extreme_groups_chunked_equals_forward_bitwise(W, oracle, dtype):
    """Channel groups on the capped-weight output evaluation (|u - w| beyond
    44 nats) next to groups on the fast one: chunked feeding still equals the
    whole-sequence forward bit for bit, and both match the oracle."""
    from test_wkv4_forward_gpu import extreme_channels
    sl = synth.wkv4_slot_inputs(S=4, C=200, dtype=dtype, seed=3, lengths=np.array([1, 17, 33, 64]))
    sl = extreme_channels(sl)
    w, u, k, v = dev(sl["w"]), dev(sl["u"]), dev(sl["k"]), dev(sl["v"])
    y, _ = feed(W, sl, 7, w, u, k, v)
    offs = sl["offsets"]
    for s in range(4):
        a, b = int(offs[s]), int(offs[s + 1])
        yf = W.wkv4_forward(w, u, k[a:b][None].contiguous(), v[a:b][None].contiguous())
        assert torch.equal(yf[0], y[a:b]), f"slot {s}"
        ref = oracle.wkv4_forward(sl["w"], sl["u"], sl["k32"][None, a:b], sl["v32"][None, a:b])
        assert rel_err(host64(y[a:b]), ref[0]) < TOL[dtype], f"slot {s}"
    assert W.device_error(reset=True) == 0
