"""GPU parity of wkv6_backward against the fp64 oracle's backward (the
gradients of RWKV6_OP, rwkv-ops package page, section "rwkv6op 使用方法"; the
op is trained: its table lists the PyTorch CUDA version).

The kernel returns glogw = w * dL/dw (the gradient with respect to log w);
the oracle's dL/dw is multiplied by the same stored w before comparing."""

import numpy as np
import pytest
import torch

from _dev import TOL, dev, host64, need_gpu, rel_err
from _pins import rel_err as rel_err_floor
from rwkv_wkv_linear_mix_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def W():
    need_gpu()
    from rwkv_wkv_linear_mix_b200 import wkv
    wkv.device_error(reset=True)
    return wkv


def draw(B, T, H, seed, **rec):
    """One workload plus dout ~ N(0, 1), stored in bf16 like r, k, v."""
    inp = synth.wkv6_inputs(synth.Wkv6Recipe("t", B, T, H, **rec), seed=seed)
    rng = np.random.Generator(np.random.PCG64(seed + 7919))
    inp["do"], inp["do32"] = synth._store(rng.standard_normal(size=(B, T, H * 64), dtype=np.float32), "bf16")
    return inp


def run(W, inp, **kw):
    return W.wkv6_backward(dev(inp["r"]), dev(inp["k"]), dev(inp["v"]), dev(inp["w"]), dev(inp["u"]),
                           dev(inp["do"]), **kw)


def ref(oracle, inp, H, **kw):
    gr, gk, gv, gw, gu, gi = oracle.wkv6_backward(inp["r32"], inp["k32"], inp["v32"], inp["w32"],
                                                  inp["u"].reshape(H, 64), inp["do32"], **kw)
    return gr, gk, gv, gw * inp["w32"], gu, gi


NAMES = ("gr", "gk", "gv", "glogw", "gu", "g_init")


def check(got, want, tol=TOL["bf16"], skip=()):
    for name, g, r in zip(NAMES, got, want):
        if name in skip or g is None:
            continue
        e = rel_err(host64(g), r)
        assert e < tol, f"{name}: {e:.3g}"


@pytest.mark.parametrize("B,T,H", [(1, 64, 1), (2, 100, 2), (1, 1, 3), (2, 257, 2), (1, 33, 1), (3, 130, 1)])
def test_matches_oracle(W, oracle, B, T, H):
    inp = draw(B, T, H, seed=B * 31 + T + H)
    rng = np.random.default_rng(T)
    init = rng.normal(size=(B, H, 64, 64)).astype(np.float32)
    gfin = rng.normal(size=(B, H, 64, 64)).astype(np.float32)
    got = run(W, inp, init_state=dev(init), g_final=dev(gfin))
    want = ref(oracle, inp, H, init_state=init, g_final=gfin)
    check(got, want)
    assert W.device_error(reset=True) == 0


def test_zero_initial_state_and_no_final_gradient(W, oracle):
    B, T, H = 2, 160, 2
    inp = draw(B, T, H, seed=3)
    got = run(W, inp)
    want = ref(oracle, inp, H)
    check(got, want)


def test_init_state_map_and_shared_state(W, oracle):
    B, T, H = 3, 70, 2
    inp = draw(B, T, H, seed=11)
    rng = np.random.default_rng(2)
    init = rng.normal(size=(2, H, 64, 64)).astype(np.float32)
    gfin = rng.normal(size=(B, H, 64, 64)).astype(np.float32)
    smap = np.array([1, 0, 1], np.int32)
    got = run(W, inp, init_state=dev(init), state_map=dev(smap), g_final=dev(gfin))
    want = ref(oracle, inp, H, init_state=init, state_map=smap, g_final=gfin)
    check(got, want)
    got1 = run(W, inp, init_state=dev(init[:1]))
    want1 = ref(oracle, inp, H, init_state=init[:1])
    check(got1, want1)
    assert W.device_error(reset=True) == 0


def test_no_decay_is_linear_attention(W, oracle):
    """w = 1 (d = -30): glogw = dL/dw exactly; G only accumulates r^T do."""
    B, T, H = 1, 192, 1
    inp = draw(B, T, H, seed=9, d_mean=-30.0, d_std=0.1)
    assert np.all(inp["w32"] == 1.0)
    check(run(W, inp), ref(oracle, inp, H))


@pytest.mark.parametrize("d_mean,d_std,seed", [(1.0, 1.5, 5), (3.0, 1.0, 6), (-0.5, 2.0, 7)])
def test_strong_decay(W, oracle, d_mean, d_std, seed):
    """Decays far below the trained range (some w round to 0 in bf16). glogw
    is formed as P_t - k_t (G_t v_t), a difference of terms of the size of
    k o (G v): its error is bounded against that size, not against glogw's own
    (which vanishes with w); the other gradients keep the plain bound."""
    B, T, H = 2, 300, 2
    inp = draw(B, T, H, seed=seed, d_mean=d_mean, d_std=d_std)
    rng = np.random.default_rng(seed)
    init = rng.normal(size=(B, H, 64, 64)).astype(np.float32)
    got = run(W, inp, init_state=dev(init))
    want = ref(oracle, inp, H, init_state=init)
    check(got, want, skip=("glogw",))
    kgv = inp["k32"].astype(np.float64) * want[1]  # k o gk: the scale of the cancelling terms
    floor = float(np.sqrt(np.mean(kgv ** 2)))
    assert rel_err_floor(host64(got[3]), want[3], floor=floor) < TOL["bf16"]
    assert W.device_error(reset=True) == 0


def test_empty_sequence(W):
    """T = 0: nothing flows through time, g_init = g_final and gu = 0."""
    B, H = 2, 2
    z = torch.zeros((B, 0, H * 64), dtype=torch.bfloat16, device="cuda")
    u = torch.zeros(H * 64, device="cuda")
    gfin = torch.randn(B, H, 64, 64, device="cuda")
    gr, gk, gv, glogw, gu, gi = W.wkv6_backward(z, z, z, z, u, z, g_final=gfin)
    torch.cuda.synchronize()
    assert torch.equal(gi, gfin)
    assert torch.count_nonzero(gu).item() == 0


def test_full_size_32_heads(W, oracle):
    """The bench shape (B=8, T=4096, H=32): every head runs on the GPU; 32
    (sample, head) pairs, four of every sample, are checked against the oracle
    run on their slices (side by side as the heads of one sample); gu, which
    sums every sample, against the oracle on all samples of one head."""
    from test_wkv6_forward_gpu import HEADS32, gather_heads
    rec = synth.WKV6_RECIPES["wkv6_fwd_bf16_c2048"]
    B, T, H = rec.B, rec.T, rec.H
    inp = draw(B, T, H, seed=0)
    got = run(W, inp)
    torch.cuda.synchronize()
    sub = gather_heads(inp, HEADS32, ("r32", "k32", "v32", "w32", "do32"))
    want = ref(oracle, sub, len(HEADS32))
    for m, (b, h) in enumerate(HEADS32):
        cols = slice(h * 64, (h + 1) * 64)
        mc = slice(m * 64, (m + 1) * 64)
        for name, g, r in zip(NAMES[:4], got[:4], want[:4]):
            e = rel_err(host64(g[b:b + 1, :, cols]), r[:, :, mc])
            assert e < TOL["bf16"], f"{name} (b={b}, h={h}): {e:.3g}"
    h = 5
    cols = slice(h * 64, (h + 1) * 64)
    sl = {n: inp[n][:, :, cols] for n in ("r32", "k32", "v32", "w32", "do32")}
    sl["u"] = inp["u"][cols]
    total = ref(oracle, sl, 1)[4]
    assert rel_err(host64(got[4])[cols], total) < TOL["bf16"]
    assert W.device_error(reset=True) == 0
