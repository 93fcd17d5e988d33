"""GPU parity of the time-shift mix (the prologue of RWKV_TimeMix.jit_func,
"代码连连看——RWKV", section RWKV_TimeMix) and its backward against the fp64
oracle.

Tolerances: the forward is one fused multiply-add per output in float32, so
float32 outputs agree to a few ulp (2e-6 relative to the output scale) and
bf16 outputs to their one final rounding (2^-9, bounded at 4e-3); gx adds
2·n_mix such products; the mix gradients are float32 sums over B·T tokens of
exactly stored inputs (1e-4 in both storage types)."""

import numpy as np
import pytest
import torch

from _dev import assert_no_device_error, dev, host64, need_gpu, rel_err
from rwkv_wkv_linear_mix_b200 import synth

pytestmark = pytest.mark.gpu

TOL_OUT = {"f32": 2e-6, "bf16": 4e-3}
TOL_GX = {"f32": 1e-5, "bf16": 4e-3}
TOL_GMIX = 1e-4


@pytest.fixture(scope="module")
def W():
    need_gpu()
    from rwkv_wkv_linear_mix_b200 import wkv
    wkv.device_error(reset=True)
    return wkv


def draw(B, T, C, n, dtype, seed):
    """x, g ~ N(0, 1) stored in `dtype`, x_prev likewise, mix ~ U(0, 1) in
    float32 (the page initialises time_mix_* in [0, 1])."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = {}
    out["x"], out["x32"] = synth._store(rng.standard_normal((B, T, C), dtype=np.float32), dtype)
    out["xp"], out["xp32"] = synth._store(rng.standard_normal((B, C), dtype=np.float32), dtype)
    out["g"], out["g32"] = synth._store(rng.standard_normal((n, B, T, C), dtype=np.float32), dtype)
    out["mix"] = rng.uniform(0, 1, size=(n, C)).astype(np.float32)
    return out


SHAPES = [(2, 64, 128), (3, 100, 72), (1, 1, 8), (2, 33, 40), (1, 257, 1032), (4, 500, 32), (2, 1000, 4104)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("n", [1, 2, 3])
@pytest.mark.parametrize("B,T,C", SHAPES)
def test_forward_and_backward_match_oracle(W, oracle, dtype, n, B, T, C):
    inp = draw(B, T, C, n, dtype, seed=B * 13 + T + C + n)
    with_prev = (B + T + n) % 2 == 0
    x, mix, g = dev(inp["x"]), dev(inp["mix"]), dev(inp["g"])
    xp = dev(inp["xp"]) if with_prev else None
    xp32 = inp["xp32"] if with_prev else None
    out = W.wkv4_time_shift_mix(x, mix, xp)
    want = oracle.time_shift_mix(inp["x32"], inp["mix"], x_prev=xp32)
    assert rel_err(host64(out), want) < TOL_OUT[dtype]
    gx, gmix, gxp = W.wkv4_time_shift_mix_backward(x, mix, g, xp, want_gx_prev=True)
    rgx, rgmix, rgxp = oracle.time_shift_mix_backward(inp["x32"], inp["mix"], inp["g32"],
                                                      x_prev=xp32 if with_prev else np.zeros((B, C)))
    assert rel_err(host64(gx), rgx) < TOL_GX[dtype], "gx"
    assert rel_err(host64(gmix), rgmix) < TOL_GMIX, "gmix"
    assert rel_err(host64(gxp), rgxp) < TOL_GX[dtype], "gx_prev"
    assert_no_device_error()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_pieces_with_x_prev_give_the_same_bits(W, dtype):
    """A sequence fed in two pieces, the second with the first's last token
    as x_prev, gives the one-call outputs bit for bit."""
    B, T, C, s = 3, 300, 264, 123
    inp = draw(B, T, C, 3, dtype, seed=5)
    x, mix = dev(inp["x"]), dev(inp["mix"])
    whole = W.wkv4_time_shift_mix(x, mix)
    a = W.wkv4_time_shift_mix(x[:, :s].contiguous(), mix)
    b = W.wkv4_time_shift_mix(x[:, s:].contiguous(), mix, x[:, s - 1].contiguous())
    assert torch.equal(torch.cat([a, b], dim=2), whole)


def test_ends_of_the_blend(W):
    """mix = 1 copies x; mix = 0 is the shifted input (torch's ZeroPad2d((0, 0,
    1, -1)), the page's time_shift), both exactly."""
    B, T, C = 2, 77, 96
    x = torch.randn(B, T, C, device="cuda")
    mix = torch.stack([torch.ones(C, device="cuda"), torch.zeros(C, device="cuda")])
    out = W.wkv4_time_shift_mix(x, mix)
    torch.cuda.synchronize()
    assert torch.equal(out[0], x)
    assert torch.equal(out[1].cpu(), torch.nn.ZeroPad2d((0, 0, 1, -1))(x.cpu()))


def test_full_size_sampled_channels(W, oracle):
    """B = 16, T = 4096, C = 4096 in bf16 with three blends (the bench shape):
    the whole problem runs on the GPU; 18 channels are checked against the
    oracle on their slices (channels are independent)."""
    B, T, C, n = 16, 4096, 4096, 3
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    x = torch.randn(B, T, C, device="cuda", generator=g).to(torch.bfloat16)
    gy = torch.randn(n, B, T, C, device="cuda", generator=g).to(torch.bfloat16)
    mix = torch.rand(n, C, device="cuda", generator=g)
    out = W.wkv4_time_shift_mix(x, mix)
    gx, gmix, _ = W.wkv4_time_shift_mix_backward(x, mix, gy)
    torch.cuda.synchronize()
    rng = np.random.default_rng(6)
    cs = np.unique(np.concatenate([rng.choice(C, size=16, replace=False), [0, C - 1]]))
    ci = torch.from_numpy(cs).cuda()
    x_s = host64(x[:, :, ci])
    mix_s = host64(mix[:, ci])
    assert rel_err(host64(out[:, :, :, ci]), oracle.time_shift_mix(x_s, mix_s)) < TOL_OUT["bf16"]
    rgx, rgmix, _ = oracle.time_shift_mix_backward(x_s, mix_s, host64(gy[:, :, :, ci]))
    assert rel_err(host64(gx[:, :, ci]), rgx) < TOL_GX["bf16"]
    assert rel_err(host64(gmix[:, ci]), rgmix) < TOL_GMIX
    assert_no_device_error()


def test_backward_is_deterministic(W):
    B, T, C = 4, 1000, 512
    inp = draw(B, T, C, 3, "f32", seed=7)
    x, mix, g = dev(inp["x"]), dev(inp["mix"]), dev(inp["g"])
    a = W.wkv4_time_shift_mix_backward(x, mix, g)
    b = W.wkv4_time_shift_mix_backward(x, mix, g)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_empty_sequence(W):
    x = torch.zeros(2, 0, 64, device="cuda")
    mix = torch.rand(3, 64, device="cuda")
    assert W.wkv4_time_shift_mix(x, mix).shape == (3, 2, 0, 64)
    g = torch.zeros(3, 2, 0, 64, device="cuda")
    gx, gmix, gxp = W.wkv4_time_shift_mix_backward(x, mix, g, want_gx_prev=True)
    torch.cuda.synchronize()
    assert torch.count_nonzero(gmix).item() == 0 and torch.count_nonzero(gxp).item() == 0
