"""Pins of the fp64 time-shift mix oracle (the prologue of
RWKV_TimeMix.jit_func, "代码连连看——RWKV", section RWKV_TimeMix): a
hand-worked case, the two ends of the blend (mix = 1 is the token itself,
mix = 0 is the page's own ZeroPad2d((0, 0, 1, -1)) shift, run through
torch's module), the chunking identity that x_prev exists for, closed forms
of the backward for g = 1, and central differences of the loss. A shift in
the wrong direction, swapped blend weights, a gradient scattered to the
wrong row or a flipped sign in the mix gradient fails one of them."""

import numpy as np
import pytest
import torch

from _pins import rel_err


def test_hand_worked(oracle):
    """x = [[1, 2], [3, 4], [5, 6]] (T = 3, C = 2), mix = [0.25, 1]:
    channel 0 blends a quarter of the token with three quarters of the one
    before (zero before t = 0): 0.25, 0.25*3 + 0.75*1 = 1.5, 0.25*5 + 0.75*3
    = 3.5; channel 1 (mix 1) is the token itself. With x_prev = [8, 9] the
    first row becomes 0.25*1 + 0.75*8 = 6.25 and 2."""
    x = np.array([[[1.0, 2.0], [3.0, 4.0], [5.0, 6.0]]])
    mix = np.array([[0.25, 1.0]])
    out = oracle.time_shift_mix(x, mix)
    assert np.array_equal(out[0, 0], [[0.25, 2.0], [1.5, 4.0], [3.5, 6.0]])
    out = oracle.time_shift_mix(x, mix, x_prev=np.array([[8.0, 9.0]]))
    assert np.array_equal(out[0, 0, 0], [6.25, 2.0])


def test_ends_of_the_blend(oracle):
    """mix = 1 returns x; mix = 0 returns ZeroPad2d((0, 0, 1, -1))(x), the
    page's time_shift, evaluated by torch on the CPU."""
    rng = np.random.default_rng(1)
    B, T, C = 3, 7, 5
    x = rng.normal(size=(B, T, C))
    out = oracle.time_shift_mix(x, np.stack([np.ones(C), np.zeros(C)]))
    assert np.array_equal(out[0], x)
    shifted = torch.nn.ZeroPad2d((0, 0, 1, -1))(torch.from_numpy(x)).numpy()
    assert np.array_equal(out[1], shifted)


def test_pieces_with_x_prev_match_one_call(oracle):
    """Cutting T at s and passing the last token of the first piece as x_prev
    of the second gives the one-call result exactly."""
    rng = np.random.default_rng(2)
    B, T, C, s = 2, 11, 4, 6
    x = rng.normal(size=(B, T, C))
    mix = rng.uniform(0, 1, size=(3, C))
    whole = oracle.time_shift_mix(x, mix)
    a = oracle.time_shift_mix(x[:, :s], mix)
    b = oracle.time_shift_mix(x[:, s:], mix, x_prev=x[:, s - 1])
    assert np.array_equal(np.concatenate([a, b], axis=2), whole)


def test_backward_closed_form_for_unit_gradient(oracle):
    """g = 1 everywhere: every output row weighs its token by mix and the one
    before by 1 - mix, so gx_t = n_mix for t < T-1 (each row is read twice),
    gx_{T-1} = sum_m mix_m, gx_prev = sum_m (1 - mix_m), and
    gmix_m = sum_{b,t} (x_t - x_{t-1}) = sum_b (x_{T-1} - x_prev) (telescoping)."""
    rng = np.random.default_rng(3)
    B, T, C = 2, 9, 3
    x = rng.normal(size=(B, T, C))
    xp = rng.normal(size=(B, C))
    mix = rng.uniform(0, 1, size=(3, C))
    gx, gmix, gxp = oracle.time_shift_mix_backward(x, mix, np.ones((3, B, T, C)), x_prev=xp)
    assert np.allclose(gx[:, :-1], 3.0, rtol=0, atol=1e-15)
    assert np.allclose(gx[:, -1], mix.sum(0), rtol=0, atol=1e-15)
    assert np.allclose(gxp, (1 - mix).sum(0), rtol=0, atol=1e-15)
    tele = (x[:, -1] - xp).sum(0)
    assert rel_err(gmix, np.tile(tele, (3, 1))) < 1e-13


@pytest.mark.parametrize("with_prev", [False, True])
def test_backward_matches_finite_differences(oracle, with_prev):
    """Central differences of L = sum(g * out) in every x, mix and x_prev
    entry (L is bilinear, so the difference is exact up to rounding)."""
    rng = np.random.default_rng(4 + with_prev)
    B, T, C, n = 2, 5, 3, 3
    x = rng.normal(size=(B, T, C))
    mix = rng.uniform(0, 1, size=(n, C))
    xp = rng.normal(size=(B, C)) if with_prev else None
    g = rng.normal(size=(n, B, T, C))
    gx, gmix, gxp = oracle.time_shift_mix_backward(x, mix, g, x_prev=xp)

    def L(x_, mix_, xp_):
        return float(np.sum(g * oracle.time_shift_mix(x_, mix_, x_prev=xp_)))

    h = 1e-5

    def fd(arr, which):
        out = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            args = [x, mix, xp]
            hi, lo = arr.copy(), arr.copy()
            hi[idx] += h
            lo[idx] -= h
            args[which] = hi
            f1 = L(*args)
            args[which] = lo
            f0 = L(*args)
            out[idx] = (f1 - f0) / (2 * h)
        return out

    assert rel_err(gx, fd(x, 0)) < 1e-8
    assert rel_err(gmix, fd(mix, 1)) < 1e-8
    if with_prev:
        assert rel_err(gxp, fd(xp, 2)) < 1e-8
    else:
        assert gxp is None


def test_empty_and_single_token(oracle):
    x = np.zeros((2, 0, 4))
    assert oracle.time_shift_mix(x, np.ones((3, 4))).shape == (3, 2, 0, 4)
    x1 = np.arange(8.0).reshape(2, 1, 4)
    mix = np.full((1, 4), 0.5)
    assert np.array_equal(oracle.time_shift_mix(x1, mix)[0], 0.5 * x1)
