"""Pins of the fp64 RWKV-7 oracle (generalized delta rule of the rwkv-ops
package page): closed forms of the delta rule, the decayed linear attention
it reduces to without its rank-one term, a hand-worked two-step case, the
state carry and linearity. Each pin is an evaluation independent of the
oracle's loop, so a dropped term, a swapped a/b, a missing exp on the log
decay or the output read before the update fails one of them."""

import numpy as np
import pytest

from _pins import rel_err


def unit_rows(rng, n, K):
    x = rng.normal(size=(n, K))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def test_delta_rule_stores_and_reads_back(oracle):
    """w = 0, a = -kappa, b = k = r = kappa (unit): S_t = (I - kappa kappa^T) S_{t-1}
    + kappa v^T, so kappa^T S_t = v_t and o_t = v_t exactly, whatever S_{t-1}."""
    rng = np.random.default_rng(1)
    B, T, H, K = 2, 9, 2, 5
    kap = unit_rows(rng, B * T * H, K).reshape(B, T, H * K)
    v = rng.normal(size=(B, T, H * K))
    zero = np.zeros_like(v)
    s0 = rng.normal(size=(B, H, K, K))
    o, _ = oracle.wkv7_forward(kap, zero, kap, v, -kap, kap, init_state=s0, head_size=K)
    assert rel_err(o, v) < 1e-12


def test_fixed_key_is_an_exponential_moving_average(oracle):
    """w = 0, one unit kappa for every token, a = -kappa, b = k = beta kappa,
    r = kappa: kappa^T S_t = (1 - beta) kappa^T S_{t-1} + beta v_t, so o_t is
    the EMA m_t = (1 - beta) m_{t-1} + beta v_t from m_{-1} = kappa^T S_{-1}."""
    rng = np.random.default_rng(2)
    T, K, beta = 12, 6, 0.3
    kap = unit_rows(rng, 1, K)[0]
    ktok = np.tile(kap, (1, T, 1))
    v = rng.normal(size=(1, T, K))
    s0 = rng.normal(size=(1, 1, K, K))
    o, _ = oracle.wkv7_forward(ktok, np.zeros_like(v), beta * ktok, v, -ktok, beta * ktok, init_state=s0,
                               head_size=K)
    m = kap @ s0[0, 0]
    want = np.empty((1, T, K))
    for t in range(T):
        m = (1 - beta) * m + beta * v[0, t]
        want[0, t] = m
    assert rel_err(o, want) < 1e-12


def decayed_linear_attention(r, w, k, v, s0, K):
    """o_t[i] = sum_j r_t[j] (prod_{tau<=t} e^{w_tau[j]} S0[j][i]
    + sum_{s<=t} prod_{s<tau<=t} e^{w_tau[j]} k_s[j] v_s[i]), by direct sums."""
    B, T, HK = r.shape
    H = HK // K
    o = np.zeros((B, T, HK))
    for b in range(B):
        for h in range(H):
            sl = slice(h * K, (h + 1) * K)
            cw = np.cumsum(w[b, :, sl], axis=0)  # sum of log decays up to t
            for t in range(T):
                acc = r[b, t, sl] * np.exp(cw[t]) @ s0[b, h]
                for s in range(t + 1):
                    fac = np.exp(cw[t] - cw[s])
                    acc = acc + (r[b, t, sl] * fac * k[b, s, sl]).sum() * v[b, s, sl]
                o[b, t, sl] = acc
    return o


@pytest.mark.parametrize("which", ["both_zero", "b_zero", "a_zero"])
def test_without_the_rank_one_term(oracle, which):
    """b a^T = 0 (a or b zero): decayed linear attention, read after the update."""
    rng = np.random.default_rng(3)
    B, T, H, K = 2, 7, 2, 4
    r, k, v = (rng.normal(size=(B, T, H * K)) for _ in range(3))
    w = -np.exp(rng.normal(-1.0, 0.5, size=(B, T, H * K)))
    a, b = rng.normal(size=(B, T, H * K)), rng.normal(size=(B, T, H * K))
    if which in ("both_zero", "b_zero"):
        b = np.zeros_like(b)
    if which in ("both_zero", "a_zero"):
        a = np.zeros_like(a)
    s0 = rng.normal(size=(B, H, K, K))
    o, _ = oracle.wkv7_forward(r, w, k, v, a, b, init_state=s0, head_size=K)
    assert rel_err(o, decayed_linear_attention(r, w, k, v, s0, K)) < 1e-12


def test_hand_worked_two_steps(oracle):
    """K = 3, w = 0, S_{-1} = 0, a = -e0, b = e1, k = e0 at both steps.
    Step 0: sa = 0, S_0 = e0 v0^T; reading r = e0 gives v0.
    Step 1: sa = -e0^T S_0 = -v0^T, S_1 = e0 v0^T - e1 v0^T + e0 v1^T;
    reading r = e1 gives -v0 (a swapped a/b would give 0)."""
    e0, e1 = np.array([1.0, 0, 0]), np.array([0, 1.0, 0])
    v = np.array([[[2.0, -1.0, 0.5], [0.25, 3.0, -2.0]]])
    r = np.stack([e0, e1])[None]
    k = np.stack([e0, e0])[None]
    a = -k
    b = np.stack([e1, e1])[None]
    o, fs = oracle.wkv7_forward(r, np.zeros((1, 2, 3)), k, v, a, b, head_size=3)
    np.testing.assert_allclose(o[0, 0], v[0, 0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(o[0, 1], -v[0, 0], rtol=0, atol=1e-15)
    want = np.outer(e0, v[0, 0]) - np.outer(e1, v[0, 0]) + np.outer(e0, v[0, 1])
    np.testing.assert_allclose(fs[0, 0], want, rtol=0, atol=1e-15)


def test_state_carry_across_a_split(oracle):
    rng = np.random.default_rng(4)
    B, T, H, K = 2, 11, 1, 4
    r, k, v = (rng.normal(size=(B, T, H * K)) for _ in range(3))
    w = -np.exp(rng.normal(-1.0, 0.5, size=(B, T, H * K)))
    kap = unit_rows(rng, B * T * H, K).reshape(B, T, H * K)
    a, b = -kap, kap * rng.uniform(0, 1, size=kap.shape)
    o, fs = oracle.wkv7_forward(r, w, k, v, a, b, head_size=K)
    o1, fs1 = oracle.wkv7_forward(r[:, :5], w[:, :5], k[:, :5], v[:, :5], a[:, :5], b[:, :5], head_size=K)
    o2, fs2 = oracle.wkv7_forward(r[:, 5:], w[:, 5:], k[:, 5:], v[:, 5:], a[:, 5:], b[:, 5:], init_state=fs1,
                                  head_size=K)
    assert rel_err(np.concatenate([o1, o2], axis=1), o) < 1e-13
    assert rel_err(fs2, fs) < 1e-13


def test_linear_in_values_and_initial_state(oracle):
    """For fixed r, w, k, a, b the map (v, S_{-1}) -> (o, S_T) is linear."""
    rng = np.random.default_rng(5)
    B, T, H, K = 1, 8, 2, 4
    r, k = (rng.normal(size=(B, T, H * K)) for _ in range(2))
    w = -np.exp(rng.normal(-1.0, 0.5, size=(B, T, H * K)))
    kap = unit_rows(rng, B * T * H, K).reshape(B, T, H * K)
    a, b = -kap, 0.5 * kap
    v1, v2 = rng.normal(size=(B, T, H * K)), rng.normal(size=(B, T, H * K))
    s1, s2 = rng.normal(size=(B, H, K, K)), rng.normal(size=(B, H, K, K))
    oa, fa = oracle.wkv7_forward(r, w, k, v1, a, b, init_state=s1, head_size=K)
    ob, fb = oracle.wkv7_forward(r, w, k, v2, a, b, init_state=s2, head_size=K)
    oc, fc = oracle.wkv7_forward(r, w, k, 2 * v1 - 3 * v2, a, b, init_state=2 * s1 - 3 * s2, head_size=K)
    assert rel_err(oc, 2 * oa - 3 * ob) < 1e-12
    assert rel_err(fc, 2 * fa - 3 * fb) < 1e-12


# ---------------------------------------------------------------------------
# backward (the page's generalized_delta_rule carries gradients)
# ---------------------------------------------------------------------------

def _wkv7_loss(oracle, args, dout, init, gfin, K):
    o, fs = oracle.wkv7_forward(*args, init_state=init, head_size=K)
    return float(np.sum(dout * o) + (0.0 if gfin is None else np.sum(gfin * fs)))


def _wkv7_draw(seed, B=1, T=5, H=2, K=3):
    rng = np.random.default_rng(seed)
    shape = (B, T, H * K)
    r, k, v = (rng.normal(size=shape) for _ in range(3))
    w = -np.exp(rng.normal(-1.0, 0.5, size=shape))
    kap = unit_rows(rng, B * T * H, K).reshape(shape)
    a, b = -kap, kap * rng.uniform(0, 1, size=shape)
    dout = rng.normal(size=shape)
    init = rng.normal(size=(B, H, K, K))
    gfin = rng.normal(size=(B, H, K, K))
    return [r, w, k, v, a, b], dout, init, gfin


@pytest.mark.parametrize("with_state", [False, True])
def test_backward_matches_finite_differences(oracle, with_state):
    """Central differences of L = sum(dout * o) (+ sum(g_final * S_final) and
    an initial state) in every entry of r, w, k, v, a, b and the initial
    state; the loss is a polynomial of low degree in each entry, so h = 1e-5
    leaves only rounding."""
    K = 3
    args, dout, init, gfin = _wkv7_draw(5 + with_state, K=K)
    if not with_state:
        init = gfin = None
    got = oracle.wkv7_backward(*args, dout, init_state=init, g_final=gfin, head_size=K)
    h = 1e-5
    for n in range(6):
        num = np.zeros_like(args[n])
        for idx in np.ndindex(args[n].shape):
            hi = [x.copy() for x in args]
            lo = [x.copy() for x in args]
            hi[n][idx] += h
            lo[n][idx] -= h
            num[idx] = (_wkv7_loss(oracle, hi, dout, init, gfin, K) - _wkv7_loss(oracle, lo, dout, init, gfin, K)) / (2 * h)
        assert rel_err(got[n], num) < 1e-7, "rwkabv"[n]
    s0 = init if init is not None else np.zeros((1, 2, K, K))
    num = np.zeros_like(s0)
    for idx in np.ndindex(s0.shape):
        hi, lo = s0.copy(), s0.copy()
        hi[idx] += h
        lo[idx] -= h
        num[idx] = (_wkv7_loss(oracle, args, dout, hi, gfin, K) - _wkv7_loss(oracle, args, dout, lo, gfin, K)) / (2 * h)
    assert rel_err(got[6], num) < 1e-7


def test_backward_homogeneity(oracle):
    """o is linear in r, and jointly linear in (v, S_init) (the state
    transition does not depend on them): Euler's identity gives
    sum r dr = L and sum v dv + sum S_init d_init = L for L = sum(dout * o)."""
    K = 4
    args, dout, init, _ = _wkv7_draw(9, T=7, K=K)
    L = _wkv7_loss(oracle, args, dout, init, None, K)
    dr, dw, dk, dv, da, db, di = oracle.wkv7_backward(*args, dout, init_state=init, head_size=K)
    assert abs(np.sum(args[0] * dr) - L) < 1e-10 * max(1.0, abs(L))
    assert abs(np.sum(args[3] * dv) + np.sum(init * di) - L) < 1e-10 * max(1.0, abs(L))
