"""Pins for the fp64 RWKV-4 oracle (CPU only).

Each test checks the oracle against something other than itself: a direct
O(T^2) evaluation of the defining sums, hand-worked values, closed forms
(T = 1, constant v, the no-decay softmax limit, the infinite-decay limit),
invariants (key shift, linearity, convexity, gradient sum rule) and central
finite differences. Definition: the RWKV-4 WKV operator that RWKV_TimeMix
calls as RUN_CUDA(B, T, C, time_decay, time_first, k, v) ("代码连连看——RWKV",
section RWKV_TimeMix).
"""

import json
import os

import numpy as np
import pytest

from _pins import rel_err as _rel, wkv4_direct_sum as _direct_sum, wkv4_fd_grads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(rng, B, T, C, td=(-6.0, 1.0), ur=(-1.0, 1.0), kstd=1.0):
    w = np.exp(rng.uniform(*td, size=C))
    u = rng.uniform(*ur, size=C)
    k = rng.normal(0.0, kstd, size=(B, T, C))
    v = rng.normal(size=(B, T, C))
    return w, u, k, v


def test_direct_sum_random(oracle):
    rng = np.random.default_rng(1)
    for (B, T, C, kstd) in [(1, 1, 3, 1.0), (2, 17, 5, 1.0), (1, 64, 8, 2.0), (2, 40, 4, 3.0)]:
        w, u, k, v = _rand_case(rng, B, T, C, kstd=kstd)
        assert _rel(oracle.wkv4_forward(w, u, k, v), _direct_sum(w, u, k, v)) < 1e-12


def test_direct_sum_model_init(oracle):
    # decay/bonus values of the fancy init in RWKV_TimeMix.__init__:
    # time_decay = -5 + 8 (h/(C-1))^(0.7 + 1.3 ratio), time_first = ln 0.3 + zigzag/2
    C, T = 8, 48
    ratio = 0.5
    h = np.arange(C)
    td = -5 + 8 * (h / (C - 1)) ** (0.7 + 1.3 * ratio)
    u = np.log(0.3) + 0.5 * (((h + 1) % 3) - 1)
    rng = np.random.default_rng(2)
    k = rng.normal(size=(1, T, C))
    v = rng.normal(size=(1, T, C))
    w = np.exp(td)
    assert _rel(oracle.wkv4_forward(w, u, k, v), _direct_sum(w, u, k, v)) < 1e-12


def test_hand_worked_golden(oracle):
    g = json.load(open(os.path.join(GOLDEN, "wkv4_hand_worked.json")))
    sh = lambda a: np.asarray(a, float).reshape(1, -1, 1)
    w, u = np.asarray(g["w"]), np.asarray(g["u"])
    k, v, gy = sh(g["k"]), sh(g["v"]), sh(g["gy"])
    y = oracle.wkv4_forward(w, u, k, v)
    np.testing.assert_allclose(y.ravel(), g["y"], rtol=1e-14, atol=1e-14)
    gk, gv, gw, gu = oracle.wkv4_backward(w, u, k, v, gy)
    np.testing.assert_allclose(gv.ravel(), g["gv"], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(gk.ravel(), g["gk"], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(gu, g["gu"], rtol=1e-13)
    np.testing.assert_allclose(gw, g["gw"], rtol=1e-13)


def test_single_token_is_v(oracle):
    rng = np.random.default_rng(3)
    w, u, k, v = _rand_case(rng, 3, 1, 7, kstd=5.0)
    # y_0 = e^{u+k_0} v_0 / e^{u+k_0}: exact up to one rounding of the product and quotient
    np.testing.assert_allclose(oracle.wkv4_forward(w, u, k, v), v, rtol=4e-16, atol=0)


def test_constant_v(oracle):
    rng = np.random.default_rng(4)
    w, u, k, _ = _rand_case(rng, 2, 50, 6, kstd=2.0)
    v = np.broadcast_to(rng.normal(size=(1, 1, 6)), k.shape).copy()
    y = oracle.wkv4_forward(w, u, k, v)
    np.testing.assert_allclose(y, v, rtol=1e-13)
    gy = rng.normal(size=k.shape)
    gk, gv, gw, gu = oracle.wkv4_backward(w, u, k, v, gy)
    assert np.max(np.abs(gk)) < 1e-12
    assert np.max(np.abs(gu)) < 1e-11
    assert np.max(np.abs(gw)) < 1e-10


def test_gradient_sum_rule(oracle):
    # y_t is a convex combination of v_0..v_t with weights independent of v,
    # so sum_t gv_t = sum_t gy_t on every lane.
    rng = np.random.default_rng(5)
    w, u, k, v = _rand_case(rng, 2, 33, 5, kstd=2.0)
    gy = rng.normal(size=k.shape)
    _, gv, _, _ = oracle.wkv4_backward(w, u, k, v, gy)
    np.testing.assert_allclose(gv.sum(axis=1), gy.sum(axis=1), rtol=1e-11, atol=1e-11)


def test_large_bonus_limit(oracle):
    rng = np.random.default_rng(6)
    w, _, k, v = _rand_case(rng, 2, 30, 4)
    u = np.full(4, 60.0)
    np.testing.assert_allclose(oracle.wkv4_forward(w, u, k, v), v, rtol=0, atol=1e-15)


def test_infinite_decay_two_token_softmax(oracle):
    # time_decay = 6 gives w = e^6 ~ 403: only the previous token survives the decay.
    rng = np.random.default_rng(7)
    C, T = 4, 25
    w = np.full(C, np.exp(6.0))
    u = rng.uniform(-1, 1, size=C)
    k = rng.normal(size=(1, T, C))
    v = rng.normal(size=(1, T, C))
    y = oracle.wkv4_forward(w, u, k, v)
    ref = np.empty_like(y)
    ref[:, 0] = v[:, 0]
    for t in range(1, T):
        e0 = np.exp(k[:, t - 1])
        e1 = np.exp(u + k[:, t])
        ref[:, t] = (e0 * v[:, t - 1] + e1 * v[:, t]) / (e0 + e1)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_no_decay_is_causal_softmax_attention(oracle):
    # time_decay = -30 (w ~ 1e-13) and u = 0: every past token and the current
    # one get weight e^{k_i}, i.e. y_t = softmax(k_0..k_t) . v_0..v_t.
    rng = np.random.default_rng(8)
    C, T = 3, 40
    w = np.full(C, np.exp(-30.0))
    u = np.zeros(C)
    k = rng.normal(0, 2, size=(2, T, C))
    v = rng.normal(size=(2, T, C))
    y = oracle.wkv4_forward(w, u, k, v)
    ref = np.empty_like(y)
    for t in range(T):
        kk = k[:, : t + 1]
        p = np.exp(kk - kk.max(axis=1, keepdims=True))
        ref[:, t] = (p * v[:, : t + 1]).sum(axis=1) / p.sum(axis=1)
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-10)


def test_key_shift_invariance(oracle):
    rng = np.random.default_rng(9)
    w, u, k, v = _rand_case(rng, 2, 45, 6, kstd=2.0)
    gy = rng.normal(size=k.shape)
    y0 = oracle.wkv4_forward(w, u, k, v)
    y1 = oracle.wkv4_forward(w, u, k + 1000.0, v)
    np.testing.assert_allclose(y1, y0, rtol=1e-9, atol=1e-9)
    g0 = oracle.wkv4_backward(w, u, k, v, gy)
    g1 = oracle.wkv4_backward(w, u, k + 1000.0, v, gy)
    for a, b in zip(g0, g1):
        assert _rel(a, b) < 1e-8


def test_linear_in_v_and_convex(oracle):
    rng = np.random.default_rng(10)
    w, u, k, v1 = _rand_case(rng, 2, 30, 5, kstd=2.0)
    v2 = rng.normal(size=v1.shape)
    y1 = oracle.wkv4_forward(w, u, k, v1)
    y2 = oracle.wkv4_forward(w, u, k, v2)
    y12 = oracle.wkv4_forward(w, u, k, 2.5 * v1 - 0.75 * v2)
    np.testing.assert_allclose(y12, 2.5 * y1 - 0.75 * y2, rtol=1e-11, atol=1e-11)
    lo = np.minimum.accumulate(v1, axis=1)
    hi = np.maximum.accumulate(v1, axis=1)
    assert np.all(y1 >= lo - 1e-12) and np.all(y1 <= hi + 1e-12)


@pytest.mark.parametrize("seed,T,C,kstd", [(11, 9, 3, 1.0), (12, 16, 4, 2.0), (13, 5, 2, 0.5)])
def test_finite_differences(oracle, seed, T, C, kstd):
    rng = np.random.default_rng(seed)
    w, u, k, v = _rand_case(rng, 1, T, C, td=(-3.0, 1.0), kstd=kstd)
    gy = rng.normal(size=k.shape)
    gk, gv, gw, gu, gwr = oracle.wkv4_backward(w, u, k, v, gy, return_reverse_gw=True)
    ngk, ngv, ngw, ngu = wkv4_fd_grads(oracle.wkv4_forward, w, u, k, v, gy)
    assert _rel(gk, ngk) < 1e-6
    assert _rel(gv, ngv) < 1e-6
    assert _rel(gw, ngw) < 1e-6
    assert _rel(gu, ngu) < 1e-6
    # the two independent derivations of gw agree
    np.testing.assert_allclose(gwr, gw, rtol=1e-10, atol=1e-12)


def test_gw_forms_agree_long(oracle):
    rng = np.random.default_rng(14)
    w, u, k, v = _rand_case(rng, 2, 300, 6, kstd=2.0)
    gy = rng.normal(size=k.shape)
    _, _, gw, _, gwr = oracle.wkv4_backward(w, u, k, v, gy, return_reverse_gw=True)
    assert _rel(gwr, gw) < 1e-9


def test_final_state(oracle):
    # a_T, b_T returned as (a_end, b_end) * e^{kmax}: compare with direct sums.
    rng = np.random.default_rng(15)
    w, u, k, v = _rand_case(rng, 2, 20, 3)
    _, st = oracle.wkv4_forward(w, u, k, v, return_state=True)
    T = k.shape[1]
    for b in range(2):
        for c in range(3):
            i = np.arange(T)
            wt = np.exp(-(T - 1 - i) * w[c] + k[b, i, c])
            a = (wt * v[b, i, c]).sum()
            bb = wt.sum()
            sc = np.exp(st["kmax"][b, c])
            np.testing.assert_allclose(st["a_end"][b, c] * sc, a, rtol=1e-12)
            np.testing.assert_allclose(st["b_end"][b, c] * sc, bb, rtol=1e-12)


def test_gated_backward_matches_finite_differences(oracle):
    """sigmoid(r) * WKV (the gate of RWKV_TimeMix.forward): every gradient of
    L = sum(g * sigmoid(r) * y), r included, against central differences."""
    rng = np.random.default_rng(41)
    B, T, C = 1, 6, 3
    w = np.exp(rng.uniform(-3, 1, size=C))
    u = rng.uniform(-1, 1, size=C)
    k, v, r, g = (rng.normal(size=(B, T, C)) for _ in range(4))
    gk, gv, gr, gw, gu = oracle.wkv4_backward_gated(w, u, k, v, r, g)

    def loss(w_, u_, k_, v_, r_):
        return float((g * oracle.wkv4_forward_gated(w_, u_, k_, v_, r_)).sum())

    def fd(args, i, idx):
        a = [np.array(x, dtype=np.float64) for x in args]
        x0 = a[i][idx]
        hh = 1e-5 * max(1.0, abs(x0))
        a[i][idx] = x0 + hh
        lp = loss(*a)
        a[i][idx] = x0 - hh
        lm = loss(*a)
        return (lp - lm) / (2 * hh)

    args = (w, u, k, v, r)
    for name, got, i in (("gk", gk, 2), ("gv", gv, 3), ("gr", gr, 4)):
        num = np.array([fd(args, i, idx) for idx in np.ndindex(*k.shape)]).reshape(k.shape)
        assert _rel(got, num) < 1e-6, name
    assert _rel(gw, np.array([fd(args, 0, (c,)) for c in range(C)])) < 1e-6
    assert _rel(gu, np.array([fd(args, 1, (c,)) for c in range(C)])) < 1e-6


def test_gate_limits(oracle):
    """r -> +inf leaves the WKV unchanged; r = 0 halves it."""
    rng = np.random.default_rng(42)
    B, T, C = 2, 9, 4
    w = np.exp(rng.uniform(-3, 1, size=C))
    u = rng.uniform(-1, 1, size=C)
    k, v = rng.normal(size=(B, T, C)), rng.normal(size=(B, T, C))
    y = oracle.wkv4_forward(w, u, k, v)
    assert _rel(oracle.wkv4_forward_gated(w, u, k, v, np.full(k.shape, 60.0)), y) < 1e-15
    assert _rel(oracle.wkv4_forward_gated(w, u, k, v, np.zeros(k.shape)), 0.5 * y) < 1e-15
