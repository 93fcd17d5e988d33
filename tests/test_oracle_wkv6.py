"""Pins for the fp64 RWKV-6 head-state oracle (CPU only).

Definition: RWKV6_OP of the rwkv-ops package page (section "rwkv6op 使用方法",
call and argument tables): o_t = r_t (S_{t-1} + diag(u) k_t^T v_t),
S_t = diag(w_t) S_{t-1} + k_t^T v_t, optional init_state / state_map.
The oracle is checked against the unrolled direct sum, a chunked evaluation,
hand-worked values and closed-form special cases.
"""

import json
import os

import numpy as np
import pytest

from _pins import rel_err, wkv6_chunked, wkv6_direct_sum

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _case(rng, B, T, H, K, wlo=0.3, whi=1.0):
    r = rng.normal(size=(B, T, H * K))
    k = rng.normal(size=(B, T, H * K))
    v = rng.normal(size=(B, T, H * K))
    w = rng.uniform(wlo, whi, size=(B, T, H * K))
    u = rng.uniform(-1, 1, size=(H, K))
    return r, k, v, w, u


@pytest.mark.parametrize("B,T,H,K", [(1, 12, 1, 4), (2, 9, 2, 3), (1, 20, 1, 8)])
def test_direct_sum(oracle, B, T, H, K):
    rng = np.random.default_rng(B * 100 + T)
    r, k, v, w, u = _case(rng, B, T, H, K)
    o, _ = oracle.wkv6_forward(r, k, v, w, u)
    assert rel_err(o, wkv6_direct_sum(r, k, v, w, u, K)) < 1e-12


def test_direct_sum_head64(oracle):
    rng = np.random.default_rng(21)
    r, k, v, w, u = _case(rng, 1, 6, 1, 64)
    o, _ = oracle.wkv6_forward(r, k, v, w, u)
    assert rel_err(o, wkv6_direct_sum(r, k, v, w, u, 64)) < 1e-12


def test_hand_worked_golden(oracle):
    g = json.load(open(os.path.join(GOLDEN, "wkv6_hand_worked.json")))
    f = lambda a: np.asarray(a, float)[None]
    o, fs = oracle.wkv6_forward(f(g["r"]), f(g["k"]), f(g["v"]), f(g["w"]), np.asarray(g["u"], float))
    np.testing.assert_allclose(o[0], g["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(fs[0, 0], g["final_state"], rtol=0, atol=1e-14)


def test_no_decay_linear_attention(oracle):
    # w = 1, u = 0: o_t = r_t sum_{s<t} k_s^T v_s (strictly causal linear attention)
    rng = np.random.default_rng(22)
    B, T, H, K = 2, 15, 2, 5
    r, k, v, _, _ = _case(rng, B, T, H, K)
    w = np.ones_like(r)
    u = np.zeros((H, K))
    o, _ = oracle.wkv6_forward(r, k, v, w, u)
    ref = np.zeros_like(o)
    for b in range(B):
        for h in range(H):
            sl = slice(h * K, (h + 1) * K)
            S = np.zeros((K, K))
            for t in range(T):
                ref[b, t, sl] = r[b, t, sl] @ S
                S = S + np.outer(k[b, t, sl], v[b, t, sl])
    assert rel_err(o, ref) < 1e-12


def test_zero_decay_keeps_last_token(oracle):
    # w = 0: S_{t-1} = k_{t-1}^T v_{t-1}
    rng = np.random.default_rng(23)
    B, T, H, K = 1, 10, 2, 4
    r, k, v, _, u = _case(rng, B, T, H, K)
    w = np.zeros_like(r)
    o, fs = oracle.wkv6_forward(r, k, v, w, u)
    for h in range(H):
        sl = slice(h * K, (h + 1) * K)
        for t in range(T):
            rk_prev = (r[0, t, sl] @ k[0, t - 1, sl]) if t > 0 else 0.0
            rk_cur = (r[0, t, sl] * u[h] * k[0, t, sl]).sum()
            np.testing.assert_allclose(o[0, t, sl], rk_prev * (v[0, t - 1, sl] if t > 0 else 0) + rk_cur * v[0, t, sl],
                                       rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(fs[0, h], np.outer(k[0, -1, sl], v[0, -1, sl]), rtol=1e-13)


@pytest.mark.parametrize("L", [4, 16])
def test_chunked_form_agrees(oracle, L):
    rng = np.random.default_rng(24 + L)
    B, T, H, K = 2, 37, 2, 8
    r, k, v, w, u = _case(rng, B, T, H, K, wlo=0.05, whi=0.99)
    o, fs = oracle.wkv6_forward(r, k, v, w, u)
    oc, fsc = wkv6_chunked(r, k, v, w, u, K, L)
    assert rel_err(o, oc) < 1e-12
    assert rel_err(fs, fsc) < 1e-12


def test_state_carry_and_mapping(oracle):
    rng = np.random.default_rng(25)
    B, T, H, K = 3, 16, 2, 4
    r, k, v, w, u = _case(rng, B, T, H, K)
    o, fs = oracle.wkv6_forward(r, k, v, w, u)
    # splitting the sequence and feeding the state back reproduces the whole run
    o1, fs1 = oracle.wkv6_forward(r[:, :7], k[:, :7], v[:, :7], w[:, :7], u)
    o2, fs2 = oracle.wkv6_forward(r[:, 7:], k[:, 7:], v[:, 7:], w[:, 7:], u, init_state=fs1)
    assert rel_err(np.concatenate([o1, o2], axis=1), o) < 1e-13
    assert rel_err(fs2, fs) < 1e-13
    # state_map picks per-sample initial states; n_state = 1 is shared
    init = rng.normal(size=(2, H, K, K))
    smap = np.array([1, 0, 1], dtype=np.int32)
    om, _ = oracle.wkv6_forward(r, k, v, w, u, init_state=init, state_map=smap)
    for b in range(B):
        ob, _ = oracle.wkv6_forward(r[b:b + 1], k[b:b + 1], v[b:b + 1], w[b:b + 1], u,
                                    init_state=init[smap[b]:smap[b] + 1])
        assert rel_err(om[b:b + 1], ob) < 1e-14
    os1, _ = oracle.wkv6_forward(r, k, v, w, u, init_state=init[:1])
    osm, _ = oracle.wkv6_forward(r, k, v, w, u, init_state=init[:1], state_map=np.zeros(B, np.int32))
    assert np.array_equal(os1, osm)
    # initial state enters the output as r_t diag(prod w) S_0
    oz, _ = oracle.wkv6_forward(r, k, v, w, u, init_state=np.zeros((1, H, K, K)))
    assert np.array_equal(oz, o)


# --------------------------------------------------------------------------
# backward (RWKV6_OP is trainable: the package page lists its CUDA backward)
# --------------------------------------------------------------------------

def _bwd_case(rng, B, T, H, K):
    r, k, v, w, u = _case(rng, B, T, H, K, wlo=0.2)
    dout = rng.normal(size=r.shape)
    s0 = rng.normal(size=(B, H, K, K))
    gf = rng.normal(size=(B, H, K, K))
    return r, k, v, w, u, dout, s0, gf


@pytest.mark.parametrize("B,T,H,K", [(1, 5, 1, 3), (2, 4, 2, 2), (1, 7, 1, 4)])
def test_backward_finite_differences(oracle, B, T, H, K):
    """Every gradient (r, k, v, w, u and the initial state) against central
    differences of L = sum(o * dout) + sum(final_state * g_final)."""
    from _pins import wkv6_fd_grads
    rng = np.random.default_rng(300 + B * 10 + T)
    r, k, v, w, u, dout, s0, gf = _bwd_case(rng, B, T, H, K)
    got = oracle.wkv6_backward(r, k, v, w, u, dout, init_state=s0, g_final=gf)
    num = wkv6_fd_grads(oracle.wkv6_forward, r, k, v, w, u, dout, init_state=s0, g_final=gf)
    for name, g, n in zip(("gr", "gk", "gv", "gw", "gu", "g_init"), got, num):
        assert rel_err(g, n) < 1e-6, name


def test_backward_homogeneity(oracle):
    """o and the final state are linear in r (o only), in k, in v, and affine
    in the initial state; the bonus part of o is linear in u. Euler's theorem
    then fixes sum(x * gx) for each, at any size."""
    rng = np.random.default_rng(41)
    B, T, H, K = 2, 40, 2, 8
    r, k, v, w, u, dout, s0, gf = _bwd_case(rng, B, T, H, K)
    gr, gk, gv, gw, gu, gi = oracle.wkv6_backward(r, k, v, w, u, dout, init_state=s0, g_final=gf)
    o, fs = oracle.wkv6_forward(r, k, v, w, u, init_state=s0)
    Lo, Lf = float((o * dout).sum()), float((fs * gf).sum())
    assert np.isclose((r * gr).sum(), Lo, rtol=1e-11)
    # with S_-1 = 0 the outputs are bilinear in k and v
    o0, fs0 = oracle.wkv6_forward(r, k, v, w, u)
    L0 = float((o0 * dout).sum() + (fs0 * gf).sum())
    gr0, gk0, gv0, _, gu0, _ = oracle.wkv6_backward(r, k, v, w, u, dout, g_final=gf)
    assert np.isclose((k * gk0).sum(), L0, rtol=1e-11)
    assert np.isclose((v * gv0).sum(), L0, rtol=1e-11)
    # the initial state's share of L
    assert np.isclose((s0 * gi).sum(), Lo + Lf - L0, rtol=1e-11)
    # the bonus share: sum_t r_t . (u * k_t) (v_t . do_t)
    uu = u.reshape(1, 1, H * K)
    vdo = (v * dout).reshape(B, T, H, K).sum(-1, keepdims=True)
    bonus = ((r * uu * k).reshape(B, T, H, K) * vdo).sum()
    assert np.isclose((u.reshape(-1) * gu).sum(), bonus, rtol=1e-11)


def test_backward_state_map(oracle):
    """With a state map every sample's g_init is dL/dS_-1 of that sample."""
    rng = np.random.default_rng(42)
    B, T, H, K = 3, 6, 1, 3
    r, k, v, w, u, dout, _, gf = _bwd_case(rng, B, T, H, K)
    init = rng.normal(size=(2, H, K, K))
    smap = np.array([1, 0, 1], np.int32)
    *_, gi = oracle.wkv6_backward(r, k, v, w, u, dout, init_state=init, state_map=smap, g_final=gf)
    for b in range(B):
        sub = lambda x: x[b:b + 1]
        *_, gib = oracle.wkv6_backward(sub(r), sub(k), sub(v), sub(w), u, sub(dout),
                                       init_state=init[smap[b]][None], g_final=sub(gf))
        assert rel_err(gi[b], gib[0]) < 1e-14
