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
