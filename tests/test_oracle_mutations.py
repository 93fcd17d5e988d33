"""Plant plausible mistakes in a copy of the oracle source and check that the
pins catch each one (CPU only; the committed oracle itself is untouched).
"""

import numpy as np
import pytest

from _pins import rel_err, wkv4_direct_sum, wkv4_fd_grads, wkv6_direct_sum

MUTATIONS = {
    # RWKV-4 forward: the bonus u dropped from the current token's weight
    "wkv4_drop_bonus": ("const double eu = exp(u[c] + k[idx] - K);    /* e^{u+k_t} (shifted) */",
                        "const double eu = exp(k[idx] - K);"),
    # RWKV-4 forward: the newest token decayed once too often
    "wkv4_extra_decay": ("a = decay * a + ek * v[idx];                 /* a_{t+1} */",
                         "a = decay * (a + ek * v[idx]);"),
    # RWKV-4 backward: wrong sign on the beta adjoint in gk
    "wkv4_gk_sign": ("gk[idx] += ek * (v[idx] * A - Bs);", "gk[idx] += ek * (v[idx] * A + Bs);"),
    # RWKV-4 backward: dropped term in the d/dw recurrence
    "wkv4_gw_term": ("const double da_next = decay * (da - a);", "const double da_next = decay * da;"),
    # RWKV-4 backward: local gu term with v and y swapped
    "wkv4_gu_swap": ("s_gu += gy[idx] * rho * (v[idx] - yt);", "s_gu += gy[idx] * rho * (yt - v[idx]);"),
    # RWKV-6: transposed outer product in the state update
    "wkv6_transpose": ("S[i * K + j] = w[row + i] * S[i * K + j] + k[row + i] * v[row + j];",
                       "S[i * K + j] = w[row + i] * S[i * K + j] + k[row + j] * v[row + i];"),
    # RWKV-6: bonus indexed by the value dimension
    "wkv6_u_index": ("u[h * K + i] * k[row + i] * v[row + j]", "u[h * K + j] * k[row + i] * v[row + j]"),
    # RWKV-6: decay indexed by the value dimension
    "wkv6_w_index": ("S[i * K + j] = w[row + i] * S[i * K + j]", "S[i * K + j] = w[row + j] * S[i * K + j]"),
    # RWKV-6 backward: bonus term dropped from gk
    "wkv6b_gk_bonus": ("gk[row + i] = b + u[h * K + i] * r[row + i] * vdo;", "gk[row + i] = b;"),
    # RWKV-6 backward: transposed outer product in the adjoint update
    "wkv6b_g_transpose": ("G[i * K + j] = w[row + i] * G[i * K + j] + r[row + i] * dout[row + j];",
                          "G[i * K + j] = w[row + i] * G[i * K + j] + r[row + j] * dout[row + i];"),
    # RWKV-6 backward: gw and gr against S_t instead of S_{t-1}
    "wkv6b_state_index": ("const double *S = Sh + t * K * K; /* S_{t-1} */",
                          "const double *S = Sh + (t + 1) * K * K;"),
    # RWKV-7: the log decay used as the decay itself
    "wkv7_no_exp": ("const double d = exp(w[row + j]);", "const double d = w[row + j];"),
    # RWKV-7: the removal projection taken with b instead of a
    "wkv7_ab_swap": ("for (int64_t j = 0; j < K; ++j) acc += a[row + j] * S[j * K + i];",
                     "for (int64_t j = 0; j < K; ++j) acc += b[row + j] * S[j * K + i];"),
    # RWKV-7: transposed outer product k v^T
    "wkv7_kv_transpose": ("b[row + j] * sa[i] + k[row + j] * v[row + i];",
                          "b[row + j] * sa[i] + k[row + i] * v[row + j];"),
    # RWKV-7: wrong sign on the rank-one term
    "wkv7_rank_one_sign": ("S[j * K + i] = d * S[j * K + i] + b[row + j] * sa[i]",
                           "S[j * K + i] = d * S[j * K + i] - b[row + j] * sa[i]"),
    # RWKV-7: the read leaves out the current token's write
    "wkv7_read_without_token": ("for (int64_t j = 0; j < K; ++j) acc += r[row + j] * S[j * K + i];",
                                "for (int64_t j = 0; j < K; ++j) acc += r[row + j] * (S[j * K + i] - k[row + j] * v[row + i]);"),
    # RWKV-7 backward: the rank-one term dropped from the adjoint walk
    "wkv7b_drop_rank_one": ("G[j * K + i] = exp(w[row + j]) * G[j * K + i] + a[row + j] * dsa[i];",
                            "G[j * K + i] = exp(w[row + j]) * G[j * K + i];"),
    # RWKV-7 backward: the decay gradient without the chain factor e^{w}
    "wkv7b_dw_factor": ("dw[row + j] = exp(w[row + j]) * sw;", "dw[row + j] = sw;"),
    # RWKV-7 backward: dr taken against S_{t-1} instead of S_t
    "wkv7b_dr_state": ("sr += St[j * K + i] * dout[row + i];", "sr += Sp[j * K + i] * dout[row + i];"),
    # time-shift mix: blend weights swapped between the token and the one before
    "tsm_swap_weights": ("const double o = xt * mix[m * C + c] + xx * (1.0 - mix[m * C + c]);",
                         "const double o = xx * mix[m * C + c] + xt * (1.0 - mix[m * C + c]);"),
    # time-shift mix: the shift taken from the next token instead of the previous one
    "tsm_shift_direction": ("                    if (t > 0)\n                        xx = x[(bi * T + t - 1) * C + c];\n"
                            "                    else if (x_prev)\n                        xx = x_prev[bi * C + c];\n"
                            "                    const double o",
                            "                    if (t + 1 < T)\n                        xx = x[(bi * T + t + 1) * C + c];\n"
                            "                    else if (x_prev)\n                        xx = x_prev[bi * C + c];\n"
                            "                    const double o"),
    # time-shift mix backward: the 1 - mix part scattered to the token's own row
    "tsmb_wrong_row": ("gx[(bi * T + t - 1) * C + c] += gm * (1.0 - mc);", "gx[(bi * T + t) * C + c] += gm * (1.0 - mc);"),
    # time-shift mix backward: flipped sign of the mix gradient
    "tsmb_gmix_sign": ("gmix[m * C + c] += gm * (xt - xx);", "gmix[m * C + c] += gm * (xx - xt);"),
}


@pytest.fixture(scope="module")
def variants(tmp_path_factory, oracle):
    src = oracle.source_text()
    out = {}
    for name, (old, new) in MUTATIONS.items():
        assert src.count(old) == 1, f"mutation {name} does not match the oracle source"
        d = tmp_path_factory.mktemp(name)
        out[name] = oracle.build_variant(src.replace(old, new), str(d))
    return out


def _wkv4_pins_fail(var):
    rng = np.random.default_rng(31)
    C, T = 3, 10
    w = np.exp(rng.uniform(-3, 1, size=C))
    u = rng.uniform(-1, 1, size=C)
    k = rng.normal(size=(1, T, C))
    v = rng.normal(size=(1, T, C))
    gy = rng.normal(size=k.shape)
    if rel_err(var.wkv4_forward(w, u, k, v), wkv4_direct_sum(w, u, k, v)) > 1e-9:
        return True
    got = var.wkv4_backward(w, u, k, v, gy)
    num = wkv4_fd_grads(var.wkv4_forward, w, u, k, v, gy)
    return any(rel_err(g, n) > 1e-6 for g, n in zip(got, num))


def _wkv6_pins_fail(var):
    rng = np.random.default_rng(32)
    B, T, H, K = 1, 8, 2, 4
    r, k, v = (rng.normal(size=(B, T, H * K)) for _ in range(3))
    w = rng.uniform(0.3, 1.0, size=(B, T, H * K))
    u = rng.uniform(-1, 1, size=(H, K))
    o, _ = var.wkv6_forward(r, k, v, w, u)
    return rel_err(o, wkv6_direct_sum(r, k, v, w, u, K)) > 1e-9


def _wkv6b_pins_fail(var):
    from _pins import wkv6_fd_grads
    rng = np.random.default_rng(33)
    B, T, H, K = 1, 5, 1, 3
    r, k, v, dout = (rng.normal(size=(B, T, H * K)) for _ in range(4))
    w = rng.uniform(0.3, 1.0, size=(B, T, H * K))
    u = rng.uniform(-1, 1, size=(H, K))
    s0, gf = rng.normal(size=(B, H, K, K)), rng.normal(size=(B, H, K, K))
    got = var.wkv6_backward(r, k, v, w, u, dout, init_state=s0, g_final=gf)
    num = wkv6_fd_grads(var.wkv6_forward, r, k, v, w, u, dout, init_state=s0, g_final=gf)
    return any(rel_err(g, n) > 1e-6 for g, n in zip(got, num))


def _wkv7_pins_fail(var):
    import test_oracle_wkv7 as p7

    class _Adapter:  # the pin functions take the oracle module; give them the variant
        wkv7_forward = staticmethod(var.wkv7_forward)
    for pin in (p7.test_delta_rule_stores_and_reads_back, p7.test_hand_worked_two_steps,
                lambda o: p7.test_without_the_rank_one_term(o, "b_zero")):
        try:
            pin(_Adapter)
        except AssertionError:
            return True
    return False


def _wkv7b_pins_fail(var):
    import test_oracle_wkv7 as p7

    class _Adapter:
        wkv7_forward = staticmethod(var.wkv7_forward)
        wkv7_backward = staticmethod(var.wkv7_backward)
    for pin in (lambda o: p7.test_backward_matches_finite_differences(o, True), p7.test_backward_homogeneity):
        try:
            pin(_Adapter)
        except AssertionError:
            return True
    return False


def _tsm_pins_fail(var):
    import test_oracle_time_shift as pt

    class _Adapter:
        time_shift_mix = staticmethod(var.time_shift_mix)
        time_shift_mix_backward = staticmethod(var.time_shift_mix_backward)
    pins = (pt.test_hand_worked, pt.test_ends_of_the_blend, pt.test_pieces_with_x_prev_match_one_call,
            pt.test_backward_closed_form_for_unit_gradient, lambda o: pt.test_backward_matches_finite_differences(o, True))
    for pin in pins:
        try:
            pin(_Adapter)
        except AssertionError:
            return True
    return False


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(variants, name):
    check = (_wkv4_pins_fail if name.startswith("wkv4") else
             _wkv7b_pins_fail if name.startswith("wkv7b") else
             _tsm_pins_fail if name.startswith("tsm") else
             _wkv7_pins_fail if name.startswith("wkv7") else
             _wkv6b_pins_fail if name.startswith("wkv6b") else _wkv6_pins_fail)
    assert check(variants[name]), f"planted mistake {name} passed every pin"


def test_unmutated_source_passes(oracle):
    class _Orig:
        wkv4_forward = staticmethod(oracle.wkv4_forward)
        wkv4_backward = staticmethod(oracle.wkv4_backward)
        wkv6_forward = staticmethod(oracle.wkv6_forward)
        wkv6_backward = staticmethod(oracle.wkv6_backward)
        wkv7_forward = staticmethod(oracle.wkv7_forward)
        wkv7_backward = staticmethod(oracle.wkv7_backward)
        time_shift_mix = staticmethod(oracle.time_shift_mix)
        time_shift_mix_backward = staticmethod(oracle.time_shift_mix_backward)
    assert not _wkv4_pins_fail(_Orig)
    assert not _tsm_pins_fail(_Orig)
    assert not _wkv7b_pins_fail(_Orig)
    assert not _wkv7_pins_fail(_Orig)
    assert not _wkv6_pins_fail(_Orig)
    assert not _wkv6b_pins_fail(_Orig)
