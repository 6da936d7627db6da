"""Pins of the oracle's certified bounds (E_key, E_val, output bound).

E_key is checked against a closed-form worst case (the tanh bound is attained),
against brute force over every extreme perturbation pattern on tiny inputs,
and, like E_val, as a valid upper bound on every head of decoded workloads.
"""

import math

import numpy as np
import pytest

from oracle import BLOCK, Thresholds, build_unit, decode, dense_attention, e_key_bound
from tests.golden import load


def _softmax(x):
    e = np.exp(x - x.max())
    return e / e.sum()


def test_tanh_branch_attained_hand_fixture():
    g = load("bounds_hand.txt")
    delta = float(g["delta"][0])
    x = np.zeros(4)
    shifted = _softmax(x + np.array([delta, -delta, -delta, -delta]))
    np.testing.assert_allclose(shifted, g["shifted"], rtol=1e-14)
    tv = 0.5 * np.abs(shifted - _softmax(x)).sum()
    assert abs(tv - g["tv"][0]) < 1e-14
    # with the whole distribution in the tail (m8 = 1) the tanh branch is active
    assert abs(e_key_bound(delta, delta, 1.0) - tv) < 1e-14


def test_mass_branch_hand_fixture():
    g = load("bounds_hand.txt")
    for d_all, want in zip(g["mass_delta_all"], g["mass_e_key"]):
        got = e_key_bound(float(g["mass_delta_tail"][0]), float(d_all), float(g["mass_m8"][0]))
        assert abs(got - want) <= 1e-15


def test_special_cases():
    assert e_key_bound(0.0, 0.0, 0.0) == 0.0
    assert e_key_bound(0.0, 0.3, 0.2) == 0.0  # no perturbation on the tail
    assert e_key_bound(0.5, 0.5, 0.0) == 0.0  # no tail mass
    # small tail mass: the mass branch is the smaller one
    b = e_key_bound(0.1, 0.1, 1e-3)
    m_ub = 1e-3 * math.exp(0.1) / (1e-3 * math.exp(0.1) + (1 - 1e-3) * math.exp(-0.1))
    assert abs(b - m_ub * math.expm1(0.2)) < 1e-15
    assert b < math.tanh(0.05)


def test_brute_force_extreme_perturbations(rng):
    """Exact TV over all +-Delta sign patterns on the tail never exceeds the bound."""
    worst_ratio = 0.0
    for trial in range(300):
        n = int(rng.integers(2, 10))
        x = rng.normal(0, 2.0, n)
        d_tok = rng.uniform(0, 0.8, n)
        tail = rng.random(n) < 0.5
        if not tail.any():
            tail[0] = True
        # INT8-estimate logits: any perturbation within +-Delta on every token
        x8 = x + d_tok * rng.choice([-1.0, 1.0], n)
        m8 = _softmax(x8)[tail].sum()
        dT, dA = d_tok[tail].max(), d_tok.max()
        bound = e_key_bound(dT, dA, m8)
        p = _softmax(x)
        tidx = np.nonzero(tail)[0]
        for mask in range(1 << tidx.size):
            y = x.copy()
            for j, i in enumerate(tidx):
                y[i] += d_tok[i] if (mask >> j) & 1 else -d_tok[i]
            # the tail keeps the exact shift; the INT8 estimate m8 used above may
            # come from a different pattern, so also test the pattern itself
            tv = 0.5 * np.abs(_softmax(y) - p).sum()
            m8_same = _softmax(y + np.where(tail, 0.0, x8 - x))[tail].sum()
            b_same = e_key_bound(dT, dA, m8_same)
            assert tv <= b_same * (1 + 1e-12) + 1e-15
            worst_ratio = max(worst_ratio, tv / max(b_same, 1e-300))
        del bound
    assert worst_ratio > 0.3  # the bound is not vacuous on these cases


def _unit_from(rng, T, d, outlier=10.0, heavy_v=False, fp16_meta=False):
    K = rng.standard_normal((T, d))
    K[:, :4] *= outlier
    V = rng.standard_t(3, (T, d)) if heavy_v else rng.standard_normal((T, d))
    return build_unit(K.astype(np.float16), V.astype(np.float16), fp16_meta)


@pytest.mark.parametrize("tau", [0.5, 0.9, 0.995])
@pytest.mark.parametrize("heavy_v", [False, True])
@pytest.mark.parametrize("fp16_meta", [False, True])
def test_bounds_hold_on_decoded_heads(rng, tau, heavy_v, fp16_meta):
    d, G, Hkv = 64, 2, 2
    for trial in range(3):
        T = int(rng.integers(4, 20)) * BLOCK + int(rng.integers(0, BLOCK))
        units = [_unit_from(rng, T, d, outlier=float(rng.choice([1.0, 10.0, 40.0])),
                            heavy_v=heavy_v, fp16_meta=fp16_meta) for _ in range(Hkv)]
        q = rng.standard_normal((G * Hkv, d)).astype(np.float16)
        th = Thresholds(tau_cov=tau, eps_key=1.0, v_tol=float("inf"), rank_r=0,
                        layer_dense_frac=2.0)
        res = decode(q, units, th)
        for gi, g in enumerate(res["groups"]):
            u = units[gi]
            for h in range(G):
                hq = gi * G + h
                assert res["rung"][hq] < 3
                s = (q[hq].astype(np.float64) @ u["K"].astype(np.float64).T) / math.sqrt(d)
                p_exact = _softmax(s)
                tv = 0.5 * np.abs(p_exact - g["p"][h]).sum()
                assert tv <= res["e_key"][hq] * (1 + 1e-4) + 1e-12
                o_dense = dense_attention(q[hq:hq + 1], u["K"], u["V"])[0]
                err = np.abs(o_dense - res["out"][hq]).max()
                assert err <= res["e_out"][hq] * (1 + 1e-4) + 1e-9
                # value part alone: same weights, exact vs reconstructed values
                v_exact = g["p"][h] @ u["V"].astype(np.float64)
                assert np.abs(v_exact - res["out"][hq]).max() <= res["e_val"][hq] + 1e-9


def _eval_fixture_unit():
    """The unit of tests/golden/eval_hand.txt: three sealed blocks and ten residual tokens."""
    d, T = 64, 3 * BLOCK + 10
    K = np.zeros((T, d), np.float16)
    K[64:128, 0] = 1.0
    K[128, 0] = -100.0
    K[129:192, 0] = 0.5
    K[192:, 0] = 1.5
    V = np.zeros((T, d), np.float16)
    V[:, 1] = 15.0
    V[0, 2], V[64, 2], V[130, 2] = 0.5, 0.25, 0.125
    q = np.zeros((1, d), np.float16)
    q[0, 0] = 8.0
    return q, build_unit(K, V)


@pytest.mark.parametrize("case", ["A", "B"])
def test_e_val_hand_fixture(case):
    """E_val = sum over INT4-valued blocks of final attention mass x eta_b, against
    the hand-worked closed form (value-promoted blocks excluded; the mass is the
    final mixed distribution, residual included, not the INT8 estimate)."""
    from oracle.cqa_oracle import decode_group
    g = load("eval_hand.txt")
    q, u = _eval_fixture_unit()
    np.testing.assert_array_equal(u["eta"], g["eta"].astype(np.float32))
    assert float(u["kscale"][2, 0]) == float(g["s_block2"][0])
    if case == "A":
        th = Thresholds(tau_cov=1.0, v_tol=float(g["v_tol"][0]))
    else:
        th = Thresholds(tau_cov=0.5, eps_key=1.0, v_tol=float(g["v_tol"][0]))
    res = decode_group(q, u, th)
    np.testing.assert_array_equal(res["P"], g[f"promoted_{case}"].astype(bool))
    np.testing.assert_array_equal(res["VP"], g["value_promoted"].astype(bool))
    want = float(g[f"e_val_{case}"][0])
    assert abs(float(res["e_val"][0]) - want) <= 1e-13 * want
