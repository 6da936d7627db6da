"""Pins of the oracle's decode step: exact dense attention (hand fixture and
closed forms), the INT8 scoring pass and its perturbation bound Delta, the
full-promotion and forced-fallback cases that must return O_dense, and the
stated rules of the ladder."""

import math

import numpy as np
import pytest

import synthetic_kv as sk
from oracle import BLOCK, Thresholds, build_unit, decode, dense_attention
from oracle.cqa_oracle import decode_group
from tests.golden import load


def test_dense_hand_fixture():
    g = load("dense_hand.txt")
    out = dense_attention(g["q"][None].astype(np.float16), g["k"].astype(np.float16),
                          g["v"].astype(np.float16))
    np.testing.assert_allclose(out[0], g["out"], rtol=0, atol=1e-15)


def test_dense_zero_query_is_mean(rng):
    K = rng.standard_normal((100, 64)).astype(np.float16)
    V = rng.standard_normal((100, 64)).astype(np.float16)
    out = dense_attention(np.zeros((1, 64), np.float16), K, V)
    np.testing.assert_allclose(out[0], V.astype(np.float64).mean(0), atol=1e-14)


def _units(rng, Hkv, T, d, outlier=10.0):
    us = []
    for _ in range(Hkv):
        K = rng.standard_normal((T, d))
        K[:, :4] *= outlier
        V = rng.standard_normal((T, d))
        us.append(build_unit(K.astype(np.float16), V.astype(np.float16)))
    return us


def _dense_all(q, units):
    G = q.shape[0] // len(units)
    return np.stack([dense_attention(q[h:h + 1], units[h // G]["K"], units[h // G]["V"])[0]
                     for h in range(q.shape[0])])


def test_full_promotion_is_dense(rng):
    """tau_cov = 1 and v_tol = 0 promote every key and value: the output is O_dense
    and both bounds vanish (Methodology §3, deterministic recovery)."""
    q = rng.standard_normal((8, 64)).astype(np.float16)
    units = _units(rng, 2, 7 * BLOCK + 9, 64)
    th = Thresholds(tau_cov=1.0, v_tol=0.0, rank_r=0, layer_dense_frac=2.0)
    res = decode(q, units, th)
    np.testing.assert_allclose(res["out"], _dense_all(q, units), atol=1e-12)
    assert np.all(res["e_key"] == 0) and np.all(res["e_val"] == 0)


def test_forced_layer_fallback_is_dense(rng):
    q = rng.standard_normal((8, 64)).astype(np.float16)
    units = _units(rng, 2, 5 * BLOCK + 3, 64)
    res = decode(q, units, Thresholds(layer_dense_frac=0.0))
    assert res["layer_dense"] and np.all(res["rung"] == 4)
    np.testing.assert_array_equal(res["out"], _dense_all(q, units))
    assert np.all(res["e_key"] == 0) and np.all(res["e_val"] == 0)


def test_forced_head_fallback(rng):
    """eps_key < 0 fails every head whose tail is not empty after max_expand rounds."""
    q = rng.standard_normal((8, 64)).astype(np.float16)
    units = _units(rng, 2, 9 * BLOCK, 64)
    th = Thresholds(tau_cov=0.3, eps_key=-1.0, max_expand=0, rank_r=0, layer_dense_frac=2.0)
    res = decode(q, units, th)
    assert np.all(res["rung"] == 3)
    np.testing.assert_array_equal(res["out"], _dense_all(q, units))


def test_int8_scores_exact_when_keys_on_the_grid(rng):
    """Keys that are integer multiples of amax/127 quantise without error, so the
    INT8 block log-masses equal the FP16 ones."""
    d, T = 64, 4 * BLOCK
    ints = rng.integers(-127, 128, (T, d))
    ints[0::BLOCK, :] = 127  # every block's amax is 127 * 2^-7 -> scale 2^-7
    K = (ints * 2.0 ** -7).astype(np.float16)
    V = rng.standard_normal((T, d)).astype(np.float16)
    u = build_unit(K, V)
    assert np.all(u["kscale"] == np.float32(2.0 ** -7))
    q = rng.standard_normal((2, d)).astype(np.float16)
    g = decode_group(q, u, Thresholds(tau_cov=1.0))
    np.testing.assert_allclose(g["ell8"], g["ell16"], atol=1e-12)


def test_delta_bounds_and_is_attained(rng):
    """|logit8 - logit16| <= Delta per token; keys at exact half steps with the
    query's signs aligned reach Delta."""
    d = 64
    sign = np.where(rng.random(d) < 0.5, -1.0, 1.0)
    q = (np.abs(rng.standard_normal(d)) * sign).astype(np.float16)
    K = np.zeros((BLOCK, d))
    K[0] = 127 * 2.0 ** -7  # amax row -> scale 2^-7
    # half steps (code + 1/2) * 2^-7 with even code below: round-half-even goes down,
    # so the error k - k_hat = +2^-8 everywhere; put it on the query's sign
    K[1:] = sign * (2 * 10 + 0.5) * 2.0 ** -7
    u = build_unit(K.astype(np.float16), np.zeros((BLOCK, d), np.float16))
    g = decode_group(q[None], u, Thresholds(tau_cov=1.0))
    sigma = 1 / math.sqrt(d)
    qd = q.astype(np.float64)
    khat = u["kcodes"][0].astype(np.float64) * u["kscale"][0].astype(np.float64)
    l8 = sigma * khat @ qd
    l16 = sigma * K @ qd
    err = np.abs(l8 - l16)
    assert np.all(err <= g["delta"][0, 0] * (1 + 1e-12))
    assert abs(err[1:].max() - g["delta"][0, 0]) <= 1e-12


def test_rung_reporting_rules(rng):
    q = rng.standard_normal((8, 64)).astype(np.float16)
    units = _units(rng, 2, 12 * BLOCK + 5, 64)
    # coverage too small for eps_key: widening happens, heads report rung 1
    th = Thresholds(tau_cov=0.2, eps_key=1e-4, v_tol=float("inf"), rank_r=0,
                    layer_dense_frac=2.0, max_expand=8)
    res = decode(q, units, th)
    assert np.all(res["rung"] == 1)
    assert all(g["rounds"] >= 1 for g in res["groups"])
    # value promotion of every block with nonzero mass: rung 2
    th = Thresholds(tau_cov=1.0, v_tol=0.0, rank_r=0, layer_dense_frac=2.0)
    res = decode(q, units, th)
    assert np.all(res["rung"] == 2)


def test_rank_rule_on_constructed_orders():
    """Rank check (stated rule): ordered top-r by INT8 log-mass equals ordered
    top-r by FP16 log-mass over the promoted blocks."""
    from oracle import rank_consistent
    ell16 = np.array([5.0, 4.0, 3.0, 2.0, 1.0, 0.0])
    allp = np.ones(6, bool)
    assert rank_consistent(ell16 + 0.01, ell16, allp, 3)
    # a swap inside the top 3 fails, a swap below it does not
    assert not rank_consistent(np.array([4.0, 5.0, 3.0, 2.0, 1.0, 0.0]), ell16, allp, 3)
    assert rank_consistent(np.array([5.0, 4.0, 3.0, 1.0, 2.0, 0.0]), ell16, allp, 3)
    # only promoted blocks take part: block 0 unpromoted hides the swap of 0 and 1
    p = allp.copy()
    p[0] = False
    assert rank_consistent(np.array([3.5, 5.0, 3.0, 2.0, 1.0, 0.0]), ell16, p, 3)
    # equal INT8 log-masses order by the lower index
    assert rank_consistent(np.array([5.0, 5.0, 3.0, 2.0, 1.0, 0.0]), ell16, allp, 2)
    assert not rank_consistent(np.array([5.0, 5.0, 3.0, 2.0, 1.0, 0.0]),
                               np.array([4.0, 5.0, 3.0, 2.0, 1.0, 0.0]), allp, 2)
    # r larger than the promoted set, and an empty promoted set
    assert rank_consistent(ell16, ell16, allp, 99)
    assert rank_consistent(ell16, ell16[::-1].copy(), np.zeros(6, bool), 4)


def test_rank_discordance_hand_cases():
    """Discordant pairs over the union of the two top-r lists, by hand."""
    from oracle import rank_discordance
    ell16 = np.array([5.0, 4.0, 3.0, 2.0, 1.0, 0.0])
    allp = np.ones(6, bool)
    # one neighbour swap: U = {0, 1, 2}, one discordant pair
    assert rank_discordance(np.array([4.0, 5.0, 3.0, 2.0, 1.0, 0.0]), ell16, allp, 3) == 1
    # the heaviest FP16 block ranked fifth by INT8: U = {0, 1, 2, 3} and block 0
    # is discordant with each of the three blocks INT8 put above it
    heavy16 = np.array([10.0, 4.0, 3.0, 2.0, 1.0, 0.0])
    assert rank_discordance(np.array([0.5, 4.0, 3.0, 2.0, 1.0, 0.0]), heavy16, allp, 3) == 3
    # a fully reversed top 3 of an otherwise agreeing ranking: 3 pairs
    assert rank_discordance(np.array([3.0, 4.0, 5.0, 2.0, 1.0, 0.0]), ell16, allp, 3) == 3
    # equal keys order by the lower index on both sides: no discordance
    assert rank_discordance(np.array([5.0, 5.0, 3.0, 2.0, 1.0, 0.0]),
                            np.array([4.0, 4.0, 3.0, 2.0, 1.0, 0.0]), allp, 4) == 0
    # unpromoted blocks take no part
    p = allp.copy()
    p[0] = False
    assert rank_discordance(np.array([0.5, 4.0, 3.0, 2.0, 1.0, 0.0]), heavy16, p, 3) == 0


def test_rank_discordance_brute_force(rng):
    """Against an independent formulation: each block's position in the full
    stable order of each ranking, and the pairs of the union whose positions
    compare differently; rank_tol = 0 is equality of the ordered top-r lists."""
    from oracle import rank_consistent, rank_discordance
    for trial in range(400):
        n = int(rng.integers(1, 14))
        e16 = np.round(rng.normal(0, 1, n), 1)  # rounding makes ties common
        e8 = np.round(e16 + rng.normal(0, 0.3, n), 1)
        P = rng.random(n) < 0.7
        r = int(rng.integers(0, 6))
        idx = np.nonzero(P)[0]
        if idx.size == 0:
            assert rank_discordance(e8, e16, P, r) == 0
            continue
        def positions(key):
            order = sorted(idx.tolist(), key=lambda j: (-key[j], j))
            return {j: k for k, j in enumerate(order)}, order
        p8, o8 = positions(e8)
        p16, o16 = positions(e16)
        rr = min(r, idx.size)
        U = set(o8[:rr]) | set(o16[:rr])
        want = sum(1 for a in U for b in U if a < b and (p8[a] < p8[b]) != (p16[a] < p16[b]))
        assert rank_discordance(e8, e16, P, r) == want
        assert rank_consistent(e8, e16, P, r, 0) == (o8[:rr] == o16[:rr])


def test_naive_mode_promotes_nothing(rng):
    q = rng.standard_normal((8, 64)).astype(np.float16)
    units = _units(rng, 2, 6 * BLOCK + 1, 64)
    res = decode(q, units, Thresholds(naive=True))
    assert np.all(res["rung"] == 0)
    assert all(not g["P"].any() and not g["VP"].any() for g in res["groups"])


def test_needle_workload_plants_fallbacks():
    """A shortened needle workload: near-tie blocks make heads of the planted group
    fail the rank check (rung 3) and the all-groups layer fall back whole (rung 4)."""
    base = sk.WORKLOADS["llama8b_128k_needle"]
    import dataclasses
    w = dataclasses.replace(base, ctx=16384, n_layers=2, tie_layer_all=1)
    th = Thresholds(**sk.default_thresholds(w))
    for layer in (0, 1):
        K, V = sk.kv_layer(w, layer, 0, w.ctx)
        q = sk.queries(w, layer, 0)
        units = [build_unit(K[0, g].numpy(), V[0, g].numpy()) for g in range(w.n_kv_heads)]
        res = decode(q[0].numpy(), units, th)
        tie_g = layer % w.n_kv_heads
        if layer == 1:
            assert res["layer_dense"] and np.all(res["rung"] == 4)
        else:
            assert not res["layer_dense"]
            assert (res["rung"][tie_g * w.group:(tie_g + 1) * w.group] == 3).sum() >= 2
