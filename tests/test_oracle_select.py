"""Pins of the oracle's coverage selection (top-K* blocks covering tau_cov of
the estimated mass) by brute force over every subset of a 16-block context."""

import itertools

import numpy as np
import pytest

from oracle import coverage_kstar


def _masses(rng, nb, res_frac):
    ell = rng.normal(0, 1.5, nb)
    w = np.exp(ell)
    m_res = res_frac
    m = (1 - m_res) * w / w.sum()
    # the oracle works from log-masses; shift them consistently
    return np.log(m), m, m_res


@pytest.mark.parametrize("tau", [0.3, 0.8, 0.95, 0.995])
def test_minimum_cardinality_and_maximum_mass(rng, tau):
    nb = 16
    for trial in range(4):
        ell, m, m_res = _masses(rng, nb, float(rng.choice([0.0, 0.05])))
        kstar, order, cum = coverage_kstar(ell, m, m_res, tau)
        chosen = set(order[:kstar].tolist())
        best_k, best_mass = None, -1.0
        for k in range(nb + 1):
            for sub in itertools.combinations(range(nb), k):
                s = m_res + m[list(sub)].sum()
                if s >= tau:
                    best_k = k
                    best_mass = max(best_mass, s)
            if best_k is not None:
                break
        assert kstar == best_k
        got = m_res + m[list(chosen)].sum()
        assert abs(got - best_mass) <= 1e-12
        assert got >= tau - 1e-12


def test_edge_cases(rng):
    ell, m, m_res = _masses(rng, 8, 0.3)
    k, order, cum = coverage_kstar(ell, m, m_res, 1.0)
    assert k == 8
    k, _, _ = coverage_kstar(ell, m, m_res, 0.25)  # residual alone covers it
    assert k == 0
    k, order, _ = coverage_kstar(np.zeros(0), np.zeros(0), 1.0, 0.995)
    assert k == 0 and order.size == 0


def test_ties_break_to_lower_index():
    ell = np.array([0.0, 1.0, 1.0, 0.5, 1.0])
    m = np.exp(ell) / np.exp(ell).sum()
    _, order, _ = coverage_kstar(ell, m, 0.0, 0.5)
    assert order.tolist() == [1, 2, 4, 3, 0]
