"""The seeded input generator: reproducible slices, the stated distributions."""

import numpy as np
import torch

import synthetic_kv as sk


def test_slices_regenerate_identically():
    w = sk.WORKLOADS["llama8b_8k_1layer"]
    K, V = sk.kv_unit(w, 0, 0, 3, 0, 512)
    K2, V2 = sk.kv_unit(w, 0, 0, 3, 128, 256)
    assert torch.equal(K[128:256], K2) and torch.equal(V[128:256], V2)
    assert not torch.equal(sk.kv_unit(w, 0, 0, 4, 0, 512)[0], K)


def test_distributions():
    w = sk.WORKLOADS["llama8b_8k_1layer"]
    K, V = sk.kv_unit(w, 0, 0, 0, 0, 8192)
    out = sk.outlier_channels(w, 0, 0, 0)
    assert len(out) == 4
    std = K.float().std(0).numpy()
    assert np.all(np.abs(std[out] - 10.0) < 0.5)
    rest = np.delete(std, out)
    assert np.all(np.abs(rest - 1.0) < 0.1)
    assert abs(float(V.float().std()) - 1.0) < 0.02
    q = sk.queries(w, 0, 0)
    assert q.shape == (1, 32, 128) and abs(float(q.float().std()) - 1.0) < 0.05


def test_student_t_values_and_drift():
    w4 = sk.WORKLOADS["llama8b_64k_b4_t3values"]
    _, V = sk.kv_unit(w4, 0, 0, 0, 0, 4096)
    kurt = float(((V.float() ** 4).mean() / (V.float() ** 2).mean() ** 2))
    assert kurt > 6.0  # heavy tails (a normal has 3)
    w3 = sk.WORKLOADS["llama8b_32k_32layer_append"]
    K0, _ = sk.kv_unit(w3, 0, 0, 0, 0, 64)
    K1, _ = sk.kv_unit(w3, 0, 0, 0, 32768 - 64, 32768)
    import dataclasses
    flat = dataclasses.replace(w3, drift_beta=0.0)
    F1, _ = sk.kv_unit(flat, 0, 0, 0, 32768 - 64, 32768)
    drift = (K1.double() - F1.double()).mean(0)
    assert float(drift.abs().mean()) > 0.5  # near beta * |u| at the end of the context


def test_ragged_rows():
    """A ragged workload lists each row's length; kv_row is the row's kv_unit stack."""
    w = sk.WORKLOADS["llama8b_ragged_b4"]
    lens = sk.row_lengths(w)
    assert len(lens) == w.batch and max(lens) == w.ctx and len(set(lens)) == w.batch
    assert sk.row_lengths(sk.WORKLOADS["tiny"]) == [1024]
    t = sk.WORKLOADS["tiny"]
    K, V = sk.kv_row(t, 0, 0, 10, 30)
    assert K.shape == (t.n_kv_heads, 20, t.head_dim) and K.is_contiguous()
    for g in range(t.n_kv_heads):
        k, v = sk.kv_unit(t, 0, 0, g, 10, 30)
        assert torch.equal(K[g], k) and torch.equal(V[g], v)
