"""Ragged batches: batch rows of one layer holding different lengths.  Each row
is checked against the oracle run on that row's own tokens (Tier-1 encoding
bit for bit, decode decisions, bounds and outputs), for the certified path,
the certification-off pass and the dense reference."""

import dataclasses

import numpy as np
import pytest
import torch

import synthetic_kv as sk
from tests.gpu_util import (TieLog, compare_decode, oracle_thresholds, row, run_decode)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cqa():
    import certified_quantized_kv_int8_b200 as m
    from certified_quantized_kv_int8_b200.build import build
    build()
    m.load_library()
    return m


def _fill_ragged(cache, w, layer, lens, chunk=None):
    """Row b of cache layer 0 <- tokens [0, lens[b]) of workload layer `layer`,
    appended one row at a time (in pieces of `chunk` tokens when given)."""
    for b, n in enumerate(lens):
        t = 0
        while t < n:
            t1 = n if chunk is None else min(n, t + chunk)
            k, v = sk.kv_row(w, layer, b, t, t1, "cuda")
            cache.append_row(0, b, k, v)
            t = t1
    torch.cuda.synchronize()


def _oracle_row(w, layer, b, n, fp16_meta=False):
    from oracle import build_unit
    K, V = sk.kv_row(w, layer, b, 0, n, "cpu")
    return [build_unit(K[g].numpy(), V[g].numpy(), fp16_meta) for g in range(w.n_kv_heads)]


def _check_decode(cache, w, layer, lens, th, step=0, label="", fp16_meta=False):
    from oracle import decode
    log = TieLog()
    q = sk.queries(w, layer, step, "cuda")
    res = run_decode(cache, 0, q, th)
    qc = q.cpu().numpy()
    for b, n in enumerate(lens):
        ora = decode(qc[b], _oracle_row(w, layer, b, n, fp16_meta), oracle_thresholds(th))
        compare_decode(row(res, b, n // 64), ora, oracle_thresholds(th), w.group, log,
                       label=f"{label} b {b} len {n}")
    for e in log.entries:
        print("tie logged:", e)
    return log


def _tiny_batch(batch):
    return dataclasses.replace(sk.WORKLOADS["tiny"], batch=batch)


TINY_LENS = [1, 37, 64 + 5, 1024 + 19]


def test_ragged_append_bit_exact(cqa):
    from oracle import pack_int4
    w = _tiny_batch(len(TINY_LENS))
    with cqa.Cache(1, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, 2048) as cache:
        _fill_ragged(cache, w, 0, TINY_LENS, chunk=100)
        assert cache.row_lengths(0) == TINY_LENS
        assert cache.length(0) == max(TINY_LENS)
        arrays = {what: cache.export(0, what) for what in range(8)}
        for b, n in enumerate(TINY_LENS):
            K, V = sk.kv_row(w, 0, b, 0, n, "cpu")
            for g, u in enumerate(_oracle_row(w, 0, b, n)):
                np.testing.assert_array_equal(arrays[0][b][g], u["kcodes"])
                np.testing.assert_array_equal(arrays[1][b][g], u["kscale"])
                np.testing.assert_array_equal(arrays[2][b][g], pack_int4(u["vcodes"]))
                np.testing.assert_array_equal(arrays[3][b][g][..., 0], u["vscale"])
                np.testing.assert_array_equal(arrays[3][b][g][..., 1], u["voffset"])
                np.testing.assert_array_equal(arrays[4][b][g], u["eta"])
                np.testing.assert_array_equal(arrays[5][b][g][0], u["vmin"])
                np.testing.assert_array_equal(arrays[5][b][g][1], u["vmax"])
                r = u["r"]
                np.testing.assert_array_equal(arrays[6][b][g][0], K[g, n - r:].numpy())
                np.testing.assert_array_equal(arrays[6][b][g][1], V[g, n - r:].numpy())
                np.testing.assert_array_equal(arrays[7][b][g][0], K[g].numpy())
                np.testing.assert_array_equal(arrays[7][b][g][1], V[g].numpy())


TINY_TH = {
    "default": {},
    "tau0.5": dict(tau_cov=0.5),
    "naive": dict(naive=True),
    "full_promotion": dict(tau_cov=1.0, v_tol=0.0),
    "head_dense": dict(tau_cov=0.3, eps_key=-1.0, max_expand=0),
    "layer_dense": dict(layer_dense_frac=0.0),
    "val_post_check": dict(tau_cov=0.9, eps_val=0.17),
}


@pytest.mark.parametrize("case", list(TINY_TH))
def test_ragged_decode_tiny(cqa, case):
    w = _tiny_batch(len(TINY_LENS))
    th = cqa.Thresholds(**{**sk.default_thresholds(w), **TINY_TH[case]})
    with cqa.Cache(1, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, 2048) as cache:
        _fill_ragged(cache, w, 0, TINY_LENS)
        log = _check_decode(cache, w, 0, TINY_LENS, th, label=case)
        assert len(log.entries) <= 2


@pytest.mark.parametrize("naive", [False, True])
def test_ragged_fp16_meta(cqa, naive):
    """Binary16 Tier-1 metadata with rows of different lengths appended in pieces:
    each row's codes, scales, offsets and eta_b bit for bit against the oracle's
    binary16 encoding of that row's tokens, then decode parity per row."""
    from oracle import pack_int4
    w = _tiny_batch(len(TINY_LENS))
    th = cqa.Thresholds(**{**sk.default_thresholds(w), "tau_cov": 0.8, "naive": naive})
    with cqa.Cache(1, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, 2048,
                   meta_fp16=True) as cache:
        _fill_ragged(cache, w, 0, TINY_LENS, chunk=100)
        arrays = {what: cache.export(0, what) for what in range(5)}
        for b, n in enumerate(TINY_LENS):
            for g, u in enumerate(_oracle_row(w, 0, b, n, fp16_meta=True)):
                np.testing.assert_array_equal(arrays[0][b][g], u["kcodes"])
                np.testing.assert_array_equal(arrays[1][b][g], u["kscale"])
                np.testing.assert_array_equal(arrays[2][b][g], pack_int4(u["vcodes"]))
                np.testing.assert_array_equal(arrays[3][b][g][..., 0], u["vscale"])
                np.testing.assert_array_equal(arrays[3][b][g][..., 1], u["voffset"])
                np.testing.assert_array_equal(arrays[4][b][g], u["eta"])
        log = _check_decode(cache, w, 0, TINY_LENS, th, label="fp16 meta", fp16_meta=True)
        assert len(log.entries) <= 2


LLAMA_LENS = [8192 + 21, 64 * 37, 2048, 5000]


@pytest.mark.parametrize("naive", [False, True])
def test_ragged_decode_llama8b_shape(cqa, naive):
    """Head shape of the 8K workload (d 128, group 4) with four rows of
    different lengths: the grids cover the longest row, shorter rows leave CTAs
    with no work."""
    w = dataclasses.replace(sk.WORKLOADS["llama8b_8k_1layer"], batch=len(LLAMA_LENS))
    th = cqa.Thresholds(**{**sk.default_thresholds(w), "naive": naive})
    with cqa.Cache(1, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, 8192 + 64) as cache:
        _fill_ragged(cache, w, 0, LLAMA_LENS)
        _check_decode(cache, w, 0, LLAMA_LENS, th, label="naive" if naive else "certified")


def test_ragged_dense_reference(cqa):
    from oracle import dense_attention
    w = _tiny_batch(len(TINY_LENS))
    G = w.group
    with cqa.Cache(1, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, 2048) as cache:
        _fill_ragged(cache, w, 0, TINY_LENS)
        q = sk.queries(w, 0, 1, "cuda")
        dense = cache.dense_reference(0, q).cpu().numpy()
        qc = q.cpu().numpy()
        for b, n in enumerate(TINY_LENS):
            K, V = sk.kv_row(w, 0, b, 0, n, "cpu")
            for h in range(w.n_q_heads):
                ref = dense_attention(qc[b, h:h + 1], K[h // G].numpy(), V[h // G].numpy())[0]
                assert np.abs(dense[b, h] - ref).max() <= 1e-4, (b, h)


def test_append_to_all_rows_of_a_ragged_layer(cqa):
    """cqa_quantize_append on rows of different lengths appends after each row's
    own tokens; the rows stay ragged."""
    w = _tiny_batch(3)
    lens = [70, 10, 200]
    n_new = 90
    with cqa.Cache(1, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, 1024) as cache:
        _fill_ragged(cache, w, 0, lens)
        ks, vs = zip(*(sk.kv_row(w, 0, b, n, n + n_new, "cuda") for b, n in enumerate(lens)))
        cache.append(0, torch.stack(ks).contiguous(), torch.stack(vs).contiguous())
        torch.cuda.synchronize()
        new = [n + n_new for n in lens]
        assert cache.row_lengths(0) == new
        th = cqa.Thresholds(**{**sk.default_thresholds(w), "tau_cov": 0.8})
        _check_decode(cache, w, 0, new, th, label="after append")


def test_prefetch_refreshes_after_a_row_seals(cqa):
    """The whole-layer key staging copies each row's sealed blocks; a block that
    seals in one row (the longest row unchanged) makes the staged copy stale."""
    w = _tiny_batch(2)
    lens = [1024, 300]
    th = cqa.Thresholds(**{**sk.default_thresholds(w), "tau_cov": 1.0})
    with cqa.Cache(1, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, 2048) as cache:
        cache.set_key_prefetch(2)
        _fill_ragged(cache, w, 0, lens)
        _check_decode(cache, w, 0, lens, th, label="staged")
        k, v = sk.kv_row(w, 0, 1, 300, 300 + 100, "cuda")
        cache.append_row(0, 1, k, v)
        lens = [1024, 400]
        _check_decode(cache, w, 0, lens, th, step=1, label="restaged")


def test_ragged_errors(cqa):
    w = _tiny_batch(2)
    with cqa.Cache(1, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, 128) as cache:
        k, v = sk.kv_row(w, 0, 0, 0, 100, "cuda")
        cache.append_row(0, 0, k, v)
        q = sk.queries(w, 0, 0, "cuda")
        with pytest.raises(cqa.CqaError) as ei:
            cache.decode(0, q, cqa.Thresholds())  # row 1 holds no token
        assert ei.value.code == -5
        with pytest.raises(cqa.CqaError) as ei:
            cache.dense_reference(0, q)
        assert ei.value.code == -5
        with pytest.raises(cqa.CqaError) as ei:
            cache.append_row(0, 0, k[:, :29].contiguous(), v[:, :29].contiguous())  # 129 > 128
        assert ei.value.code == -4
        with pytest.raises(cqa.CqaError) as ei:
            cqa.cqa_quantize_append_row(cache.handle, 0, 2, k, v)  # no row 2
        assert ei.value.code == -1
        assert cache.row_lengths(0) == [100, 0]
        torch.cuda.synchronize()
        assert cache.device_status() == 0
