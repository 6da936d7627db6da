"""GPU parity of the certified decode step and of the dense reference against the oracle."""

import dataclasses

import numpy as np
import pytest
import torch

import synthetic_kv as sk
from tests.gpu_util import (OUT_TOL, TieLog, compare_decode, fill_cache, oracle_thresholds,
                            oracle_units, row, run_decode)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cqa():
    import certified_quantized_kv_int8_b200 as m
    from certified_quantized_kv_int8_b200.build import build
    build()
    m.load_library()
    return m


def _check(cqa, w, ctx, th, layers=(0,), step=0, label="", fp16_meta=False):
    from oracle import decode
    log = TieLog()
    with cqa.Cache(len(layers), w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, ctx,
                   meta_fp16=fp16_meta) as cache:
        fill_cache(cache, w, list(layers), ctx)
        for i, layer in enumerate(layers):
            q = sk.queries(w, layer, step, "cuda")
            res = run_decode(cache, i, q, th)
            qc = q.cpu().numpy()
            for b in range(w.batch):
                units = oracle_units(w, layer, b, ctx, fp16_meta)
                ora = decode(qc[b], units, oracle_thresholds(th))
                compare_decode(row(res, b), ora, oracle_thresholds(th), w.group, log,
                               label=f"{label} layer {layer} b {b}")
    for e in log.entries:
        print("tie logged:", e)
    return log


TINY_TH = {
    "default": {},
    "tau0.5": dict(tau_cov=0.5),
    "tau0.9_vtol": dict(tau_cov=0.9, v_tol=2e-3),
    "widen": dict(tau_cov=0.3, eps_key=1e-3, max_expand=6),
    "naive": dict(naive=True),
    "full_promotion": dict(tau_cov=1.0, v_tol=0.0),
    "head_dense": dict(tau_cov=0.3, eps_key=-1.0, max_expand=0),
    "layer_dense": dict(layer_dense_frac=0.0),
    "rank2": dict(rank_r=2, tau_cov=0.8),
    "val_post_check": dict(tau_cov=0.9, eps_val=0.17),
    "val_post_check_tight": dict(eps_val=0.0),
}


@pytest.mark.parametrize("case", list(TINY_TH))
@pytest.mark.parametrize("ctx", [1024, 1024 + 19])
def test_decode_tiny(cqa, case, ctx):
    w = sk.WORKLOADS["tiny"]
    th = cqa.Thresholds(**{**sk.default_thresholds(w), **TINY_TH[case]})
    log = _check(cqa, w, ctx, th, label=case)
    assert len(log.entries) <= 1


@pytest.mark.parametrize("ctx", [1, 37, 64, 65, 128 + 63])
@pytest.mark.parametrize("naive", [False, True])
def test_decode_short_contexts(cqa, ctx, naive):
    """No sealed block, one, two: the streaming passes then run fewer CTAs per unit
    than their grid target, down to one that holds only the residual block."""
    w = sk.WORKLOADS["tiny"]
    th = cqa.Thresholds(**{**sk.default_thresholds(w), "tau_cov": 0.7, "naive": naive})
    _check(cqa, w, ctx, th, label=f"ctx{ctx}{' naive' if naive else ''}")


@pytest.mark.parametrize("name,ctx", [("tiny", 1024 + 19), ("llama8b_8k_1layer", 8192 + 21),
                                      ("llama8b_64k_b4_t3values", 4096 + 5)])
@pytest.mark.parametrize("naive", [False, True])
def test_decode_fp16_meta(cqa, name, ctx, naive):
    """Binary16 Tier-1 metadata through the certified and the INT8/INT4 paths."""
    w = sk.WORKLOADS[name]
    th = cqa.Thresholds(**{**sk.default_thresholds(w), "tau_cov": 0.8, "naive": naive})
    log = _check(cqa, w, ctx, th, label=f"fp16 meta {name}", fp16_meta=True)
    assert len(log.entries) <= 2


@pytest.mark.parametrize("nb", [40, 200, 256, 257])
@pytest.mark.parametrize("case", ["default", "widen", "tau0.9_vtol", "naive"])
def test_decode_selection_sizes(cqa, nb, case):
    """Coverage selection runs one warp per query head with the head's blocks in
    registers up to 256 sealed blocks (32, 64, 128 or 256 sort keys per head),
    and the 1024-thread kernel above that: rows on both sides of each size, with
    widening, a tail with value promotion, and certification off."""
    w = sk.WORKLOADS["tiny"]
    th = cqa.Thresholds(**{**sk.default_thresholds(w), **TINY_TH[case]})
    log = _check(cqa, w, nb * 64 + 17, th, label=f"nb{nb} {case}")
    assert len(log.entries) <= 1


@pytest.mark.parametrize("nb", [200, 300])
def test_decode_selection_sizes_g4(cqa, nb):
    """The same two selection kernels at head_dim 128 with four query heads per kv
    head (eight kv heads, a tail and value promotion)."""
    w = sk.WORKLOADS["llama8b_8k_1layer"]
    th = cqa.Thresholds(**{**sk.default_thresholds(w), "tau_cov": 0.9, "v_tol": 2e-3})
    log = _check(cqa, w, nb * 64 + 9, th, label=f"g4 nb{nb}")
    assert len(log.entries) <= 2


def test_decode_llama8b_8k(cqa):
    w = sk.WORKLOADS["llama8b_8k_1layer"]
    th = cqa.Thresholds(**sk.default_thresholds(w))
    _check(cqa, w, w.ctx, th, label="8k")
    th2 = cqa.Thresholds(**{**sk.default_thresholds(w), "tau_cov": 0.6, "v_tol": 2e-3})
    _check(cqa, w, w.ctx + 21, th2, label="8k-tail")


def test_full_promotion_equals_dense_reference(cqa):
    w = sk.WORKLOADS["llama8b_8k_1layer"]
    from oracle import dense_attention
    ctx = w.ctx + 9
    with cqa.Cache(1, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, ctx) as cache:
        fill_cache(cache, w, [0], ctx)
        q = sk.queries(w, 0, 0, "cuda")
        dense = cache.dense_reference(0, q).cpu().numpy()
        out, ek, ev, rung = cache.decode(0, q, cqa.Thresholds(tau_cov=1.0, v_tol=0.0, rank_r=0,
                                                              layer_dense_frac=2.0))
        torch.cuda.synchronize()
        assert np.all(ek.cpu().numpy() == 0) and np.all(ev.cpu().numpy() == 0)
        assert np.abs(out.cpu().numpy() - dense).max() <= 1e-5
        forced, fk, fv, frung = cache.decode(0, q, cqa.Thresholds(layer_dense_frac=0.0))
        torch.cuda.synchronize()
        assert np.all(frung.cpu().numpy() == 4) and np.all(fk.cpu().numpy() == 0)
        # the forced whole-layer fallback is exact attention (float32 rounding apart)
        assert np.abs(forced.cpu().numpy() - dense).max() <= 1e-5
        K, V = sk.kv_layer(w, 0, 0, ctx, "cpu")
        qc = q.cpu().numpy()[0]
        G = w.group
        for h in range(w.n_q_heads):
            ref = dense_attention(qc[h:h + 1], K[0, h // G].numpy(), V[0, h // G].numpy())[0]
            assert np.abs(dense[0, h] - ref).max() <= 1e-4


def test_bounds_certify_the_device_output(cqa):
    """max_c |out - O_dense| <= R_V E_key + E_val on every certified head."""
    w = sk.WORKLOADS["llama8b_8k_1layer"]
    ctx = w.ctx
    with cqa.Cache(1, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, ctx) as cache:
        fill_cache(cache, w, [0], ctx)
        q = sk.queries(w, 0, 3, "cuda")
        for tau in (0.5, 0.9, 0.995):
            th = cqa.Thresholds(tau_cov=tau, eps_key=1.0, rank_r=0, layer_dense_frac=2.0,
                                v_tol=float("inf"))
            out, ek, ev, rung = cache.decode(0, q, th)
            dense = cache.dense_reference(0, q)
            torch.cuda.synchronize()
            vr = cache.export(0, 5)[0]
            rv = (vr[:, 1] - vr[:, 0]).max(axis=1)
            err = (out - dense).abs().amax(dim=2).cpu().numpy()[0]
            bound = np.repeat(rv, w.group) * ek.cpu().numpy()[0] + ev.cpu().numpy()[0]
            assert np.all(err <= bound * (1 + 1e-3) + 1e-5)


@pytest.mark.parametrize("name,layers,ctx_extra", [
    ("llama8b_32k_32layer_append", (0, 11, 31), 0),
    ("llama8b_64k_b4_t3values", (5,), 0),
    ("llama8b_128k_needle", (17, 3, 30), 0),
])
def test_decode_full_size_sampled(cqa, name, layers, ctx_extra):
    """Full-context decode in the launch configuration of the benchmark, checked
    against the oracle on sampled layers (every batch row and head of them)."""
    w = sk.WORKLOADS[name]
    th = cqa.Thresholds(**sk.default_thresholds(w))
    log = _check(cqa, w, w.ctx + ctx_extra, th, layers=layers, label=name)
    assert len(log.entries) <= 4


def test_appended_steps_match_oracle(cqa):
    """The 32K workload appends one token per layer before each decode step."""
    from oracle import decode
    w = sk.WORKLOADS["llama8b_32k_32layer_append"]
    w = dataclasses.replace(w, ctx=4096, appends=8)
    th = cqa.Thresholds(**sk.default_thresholds(w))
    log = TieLog()
    with cqa.Cache(1, 1, w.n_q_heads, w.n_kv_heads, w.head_dim, w.max_ctx) as cache:
        fill_cache(cache, w, [7], w.ctx)
        for step in range(w.appends):
            t = w.ctx + step
            K, V = sk.kv_layer(w, 7, t, t + 1, "cuda")
            cache.append(0, K, V)
            q = sk.queries(w, 7, step, "cuda")
            res = run_decode(cache, 0, q, th)
            if step in (0, 5, 7):
                units = oracle_units(w, 7, 0, t + 1)
                ora = decode(q.cpu().numpy()[0], units, oracle_thresholds(th))
                compare_decode(row(res, 0), ora, oracle_thresholds(th), w.group, log,
                               label=f"step {step}")
    assert len(log.entries) <= 1


def test_key_prefetch_changes_no_result(cqa):
    """Staging a layer's keys with the copy engine gives bit-identical decodes,
    across appends that seal new blocks between the copy and its use."""
    w = sk.WORKLOADS["llama8b_8k_1layer"]
    ctx = 4096 + 60
    th = cqa.Thresholds(**sk.default_thresholds(w))
    results = {}
    for mode in (0, 2, 1):
        with cqa.Cache(2, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, ctx + 16) as cache:
            cache.set_key_prefetch(mode, 0.5)
            fill_cache(cache, w, [0, 1], ctx)
            outs = []
            for step in range(3):
                for layer in (0, 1):
                    t = ctx + 4 * step
                    K, V = sk.kv_layer(w, layer, t, t + 4, "cuda")  # seals a block at step 1
                    cache.append(layer, K, V)
                    q = sk.queries(w, layer, step, "cuda")
                    o = cache.decode(layer, q, th)
                    torch.cuda.synchronize()
                    outs.append([x.cpu().numpy() for x in o])
            results[mode] = outs
    for mode in (2, 1):
        for a, b in zip(results[0], results[mode]):
            for x, y in zip(a, b):
                assert np.array_equal(x, y), f"prefetch mode {mode} changed a result"


@pytest.mark.parametrize("name,layer", [("llama8b_8k_1layer", 0), ("llama8b_64k_b4_t3values", 2),
                                        ("llama8b_128k_needle", 17)])
def test_naive_path_full_size(cqa, name, layer):
    """Certification off: the fused INT8/INT4 streaming pass against the oracle's
    naive mode (no promotion, bounds over the whole tail)."""
    w = sk.WORKLOADS[name]
    th = cqa.Thresholds(**{**sk.default_thresholds(w), "naive": True})
    log = _check(cqa, w, w.ctx + 33, th, layers=(layer,), label=f"naive {name}")
    assert not log.entries


@pytest.mark.parametrize("d,hq,hkv", [(128, 8, 8), (128, 8, 4), (128, 16, 2), (64, 2, 2),
                                      (64, 8, 2)])
@pytest.mark.parametrize("naive", [False, True])
def test_head_shapes(cqa, d, hq, hkv, naive):
    """Every supported (head_dim, query heads per kv head) pair against the oracle,
    with a tail (tau 0.8), value promotion and a batch of two."""
    base = sk.WORKLOADS["tiny"]
    w = dataclasses.replace(base, name=f"shape{d}_{hq}_{hkv}", batch=2, n_q_heads=hq,
                            n_kv_heads=hkv, head_dim=d, n_outlier=2)
    th = cqa.Thresholds(**{**sk.default_thresholds(w), "tau_cov": 0.8, "v_tol": 3e-3,
                           "naive": naive})
    log = _check(cqa, w, 20 * 64 + 11, th, label=f"d{d} g{hq // hkv}")
    assert len(log.entries) <= 1
