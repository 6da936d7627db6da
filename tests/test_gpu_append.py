"""GPU parity of the append path (Tier-1 encoding) against the oracle, bit for bit."""

import numpy as np
import pytest
import torch

import synthetic_kv as sk
from tests.gpu_util import fill_cache

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cqa():
    import certified_quantized_kv_int8_b200 as m
    from certified_quantized_kv_int8_b200.build import build
    build()
    m.load_library()
    return m


def test_generator_identical_on_device():
    for name in ("tiny", "llama8b_32k_32layer_append", "llama8b_64k_b4_t3values",
                 "llama8b_128k_needle"):
        w = sk.WORKLOADS[name]
        nb = w.ctx // 64
        needle, ties = sk.plant_positions(w, nb)
        lo = needle * 64 - 100 if w.needle else 3000
        for layer in (0, w.tie_layer_all if w.needle and w.n_layers > w.tie_layer_all else 0):
            kc, vc = sk.kv_unit(w, layer, w.batch - 1, w.n_kv_heads - 1, lo, lo + 300, "cpu")
            kg, vg = sk.kv_unit(w, layer, w.batch - 1, w.n_kv_heads - 1, lo, lo + 300, "cuda")
            assert torch.equal(kc, kg.cpu()) and torch.equal(vc, vg.cpu()), name
        qc = sk.queries(w, 0, 5, "cpu")
        assert torch.equal(qc, sk.queries(w, 0, 5, "cuda").cpu())


def _check_unit_arrays(cache, layer, w, wl, ctx, fp16_meta=False):
    from oracle import build_unit, pack_int4
    kc = cache.export(layer, 0)
    ks = cache.export(layer, 1)
    vc = cache.export(layer, 2)
    vm = cache.export(layer, 3)
    eta = cache.export(layer, 4)
    vr = cache.export(layer, 5)
    res = cache.export(layer, 6)
    t2 = cache.export(layer, 7)
    K, V = sk.kv_layer(w, wl, 0, ctx, "cpu")
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            u = build_unit(K[b, g].numpy(), V[b, g].numpy(), fp16_meta)
            np.testing.assert_array_equal(kc[b, g], u["kcodes"])
            np.testing.assert_array_equal(ks[b, g], u["kscale"])
            np.testing.assert_array_equal(vc[b, g], pack_int4(u["vcodes"]))
            np.testing.assert_array_equal(vm[b, g, ..., 0], u["vscale"])
            np.testing.assert_array_equal(vm[b, g, ..., 1], u["voffset"])
            np.testing.assert_array_equal(eta[b, g], u["eta"])
            np.testing.assert_array_equal(vr[b, g, 0], u["vmin"])
            np.testing.assert_array_equal(vr[b, g, 1], u["vmax"])
            r = u["r"]
            np.testing.assert_array_equal(res[b, g, 0], K[b, g, ctx - r:].numpy())
            np.testing.assert_array_equal(res[b, g, 1], V[b, g, ctx - r:].numpy())
            np.testing.assert_array_equal(t2[b, g, 0], K[b, g].numpy())
            np.testing.assert_array_equal(t2[b, g, 1], V[b, g].numpy())


@pytest.mark.parametrize("chunks", [None, [1, 63, 64, 100, 1, 700]])
def test_append_tiny_bit_exact(cqa, chunks):
    w = sk.WORKLOADS["tiny"]
    ctx = w.ctx + 37
    with cqa.Cache(1, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, ctx) as cache:
        fill_cache(cache, w, [0], ctx, chunks=chunks)
        assert cache.length(0) == ctx
        _check_unit_arrays(cache, 0, w, 0, ctx)


@pytest.mark.parametrize("name,ctx", [("llama8b_8k_1layer", 8192 + 45),
                                      ("llama8b_64k_b4_t3values", 4096 + 64)])
def test_append_d128_bit_exact(cqa, name, ctx):
    w = sk.WORKLOADS[name]
    with cqa.Cache(1, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, ctx) as cache:
        fill_cache(cache, w, [0], ctx, chunks=[500, 3000, 17])
        _check_unit_arrays(cache, 0, w, 0, ctx)


@pytest.mark.parametrize("name,ctx,chunks", [("tiny", 1024 + 37, [1, 63, 64, 100, 1, 700]),
                                             ("llama8b_8k_1layer", 4096 + 45, None),
                                             ("llama8b_64k_b4_t3values", 2048 + 64, [500, 17])])
def test_append_fp16_meta_bit_exact(cqa, name, ctx, chunks):
    """Binary16 metadata: scales rounded up, codes taken against them, offsets exact."""
    w = sk.WORKLOADS[name]
    with cqa.Cache(1, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, ctx,
                   meta_fp16=True) as cache:
        fill_cache(cache, w, [0], ctx, chunks=chunks)
        _check_unit_arrays(cache, 0, w, 0, ctx, fp16_meta=True)


def test_append_errors(cqa):
    w = sk.WORKLOADS["tiny"]
    with cqa.Cache(2, 1, 4, 2, 64, 128) as cache:
        K, V = sk.kv_layer(w, 0, 0, 100, "cuda")
        cache.append(0, K, V)
        with pytest.raises(cqa.CqaError) as e:
            cache.append(0, K, V)  # 200 > 128
        assert e.value.code == -4
        assert cache.length(0) == 100
        with pytest.raises(cqa.CqaError) as e:
            cqa.cqa_quantize_append(cache.handle, 5, K, V)
        assert e.value.code == -1
        q = sk.queries(w, 0, 0, "cuda")
        with pytest.raises(cqa.CqaError) as e:
            cache.decode(1, q, cqa.Thresholds())  # empty layer
        assert e.value.code == -5
    with pytest.raises(cqa.CqaError):
        cqa.Cache(1, 1, 6, 4, 64, 128)  # 6 query heads over 4 kv heads
    with pytest.raises(cqa.CqaError):
        cqa.Cache(1, 1, 4, 2, 96, 128)  # unsupported head_dim


def test_bounded_wait_reports_instead_of_hanging(cqa):
    """Failure detection without a fault: a device wait that nothing completes
    gives up after its poll limit and the status word says so."""
    with cqa.Cache(1, 1, 4, 2, 64, 128) as cache:
        assert cache.device_status() == 0
        cqa.cqa_selftest_bounded_wait(cache.handle, 2000)
        assert cache.device_status() == 1  # read and cleared
        assert cache.device_status() == 0
        # the context stays usable
        w = sk.WORKLOADS["tiny"]
        K, V = sk.kv_layer(w, 0, 0, 100, "cuda")
        cache.append(0, K, V)
        out = cache.decode(0, sk.queries(w, 0, 0, "cuda"), cqa.Thresholds())[0]
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()


def test_allocation_failure_is_reported(cqa):
    """A cache far larger than the device reports CQA_ERR_OOM and leaves nothing behind."""
    with pytest.raises(cqa.CqaError) as e:
        cqa.Cache(4096, 64, 32, 8, 128, 8192)  # ~2 TB of Tier 1
    assert e.value.code == -3
    with cqa.Cache(1, 1, 4, 2, 64, 128) as cache:  # the device still works
        assert cache.device_status() == 0
