"""Host-side fault injection: the library's error paths run without faulting a GPU.

A test hook in libcqa (cqa_test_inject_fault) makes one pinned host allocation
or one key-prefetch copy report failure on the host.  The recovery the method
promises (Key Contributions: deterministic recovery) needs these paths to
leave nothing behind: a failed cache creation frees what it had allocated,
and a decode whose copy fails returns an error before launching anything, so
the caller's outputs keep their contents.
"""

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
    yield m
    m.cqa_test_inject_fault(m.FAULT_NONE)


@pytest.mark.parametrize("skip", [0, 1, 2])
def test_failed_pinned_allocation_reports_oom_and_leaks_nothing(cqa, skip):
    """Each of the three pinned allocations of cqa_cache_create failing in turn."""
    w = sk.WORKLOADS["llama8b_8k_1layer"]
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    cqa.cqa_test_inject_fault(cqa.FAULT_PINNED_ALLOC, skip)
    with pytest.raises(cqa.CqaError) as ei:
        cqa.cqa_cache_create(2, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, 8192)
    assert ei.value.code == -3  # CQA_ERR_OOM
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0, "device memory of the failed create leaked"
    # disarmed after firing: the next create succeeds and works
    with cqa.Cache(1, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, 1024) as cache:
        fill_cache(cache, w, [0], 1024)
        out = cache.dense_reference(0, sk.queries(w, 0, 0, "cuda"))
        torch.cuda.synchronize()
        assert np.all(np.isfinite(out.cpu().numpy()))


@pytest.mark.parametrize("skip", [0, 1])
def test_failed_prefetch_copy_leaves_outputs_untouched(cqa, skip):
    """skip 0: the copy of the decoded layer's keys fails; skip 1: the copy of the
    next layer's keys, issued by the same call, fails."""
    w = sk.WORKLOADS["llama8b_8k_1layer"]
    ctx = 4096 + 7
    th = cqa.Thresholds(**sk.default_thresholds(w))
    with cqa.Cache(2, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, ctx) as cache:
        cache.set_key_prefetch(2)  # always stage: every decode issues the copies
        fill_cache(cache, w, [0, 1], ctx)
        q = sk.queries(w, 0, 0, "cuda")
        outs = cache.alloc_outputs()
        for t in outs[:3]:
            t.fill_(float("nan"))
        outs[3].fill_(255)
        cqa.cqa_test_inject_fault(cqa.FAULT_PREFETCH_COPY, skip)
        with pytest.raises(cqa.CqaError) as ei:
            cache.decode(0, q, th, outputs=outs)
        assert ei.value.code == -2  # CQA_ERR_CUDA
        torch.cuda.synchronize()
        for t in outs[:3]:
            assert torch.isnan(t).all(), "a failed decode wrote an output"
        assert (outs[3] == 255).all()
        assert cache.device_status() == 0
        # the next decode (the hook disarmed itself) stages again and agrees with a
        # decode that reads the keys from Tier 2 directly
        good = [x.cpu().numpy() for x in cache.decode(0, q, th)]
        cache.set_key_prefetch(0)
        plain = [x.cpu().numpy() for x in cache.decode(0, q, th)]
        torch.cuda.synchronize()
        for a, b in zip(good, plain):
            assert np.array_equal(a, b)


def test_inject_fault_rejects_bad_arguments(cqa):
    lib = cqa.load_library()
    assert lib.cqa_test_inject_fault(3, 0) == -1
    assert lib.cqa_test_inject_fault(1, -1) == -1
    assert lib.cqa_test_inject_fault(0, 0) == 0
