"""cqa_dense_attention_noalloc, the entry point that allocates nothing.

Some callers cannot call cudaMalloc: code running while a stream is captured
into a CUDA graph, hosts whose only allocator belongs to another framework,
latency-critical paths that must not synchronise on the allocator.  This entry
point serves them with its scratch in a fixed device array.  It must give the
same exact attention as cqa_dense_reference, call after call, while sharing
that one array; and it must refuse shapes whose scratch would not fit, before
launching anything.
"""

import ctypes

import numpy as np
import pytest
import torch

import synthetic_kv as sk

pytestmark = pytest.mark.gpu

OUT_TOL = 2e-3  # the max-abs output tolerance of the other parity tests


@pytest.fixture(scope="module")
def cqa():
    import certified_quantized_kv_int8_b200 as m
    from certified_quantized_kv_int8_b200.build import build
    build()
    m.load_library()
    return m


@pytest.mark.parametrize("name,ctx", [("tiny", 1024 + 19), ("llama8b_8k_1layer", 8192 + 5)])
def test_noalloc_matches_dense_reference_on_two_calls(cqa, name, ctx):
    w = sk.WORKLOADS[name]
    K, V = sk.kv_layer(w, 0, 0, ctx, device="cuda")
    with cqa.Cache(1, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, ctx) as cache:
        cache.append(0, K, V)
        for call in range(2):
            q = sk.queries(w, 0, call, device="cuda")
            ref = cache.dense_reference(0, q)
            out = torch.full((w.batch, w.n_q_heads, w.head_dim), float("nan"),
                             dtype=torch.float32, device="cuda")
            cqa.cqa_dense_attention_noalloc(q, K, V, out)
            torch.cuda.synchronize()
            o, r = out.cpu().numpy(), ref.cpu().numpy()
            assert np.all(np.isfinite(o))
            assert float(np.abs(o - r).max()) <= OUT_TOL, f"call {call}"


def test_noalloc_rejects_shapes_beyond_its_scratch(cqa):
    lib = cqa.load_library()
    small = torch.zeros(64, dtype=torch.float16, device="cuda")
    out = torch.zeros(64, dtype=torch.float32, device="cuda")
    p = ctypes.c_void_p(small.data_ptr())
    # 9000 kv heads x (128 + 3) floats of partials exceed the 4 MiB array; the
    # shape check refuses the call before any pointer is dereferenced
    rc = lib.cqa_dense_attention_noalloc(p, p, p, 9000, 1, 1, 128, 64,
                                         ctypes.c_void_p(out.data_ptr()), None)
    assert rc == -4
    assert "capacity" in cqa.cqa_error_string(rc)
    torch.cuda.synchronize()
