"""cqa_dense_attention_noalloc, the entry point that allocates nothing.

Some callers cannot call cudaMalloc: hosts whose only device allocator belongs
to another framework under a fixed memory budget, and latency-critical paths
that must not synchronise on the allocator.  This entry point serves them with
its scratch in a fixed device array.  It must give the same exact attention as
cqa_dense_reference (and as the oracle's dense attention), call after call,
while sharing that one array, for every supported head shape; and it must
refuse shapes whose scratch would not fit, before launching anything.

This file is collected last, so a run that stops at its first failure has run
every other test before it.
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


def _two_calls(cqa, w, ctx, check_oracle):
    from oracle import dense_attention
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
            if check_oracle:
                qc, Kc, Vc = q.cpu().numpy(), K.cpu().numpy(), V.cpu().numpy()
                G = w.group
                for b in range(w.batch):
                    for h in range(w.n_q_heads):
                        want = dense_attention(qc[b, h:h + 1], Kc[b, h // G], Vc[b, h // G])[0]
                        assert float(np.abs(o[b, h] - want).max()) <= OUT_TOL, \
                            f"call {call} row {b} head {h} against the oracle"


@pytest.mark.parametrize("name,ctx", [("tiny", 1024 + 19), ("llama8b_8k_1layer", 8192 + 5)])
def test_noalloc_matches_dense_reference_on_two_calls(cqa, name, ctx):
    _two_calls(cqa, sk.WORKLOADS[name], ctx, check_oracle=(name == "tiny"))


@pytest.mark.parametrize("d,hq,hkv", [(128, 4, 4), (128, 4, 2), (128, 8, 2), (128, 16, 2),
                                      (64, 2, 2), (64, 4, 2), (64, 8, 2)])
def test_noalloc_every_head_shape(cqa, d, hq, hkv):
    """Every supported (head_dim, query heads per kv head) pair: G = 1, 2, 4, 8 at
    head_dim 128 and G = 1, 2, 4 at head_dim 64, with a ragged last block."""
    import dataclasses
    w = dataclasses.replace(sk.WORKLOADS["tiny"], name=f"noalloc{d}_{hq}_{hkv}", batch=2,
                            n_q_heads=hq, n_kv_heads=hkv, head_dim=d, n_outlier=2)
    _two_calls(cqa, w, 5 * 64 + 23, check_oracle=True)


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
    # unsupported head shapes: G = 8 at head_dim 64, G = 3, head_dim 96
    o = ctypes.c_void_p(out.data_ptr())
    assert lib.cqa_dense_attention_noalloc(p, p, p, 1, 8, 1, 64, 64, o, None) == -1
    assert lib.cqa_dense_attention_noalloc(p, p, p, 1, 3, 1, 128, 64, o, None) == -1
    assert lib.cqa_dense_attention_noalloc(p, p, p, 1, 1, 1, 96, 64, o, None) == -1
    torch.cuda.synchronize()
