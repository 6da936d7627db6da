"""Python binding of libcqa.so: certified quantized KV-cache decode attention on B200.

Argument marshalling only.  Every step of the decode path runs in the CUDA
library; torch is used for device buffers and streams.  The functions carry
the names of the C entry points declared in include/cqa.h:

    cqa_cache_create, cqa_cache_destroy, cqa_cache_length,
    cqa_quantize_append, cqa_decode, cqa_dense_reference,
    cqa_debug_export, cqa_error_string

and ``Cache`` wraps a handle with the same calls as methods.  Importing this
module does not load the library; the first call does, and fails loudly if
libcqa.so has not been built (``python -m certified_quantized_kv_int8_b200.build``).
"""

from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, asdict

import numpy as np
import torch

from .build import LIB

__all__ = [
    "CqaError", "Thresholds", "Cache", "load_library",
    "cqa_cache_create", "cqa_cache_destroy", "cqa_cache_length", "cqa_cache_row_lengths",
    "cqa_quantize_append", "cqa_quantize_append_row", "cqa_decode", "cqa_dense_reference", "cqa_debug_export", "cqa_error_string",
    "cqa_profile_begin", "cqa_profile_end", "PHASES", "cqa_dense_attention_noalloc",
    "cqa_set_key_prefetch", "cqa_device_status",
    "EXPORT_KCODES", "EXPORT_KSCALE", "EXPORT_VCODES", "EXPORT_VMETA", "EXPORT_ETA",
    "EXPORT_VRANGE", "EXPORT_RESIDUAL", "EXPORT_TIER2",
]

EXPORT_KCODES, EXPORT_KSCALE, EXPORT_VCODES, EXPORT_VMETA = 0, 1, 2, 3
EXPORT_ETA, EXPORT_VRANGE, EXPORT_RESIDUAL, EXPORT_TIER2 = 4, 5, 6, 7

EXPORTED_SYMBOLS = (
    "cqa_cache_create", "cqa_cache_destroy", "cqa_cache_length", "cqa_cache_row_lengths",
    "cqa_quantize_append", "cqa_quantize_append_row", "cqa_decode", "cqa_dense_reference", "cqa_debug_export", "cqa_error_string",
    "cqa_profile_begin", "cqa_profile_end", "cqa_dense_attention_noalloc",
    "cqa_set_key_prefetch", "cqa_device_status", "cqa_selftest_bounded_wait",
    "cqa_test_inject_fault",
)

PHASES = ("append_seal", "append_tail", "score", "select", "promote", "decide", "dense_keys",
          "attend", "combine", "dense_attend", "dense_combine", "prefetch", "naive",
          "naive_combine", "promote_staged")


class _Config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("batch", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("max_ctx", ctypes.c_int32),
                ("device", ctypes.c_int32), ("meta_fp16", ctypes.c_int32)]


class _Thresholds(ctypes.Structure):
    _fields_ = [("tau_cov", ctypes.c_float), ("eps_key", ctypes.c_float),
                ("max_expand", ctypes.c_int32), ("v_tol", ctypes.c_float),
                ("rank_r", ctypes.c_int32), ("eps_val", ctypes.c_float),
                ("layer_dense_frac", ctypes.c_float), ("naive", ctypes.c_int32),
                ("rank_tol", ctypes.c_int32)]


class _Trace(ctypes.Structure):
    _fields_ = [("kstar", ctypes.c_void_p), ("block_flags", ctypes.c_void_p),
                ("ell8", ctypes.c_void_p), ("ell16", ctypes.c_void_p),
                ("delta", ctypes.c_void_p), ("head_flags", ctypes.c_void_p),
                ("ell_res", ctypes.c_void_p)]


@dataclass
class Thresholds:
    """Decode thresholds (see cqa_thresholds in include/cqa.h)."""

    tau_cov: float = 0.995
    eps_key: float = 5e-3
    max_expand: int = 4
    v_tol: float = 0.05
    rank_r: int = 8
    eps_val: float = float("inf")
    layer_dense_frac: float = 0.5
    naive: bool = False
    rank_tol: int = 2

    def as_c(self) -> _Thresholds:
        return _Thresholds(self.tau_cov, self.eps_key, int(self.max_expand), self.v_tol,
                           int(self.rank_r), self.eps_val, self.layer_dense_frac,
                           1 if self.naive else 0, int(self.rank_tol))

    def float32_rounded(self) -> dict:
        """The values the library sees (floats rounded to float32), as a dict."""
        d = asdict(self)
        for k in ("tau_cov", "eps_key", "v_tol", "eps_val", "layer_dense_frac"):
            d[k] = float(np.float32(d[k]))
        return d


class CqaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {cqa_error_string(code)} ({code})")


_lib = None


def load_library() -> ctypes.CDLL:
    """Load libcqa.so (built in-tree); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB):
        raise RuntimeError(
            f"{LIB} is missing: build it with `python -m certified_quantized_kv_int8_b200.build`")
    lib = ctypes.CDLL(LIB)
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    lib.cqa_cache_create.argtypes = [ctypes.POINTER(_Config), ctypes.POINTER(vp)]
    lib.cqa_cache_destroy.argtypes = [vp]
    lib.cqa_cache_length.argtypes = [vp, i32, ctypes.POINTER(ctypes.c_int32)]
    lib.cqa_cache_row_lengths.argtypes = [vp, i32, ctypes.POINTER(ctypes.c_int32)]
    lib.cqa_quantize_append.argtypes = [vp, i32, vp, vp, i32, vp]
    lib.cqa_quantize_append_row.argtypes = [vp, i32, i32, vp, vp, i32, vp]
    lib.cqa_decode.argtypes = [vp, i32, vp, ctypes.POINTER(_Thresholds), vp, vp, vp, vp,
                               ctypes.POINTER(_Trace), vp]
    lib.cqa_dense_reference.argtypes = [vp, i32, vp, vp, vp]
    lib.cqa_debug_export.argtypes = [vp, i32, i32, vp, ctypes.c_size_t]
    lib.cqa_debug_export.restype = ctypes.c_int64
    lib.cqa_profile_begin.argtypes = [vp, i32]
    lib.cqa_profile_end.argtypes = [vp, ctypes.POINTER(ctypes.c_double),
                                    ctypes.POINTER(ctypes.c_int64)]
    lib.cqa_dense_attention_noalloc.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, vp, vp]
    lib.cqa_set_key_prefetch.argtypes = [vp, i32, ctypes.c_float]
    lib.cqa_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
    lib.cqa_selftest_bounded_wait.argtypes = [vp, ctypes.c_int32]
    lib.cqa_test_inject_fault.argtypes = [i32, i32]
    lib.cqa_error_string.argtypes = [i32]
    lib.cqa_error_string.restype = ctypes.c_char_p
    for name in ("cqa_cache_create", "cqa_cache_destroy", "cqa_cache_length",
                 "cqa_cache_row_lengths", "cqa_quantize_append", "cqa_quantize_append_row",
                 "cqa_decode", "cqa_dense_reference",
                 "cqa_profile_begin", "cqa_profile_end", "cqa_dense_attention_noalloc",
                 "cqa_set_key_prefetch", "cqa_device_status", "cqa_selftest_bounded_wait",
                 "cqa_test_inject_fault"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _check(code: int, where: str):
    if code < 0:
        raise CqaError(code, where)
    return code


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t: torch.Tensor, dtype, shape, name):
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous() and tuple(t.shape) == tuple(shape)):
        raise ValueError(f"{name}: expected a contiguous {dtype} CUDA tensor of shape {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


def cqa_error_string(code: int) -> str:
    return load_library().cqa_error_string(int(code)).decode()


def cqa_cache_create(n_layers, batch, n_q_heads, n_kv_heads, head_dim, max_ctx, device=0,
                     meta_fp16=False):
    cfg = _Config(n_layers, batch, n_q_heads, n_kv_heads, head_dim, max_ctx, device,
                  1 if meta_fp16 else 0)
    h = ctypes.c_void_p()
    _check(load_library().cqa_cache_create(ctypes.byref(cfg), ctypes.byref(h)), "cqa_cache_create")
    return h


def cqa_cache_destroy(handle):
    return _check(load_library().cqa_cache_destroy(handle), "cqa_cache_destroy")


def cqa_cache_length(handle, layer: int) -> int:
    out = ctypes.c_int32()
    _check(load_library().cqa_cache_length(handle, layer, ctypes.byref(out)), "cqa_cache_length")
    return int(out.value)


def cqa_cache_row_lengths(handle, layer: int, batch: int) -> list:
    out = (ctypes.c_int32 * batch)()
    _check(load_library().cqa_cache_row_lengths(handle, layer, out), "cqa_cache_row_lengths")
    return [int(x) for x in out]


def cqa_quantize_append(handle, layer, k, v, stream=None):
    """k, v: CUDA float16 [batch][n_kv_heads][n_new][head_dim]."""
    n_new = int(k.shape[2])
    return _check(load_library().cqa_quantize_append(handle, layer, _ptr(k), _ptr(v), n_new,
                                                     _stream(stream)), "cqa_quantize_append")


def cqa_quantize_append_row(handle, layer, row, k, v, stream=None):
    """k, v: CUDA float16 [n_kv_heads][n_new][head_dim], appended to batch row `row`."""
    n_new = int(k.shape[1])
    return _check(load_library().cqa_quantize_append_row(handle, layer, row, _ptr(k), _ptr(v),
                                                         n_new, _stream(stream)),
                  "cqa_quantize_append_row")


def cqa_decode(handle, layer, q, th: Thresholds, out, e_key, e_val, rung, trace=None, stream=None):
    """q: CUDA float16 [batch][n_q_heads][head_dim]; out float32 like q; e_key, e_val float32
    [batch][n_q_heads]; rung uint8 [batch][n_q_heads].  trace: dict of CUDA tensors keyed by
    the cqa_trace field names (any subset)."""
    tr = None
    if trace:
        tr = _Trace(**{k: (v.data_ptr() if v is not None else None) for k, v in trace.items()})
    return _check(load_library().cqa_decode(
        handle, layer, _ptr(q), ctypes.byref(th.as_c()), _ptr(out), _ptr(e_key), _ptr(e_val),
        _ptr(rung), ctypes.byref(tr) if tr is not None else None, _stream(stream)), "cqa_decode")


def cqa_dense_reference(handle, layer, q, out, stream=None):
    return _check(load_library().cqa_dense_reference(handle, layer, _ptr(q), _ptr(out),
                                                     _stream(stream)), "cqa_dense_reference")


def cqa_debug_export(handle, layer, what, dst: np.ndarray | None = None):
    """Copy one Tier-1 array to a numpy buffer (synchronous); with dst None return its size."""
    lib = load_library()
    if dst is None:
        return _check(lib.cqa_debug_export(handle, layer, what, None, 0), "cqa_debug_export")
    return _check(lib.cqa_debug_export(handle, layer, what, dst.ctypes.data_as(ctypes.c_void_p),
                                       dst.nbytes), "cqa_debug_export")


def cqa_profile_begin(handle, max_launches: int = 1 << 16):
    return _check(load_library().cqa_profile_begin(handle, int(max_launches)), "cqa_profile_begin")


def cqa_profile_end(handle):
    """Returns ({phase: ms}, {phase: launches}, untimed launches)."""
    ms = (ctypes.c_double * len(PHASES))()
    n = (ctypes.c_int64 * len(PHASES))()
    untimed = _check(load_library().cqa_profile_end(handle, ms, n), "cqa_profile_end")
    return ({p: ms[i] for i, p in enumerate(PHASES)}, {p: int(n[i]) for i, p in enumerate(PHASES)},
            untimed)


def cqa_set_key_prefetch(handle, mode: int = 1, min_fraction: float = 0.75):
    """0 off, 1 adaptive (default), 2 always; see include/cqa.h."""
    return _check(load_library().cqa_set_key_prefetch(handle, int(mode), float(min_fraction)),
                  "cqa_set_key_prefetch")


def cqa_device_status(handle) -> int:
    """Synchronise and return (then clear) the device status word; 0 = all kernels normal."""
    out = ctypes.c_int32()
    _check(load_library().cqa_device_status(handle, ctypes.byref(out)), "cqa_device_status")
    return int(out.value)


def cqa_selftest_bounded_wait(handle, polls: int = 1000):
    """Launch a kernel whose bounded wait must give up (see include/cqa.h)."""
    return _check(load_library().cqa_selftest_bounded_wait(handle, int(polls)),
                  "cqa_selftest_bounded_wait")


FAULT_NONE, FAULT_PINNED_ALLOC, FAULT_PREFETCH_COPY = 0, 1, 2


def cqa_test_inject_fault(site: int, skip: int = 0):
    """Arm the library's host-side fault injection (a test hook, see cqa.h)."""
    _check(load_library().cqa_test_inject_fault(int(site), int(skip)), "cqa_test_inject_fault")


def cqa_dense_attention_noalloc(q, k, v, out, stream=None):
    """Exact attention over caller-held FP16 keys and values that allocates no
    device memory (for callers that cannot call cudaMalloc; see include/cqa.h).
    q: CUDA float16 [batch][n_q_heads][head_dim]; k, v: CUDA float16
    [batch][n_kv_heads][n_tokens][head_dim]; out: CUDA float32 like q."""
    B, Hq, d = q.shape
    _, Hkv, T, _ = k.shape
    _dev(q, torch.float16, (B, Hq, d), "q")
    _dev(k, torch.float16, (B, Hkv, T, d), "k")
    _dev(v, torch.float16, (B, Hkv, T, d), "v")
    _dev(out, torch.float32, (B, Hq, d), "out")
    return _check(load_library().cqa_dense_attention_noalloc(
        _ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, d, T, _ptr(out), _stream(stream)),
        "cqa_dense_attention_noalloc")


class Cache:
    """A cqa_cache handle with its shape; methods mirror the C entry points."""

    def __init__(self, n_layers, batch, n_q_heads, n_kv_heads, head_dim, max_ctx, device=0,
                 meta_fp16=False):
        self.n_layers, self.batch = n_layers, batch
        self.n_q_heads, self.n_kv_heads, self.head_dim = n_q_heads, n_kv_heads, head_dim
        self.max_ctx, self.device, self.meta_fp16 = max_ctx, device, bool(meta_fp16)
        self.handle = cqa_cache_create(n_layers, batch, n_q_heads, n_kv_heads, head_dim,
                                       max_ctx, device, meta_fp16)

    def close(self):
        # cqa_cache_destroy frees everything even when it reports an error (a
        # failed device synchronisation), so the handle is dropped first: a
        # second close, or __del__ after a raising close, must not free it again
        h, self.handle = self.handle, None
        if h is not None and h.value:
            cqa_cache_destroy(h)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def device_status(self) -> int:
        return cqa_device_status(self.handle)

    def set_key_prefetch(self, mode: int = 1, min_fraction: float = 0.75):
        return cqa_set_key_prefetch(self.handle, mode, min_fraction)

    def profile_begin(self, max_launches: int = 1 << 16):
        return cqa_profile_begin(self.handle, max_launches)

    def profile_end(self):
        return cqa_profile_end(self.handle)

    def length(self, layer):
        """Tokens of the layer's longest batch row."""
        return cqa_cache_length(self.handle, layer)

    def row_lengths(self, layer):
        return cqa_cache_row_lengths(self.handle, layer, self.batch)

    def append(self, layer, k, v, stream=None):
        B, H, d = self.batch, self.n_kv_heads, self.head_dim
        _dev(k, torch.float16, (B, H, k.shape[2], d), "k")
        _dev(v, torch.float16, (B, H, k.shape[2], d), "v")
        return cqa_quantize_append(self.handle, layer, k, v, stream)

    def append_row(self, layer, row, k, v, stream=None):
        H, d = self.n_kv_heads, self.head_dim
        _dev(k, torch.float16, (H, k.shape[1], d), "k")
        _dev(v, torch.float16, (H, k.shape[1], d), "v")
        return cqa_quantize_append_row(self.handle, layer, row, k, v, stream)

    def alloc_outputs(self):
        dev = torch.device("cuda", self.device)
        B, Hq, d = self.batch, self.n_q_heads, self.head_dim
        return (torch.empty(B, Hq, d, dtype=torch.float32, device=dev),
                torch.empty(B, Hq, dtype=torch.float32, device=dev),
                torch.empty(B, Hq, dtype=torch.float32, device=dev),
                torch.empty(B, Hq, dtype=torch.uint8, device=dev))

    def alloc_trace(self, layer):
        dev = torch.device("cuda", self.device)
        B, Hq, Hkv = self.batch, self.n_q_heads, self.n_kv_heads
        nb = max(1, self.length(layer) // 64)
        return dict(
            kstar=torch.empty(B, Hq, dtype=torch.int32, device=dev),
            block_flags=torch.empty(B, Hkv, nb, dtype=torch.uint8, device=dev),
            ell8=torch.empty(B, Hq, nb, dtype=torch.float32, device=dev),
            ell16=torch.full((B, Hq, nb), math.nan, dtype=torch.float32, device=dev),
            delta=torch.empty(B, Hq, nb, dtype=torch.float32, device=dev),
            head_flags=torch.empty(B, Hq, dtype=torch.uint8, device=dev),
            ell_res=torch.empty(B, Hq, dtype=torch.float32, device=dev),
        )

    def decode(self, layer, q, th: Thresholds, outputs=None, trace=None, stream=None):
        B, Hq, d = self.batch, self.n_q_heads, self.head_dim
        _dev(q, torch.float16, (B, Hq, d), "q")
        out, e_key, e_val, rung = outputs if outputs is not None else self.alloc_outputs()
        cqa_decode(self.handle, layer, q, th, out, e_key, e_val, rung, trace, stream)
        return out, e_key, e_val, rung

    def dense_reference(self, layer, q, out=None, stream=None):
        B, Hq, d = self.batch, self.n_q_heads, self.head_dim
        _dev(q, torch.float16, (B, Hq, d), "q")
        if out is None:
            out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
        cqa_dense_reference(self.handle, layer, q, out, stream)
        return out

    def export(self, layer, what):
        """Tier-1 array of `layer` as a numpy array shaped per include/cqa.h; when the
        rows' extents differ (a ragged layer), a list of per-row arrays (each
        without the batch axis)."""
        H, d = self.n_kv_heads, self.head_dim
        lens = self.row_lengths(layer)

        def spec(T):
            nb, r = T // 64, T % 64
            return {
                EXPORT_KCODES: (np.int8, (H, nb, 64, d)),
                EXPORT_KSCALE: (np.float32, (H, nb, d)),
                EXPORT_VCODES: (np.uint8, (H, nb, 64, d // 2)),
                EXPORT_VMETA: (np.float32, (H, nb, 64, d // 32, 2)),
                EXPORT_ETA: (np.float32, (H, nb)),
                EXPORT_VRANGE: (np.float32, (H, 2, d)),
                EXPORT_RESIDUAL: (np.float16, (H, 2, r, d)),
                EXPORT_TIER2: (np.float16, (H, 2, T, d)),
            }[what]

        specs = [spec(T) for T in lens]
        sizes = [int(np.prod(sh)) * np.dtype(dt).itemsize for dt, sh in specs]
        flat = np.empty(sum(sizes), dtype=np.uint8)
        n = cqa_debug_export(self.handle, layer, what, flat)
        assert n == flat.nbytes
        rows, off = [], 0
        for (dt, sh), size in zip(specs, sizes):
            rows.append(flat[off:off + size].view(dt).reshape(sh))
            off += size
        if len({sh for _, sh in specs}) == 1:  # equal shapes: one array
            return np.stack(rows)
        return rows
