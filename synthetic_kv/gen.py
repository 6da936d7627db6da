"""Counter-based generator for the synthetic decode-attention workloads.

Every value is a pure function of (workload seed, stream, layer, batch row,
head, token, channel): a 32-bit integer hash of that counter picks one of
2^16 equiprobable quantiles of the target distribution.  Hashing uses only
integer shifts, xors, masks and products below 2^63, and the remaining float
steps are single IEEE-rounded float64 operations followed by float64 ->
float32 -> float16 round-to-nearest-even, so the CPU and a CUDA device give
the same bits.  Nothing here computes any part of the attention method.

Workload shapes follow the LLaMA-3.1-8B evaluation of *Runtime-Certified
Bounded-Error Quantized Attention* (Experimental results: LLaMA 3.1-8B at
8K, 32K, 64K and 128K context); the distributions (N(0,1) keys with scaled
outlier channels, a linear key drift, Student-t values, a planted needle with
near-tie blocks) are synthetic stand-ins for its PG-19 / NIAH / RULER runs.
"""

from __future__ import annotations

import functools
import math
from dataclasses import dataclass, field

import numpy as np
import torch

M32 = 0xFFFFFFFF
_MUL = 0x45D9F3B  # < 2^27, so every product of a 32-bit word stays below 2^59

BLOCK = 64  # tokens per KV block (fixed by the cache layout)

# stream ids: one independent counter space per kind of draw
S_K, S_V, S_Q, S_OUTLIER, S_DRIFT, S_NEEDLE, S_TIE_BASE, S_TIE_JITTER = range(8)


def hash32(x):
    """Integer mixing hash on int64 arrays (numpy or torch) holding 32-bit words."""
    x = (((x >> 16) ^ x) * _MUL) & M32
    x = (((x >> 16) ^ x) * _MUL) & M32
    return (x >> 16) ^ x


def _hash_py(x: int) -> int:
    x &= M32
    x = (((x >> 16) ^ x) * _MUL) & M32
    x = (((x >> 16) ^ x) * _MUL) & M32
    return ((x >> 16) ^ x) & M32


def _key(*parts: int) -> int:
    h = 0x2545F491
    for p in parts:
        h = _hash_py(h ^ _hash_py(int(p) & M32))
        h = _hash_py(h + 0x9E37)
    return h


@functools.lru_cache(maxsize=None)
def _tables_cpu():
    """2^16 equiprobable quantiles of N(0,1) and of Student-t(3), float32."""
    from scipy.special import ndtri
    from scipy.stats import t as student_t

    u = (np.arange(1 << 16, dtype=np.float64) + 0.5) / float(1 << 16)
    normal = ndtri(u).astype(np.float32)
    t3 = student_t.ppf(u, 3).astype(np.float32)
    return torch.from_numpy(normal), torch.from_numpy(t3)


_DEV_TABLES: dict = {}


def _tables(device):
    device = torch.device(device)
    key = str(device)
    if key not in _DEV_TABLES:
        n, t = _tables_cpu()
        _DEV_TABLES[key] = (n.to(device), t.to(device))
    return _DEV_TABLES[key]


def _draw(device, key: int, idx: torch.Tensor, dist: str) -> torch.Tensor:
    """float32 draws for counters idx (int64 tensor) in stream `key`."""
    k1 = key & M32
    k2 = _hash_py(key ^ 0x5BD1E995)
    h = hash32((idx ^ k1) & M32)
    h = hash32((h + k2) & M32)
    normal, t3 = _tables(device)
    table = normal if dist == "normal" else t3
    return table[(h >> 16) & 0xFFFF]


@dataclass(frozen=True)
class Workload:
    """One synthetic decode-attention workload (shapes of one model layer stack)."""

    name: str
    n_layers: int
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ctx: int  # tokens already in the cache when timing starts
    n_outlier: int  # key channels per kv head scaled by outlier_mult
    outlier_mult: float
    value_dist: str = "normal"  # "normal" or "student_t3"
    drift_beta: float = 0.0  # k_t += beta * (t / ctx) * u, u ~ N(0, I) per kv head
    appends: int = 0  # decode steps that append one token per layer before decoding
    needle: bool = False
    seed: int = 0
    # planted structure (needle workloads only)
    needle_depth: float = 0.37
    needle_logit: float = 6.0
    n_ties: int = 16
    tie_logit: float = 6.0
    tie_jitter: float = 0.02
    tie_layer_all: int = 17  # layer whose every kv group gets near-tie blocks
    row_ctx: tuple = ()  # ragged batch: tokens of each batch row (ctx = the longest)
    extra: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def max_ctx(self) -> int:
        return self.ctx + self.appends


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 4, 2, 64, 1024, 2, 8.0),
    "llama8b_8k_1layer": Workload("llama8b_8k_1layer", 1, 1, 32, 8, 128, 8192, 4, 10.0),
    "llama8b_32k_32layer_append": Workload(
        "llama8b_32k_32layer_append", 32, 1, 32, 8, 128, 32768, 4, 10.0,
        drift_beta=1.0, appends=64),
    "llama8b_64k_b4_t3values": Workload(
        "llama8b_64k_b4_t3values", 32, 4, 32, 8, 128, 65536, 4, 10.0,
        value_dist="student_t3"),
    "llama8b_128k_needle": Workload(
        "llama8b_128k_needle", 32, 1, 32, 8, 128, 131072, 4, 10.0, needle=True),
    # a ragged batch: four rows of different lengths, the longest 32K
    "llama8b_ragged_b4": Workload(
        "llama8b_ragged_b4", 32, 4, 32, 8, 128, 32768, 4, 10.0,
        row_ctx=(32768, 4096 + 37, 16384 + 5, 8192)),
}


def row_lengths(w: Workload) -> list[int]:
    """Tokens of each batch row when timing starts."""
    return list(w.row_ctx) if w.row_ctx else [w.ctx] * w.batch


def default_thresholds(w: Workload) -> dict:
    """Runtime thresholds for a workload.  Only tau_cov and v_tol are named by the
    method; the others are this implementation's choices (all are plain inputs)."""
    th = dict(tau_cov=0.995, eps_key=5e-3, eps_val=float("inf"), v_tol=0.05,
              rank_r=8, rank_tol=2, max_expand=4, layer_dense_frac=0.5)
    if w.value_dist == "student_t3":
        th["v_tol"] = 5e-3
    return th


def outlier_channels(w: Workload, layer: int, b: int, kvh: int) -> list[int]:
    """The w.n_outlier key channels of this kv head that carry the outlier scale."""
    key = _key(w.seed, S_OUTLIER, layer, b, kvh)
    scores = [(_hash_py(c ^ key), c) for c in range(w.head_dim)]
    scores.sort()
    return sorted(c for _, c in scores[: w.n_outlier])


def plant_positions(w: Workload, nb: int) -> tuple[int, list[int]]:
    """Block indices of the needle and of the near-tie blocks (needle workloads)."""
    needle = int(w.needle_depth * nb)
    ties = []
    for i in range(w.n_ties):
        j = int((0.05 + 0.9 * i / max(1, w.n_ties)) * nb)
        while j == needle or j in ties:
            j += 1
        ties.append(j)
    return needle, ties


def _tie_groups(w: Workload, layer: int) -> list[int]:
    if not w.needle:
        return []
    if layer == w.tie_layer_all:
        return list(range(w.n_kv_heads))
    return [layer % w.n_kv_heads]


def queries(w: Workload, layer: int, step: int, device="cpu") -> torch.Tensor:
    """q for one decode step: float16 [batch][n_q_heads][head_dim], N(0,1).
    Needle workloads keep q fixed per (layer, head) across steps."""
    s = 0 if w.needle else step
    out = torch.empty(w.batch, w.n_q_heads, w.head_dim, dtype=torch.float16, device=device)
    idx = torch.arange(w.n_q_heads * w.head_dim, dtype=torch.int64, device=device)
    for b in range(w.batch):
        key = _key(w.seed, S_Q, layer, b, s)
        out[b] = _draw(device, key, idx, "normal").reshape(w.n_q_heads, w.head_dim).half()
    return out


def _group_mean_q(w: Workload, layer: int, b: int, kvh: int) -> tuple[torch.Tensor, float]:
    """Mean query of one GQA group and its squared norm, both computed on the CPU
    (a fixed summation order) so that every device plants the same keys."""
    q = queries(w, layer, 0, "cpu")[b].double()
    g = w.group
    qbar = q[kvh * g:(kvh + 1) * g].mean(0)
    return qbar, float((qbar * qbar).sum())


def kv_unit(w: Workload, layer: int, b: int, kvh: int, t0: int, t1: int,
            device="cpu") -> tuple[torch.Tensor, torch.Tensor]:
    """FP16 keys and values of one (layer, batch row, kv head) for tokens [t0, t1):
    two float16 tensors [t1 - t0][head_dim] on `device`."""
    d = w.head_dim
    n = t1 - t0
    t = torch.arange(t0, t1, dtype=torch.int64, device=device)
    c = torch.arange(d, dtype=torch.int64, device=device)
    idx = (t[:, None] * d + c[None, :]).reshape(-1)

    z = _draw(device, _key(w.seed, S_K, layer, b, kvh), idx, "normal").reshape(n, d)
    mult = torch.ones(d, dtype=torch.float64, device=device)
    for ch in outlier_channels(w, layer, b, kvh):
        mult[ch] = w.outlier_mult
    k64 = z.double() * mult[None, :]
    if w.drift_beta != 0.0:
        u = _draw(device, _key(w.seed, S_DRIFT, layer, b, kvh), c, "normal").double()
        ramp = w.drift_beta * (t.double() / float(w.ctx))
        k64 = k64 + ramp[:, None] * u[None, :]
    k = k64.float().half()

    vdist = "normal" if w.value_dist == "normal" else "t3"
    v = _draw(device, _key(w.seed, S_V, layer, b, kvh), idx, vdist).reshape(n, d).half()

    if w.needle:
        k = _plant(w, layer, b, kvh, t0, t1, k, device)
    return k, v


def _plant(w, layer, b, kvh, t0, t1, k, device):
    nb = w.ctx // BLOCK
    needle, ties = plant_positions(w, nb)
    d = w.head_dim
    sigma = 1.0 / math.sqrt(d)
    qbar = None

    def block_rows(j):
        lo, hi = max(t0, j * BLOCK), min(t1, (j + 1) * BLOCK)
        return lo, hi

    def noise(stream, j, lo, hi, extra=0):
        tt = torch.arange(lo, hi, dtype=torch.int64, device=device) - j * BLOCK
        cc = torch.arange(d, dtype=torch.int64, device=device)
        idx = (tt[:, None] * d + cc[None, :]).reshape(-1)
        key = _key(w.seed, stream, layer, b, kvh, extra)
        return _draw(device, key, idx, "normal").reshape(hi - lo, d).double()

    lo, hi = block_rows(needle)
    if lo < hi:
        qbar, qn2 = _group_mean_q(w, layer, b, kvh)
        qbar = qbar.to(device)
        cn = w.needle_logit / (sigma * qn2)
        val = cn * qbar[None, :] + 0.01 * noise(S_NEEDLE, needle, lo, hi)
        k[lo - t0:hi - t0] = val.float().half()
    if kvh in _tie_groups(w, layer):
        for i, j in enumerate(ties):
            lo, hi = block_rows(j)
            if lo >= hi:
                continue
            if qbar is None:
                qbar, qn2 = _group_mean_q(w, layer, b, kvh)
                qbar = qbar.to(device)
            ct = w.tie_logit / (sigma * qn2)
            # all tie blocks share one base pattern; a small per-block jitter
            # separates their exact block masses by far less than INT8 noise
            base = noise(S_TIE_BASE, 0, lo - j * BLOCK, hi - j * BLOCK)
            jit = noise(S_TIE_JITTER, 0, lo - j * BLOCK, hi - j * BLOCK, extra=i)
            val = ct * qbar[None, :] + 0.3 * base + w.tie_jitter * jit
            k[lo - t0:hi - t0] = val.float().half()
    return k


def kv_row(w: Workload, layer: int, b: int, t0: int, t1: int, device="cpu"):
    """Keys and values of one batch row: float16 [n_kv_heads][t1 - t0][head_dim]."""
    ks, vs = zip(*(kv_unit(w, layer, b, g, t0, t1, device) for g in range(w.n_kv_heads)))
    return torch.stack(ks).contiguous(), torch.stack(vs).contiguous()


def kv_layer(w: Workload, layer: int, t0: int, t1: int, device="cpu"):
    """Keys and values of a whole layer: float16 [batch][n_kv_heads][t1 - t0][head_dim]."""
    n = t1 - t0
    K = torch.empty(w.batch, w.n_kv_heads, n, w.head_dim, dtype=torch.float16, device=device)
    V = torch.empty_like(K)
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            K[b, g], V[b, g] = kv_unit(w, layer, b, g, t0, t1, device)
    return K, V
