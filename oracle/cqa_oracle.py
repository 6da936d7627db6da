"""Plain numpy restatement of runtime-certified bounded-error quantized decode attention.

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the
library.  Floating point is float64 except where a quantity decides an integer
or is stored as a float32 annotation (scales, codes, offsets, eta_b); those
steps use single IEEE float32 operations, one rounding each, in the order
written, so that a float32 implementation can reproduce them bit for bit.

Source: *Runtime-Certified Bounded-Error Quantized Attention* (gist.science
summary of paper 2605.20868), technical summary:
  - Methodology §1 "Tiered storage with deterministic fallback": Tier 1 holds
    per-channel INT8 keys, per-group INT4 values, scales/offsets and per-block
    error annotations; Tier 2 holds the FP16 originals in pinned host RAM.
  - Methodology §2 "Two-term error decomposition": E_key, a total-variation
    bound driven by the per-token score perturbation Delta; E_val, the
    attention-mass-weighted sum of per-block reconstruction errors eta_b;
    both computed online from scales, query norms and value ranges.
  - Methodology §3 "Adaptive precision and fallback ladder": an INT8 scoring
    pass estimates block masses, the top-K* blocks covering tau_cov are
    promoted to FP16 keys, a rank-consistency check compares INT8 and FP16
    block rankings over the promoted blocks, and a four-rung ladder (widen
    coverage, FP16 values, per-head dense, whole-layer dense) ends in the
    exact dense output O_dense.

The pages give no formulas.  Each function states the reading it implements.
Parity pins: every function here is checked by tests/test_oracle_*.py against
closed forms, brute force or hand-worked fixtures, except the rank-consistency
rule and the whole-layer trigger, whose exact form the pages leave open
(parity unpinned: GPU and oracle are held to the same stated rule).
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

BLOCK = 64  # tokens per KV block
VGROUP = 32  # channels per INT4 value group
F32 = np.float32


# ---------------------------------------------------------------------------
# Tier 1 encoding (Methodology §1)
# ---------------------------------------------------------------------------

def fp16_round_up(x: np.ndarray) -> np.ndarray:
    """The smallest IEEE binary16 value >= x, for float32 0 <= x <= 65504, returned
    as float32: round to nearest, then one step up when that fell below x."""
    h = np.asarray(x, F32).astype(np.float16)
    low = h.astype(F32) < x
    h[low] = np.nextafter(h[low], np.float16(np.inf))
    return h.astype(F32)


def quantize_keys_block(k16: np.ndarray, fp16_meta: bool = False):
    """Per-channel symmetric INT8 keys for one block (Methodology §1).

    Reading: one scale per (block, channel) over the block's tokens,
    s = amax / 127 (float32), code = clamp(round_half_even(k / s), -127, 127);
    an all-zero channel gets s = 0 and codes 0.  Dequantised key = code * s.

    fp16_meta: the scale is stored as binary16, rounded up (the smallest fp16
    >= amax / 127), and the codes are taken against that stored scale.  Then
    |k / s| <= 127 still (no code is clamped) and |k - code * s| <= s / 2 for
    the stored s, so Delta computed from the stored scales stays a valid
    per-token perturbation bound.

    k16: float16 [BLOCK, d].  Returns (codes int8 [BLOCK, d], scale float32 [d]).
    """
    k = k16.astype(F32)
    amax = np.max(np.abs(k), axis=0)
    scale = (amax / F32(127.0)).astype(F32)
    if fp16_meta:
        scale = fp16_round_up(scale)
    ratio = np.zeros_like(k)
    nz = scale > 0
    ratio[:, nz] = k[:, nz] / scale[nz]
    codes = np.clip(np.rint(ratio), -127, 127).astype(np.int8)
    return codes, scale


def quantize_values_block(v16: np.ndarray, fp16_meta: bool = False):
    """Per-group asymmetric INT4 values for one block, with its error annotation.

    Reading (Methodology §1, "per-group INT4 values ... scales/offsets ...
    per-block error annotations"): groups are VGROUP consecutive channels of
    one token; offset z = group min, scale s = (max - min) / 15 (float32),
    code = clamp(round_half_even((v - z) / s), 0, 15), or 0 when s = 0;
    reconstruction v_hat = (s * code) + z with one float32 rounding per
    operation; eta_b = max over the block of |v - v_hat| (float32), the
    measured reconstruction error written when the originals are at hand.

    fp16_meta: offset and scale are stored as binary16.  The offset, the min of
    binary16 values, is one of them and stays exact; the scale is rounded up
    (the smallest fp16 >= (max - min) / 15), so (v - z) / s <= 15 and no code is
    clamped; v_hat and eta_b use the stored values, so eta_b still bounds
    |v - v_hat| exactly as measured.

    v16: float16 [BLOCK, d].  Returns (codes uint8 [BLOCK, d] unpacked,
    scale float32 [BLOCK, d/VGROUP], offset float32 [BLOCK, d/VGROUP],
    v_hat float32 [BLOCK, d], eta float32 scalar).
    """
    n, d = v16.shape
    v = v16.astype(F32).reshape(n, d // VGROUP, VGROUP)
    lo = v.min(axis=2)
    hi = v.max(axis=2)
    scale = ((hi - lo).astype(F32) / F32(15.0)).astype(F32)
    if fp16_meta:
        scale = fp16_round_up(scale)
    diff = (v - lo[:, :, None]).astype(F32)
    ratio = np.zeros_like(v)
    nz = scale > 0
    ratio[nz] = diff[nz] / scale[nz][:, None]
    codes = np.clip(np.rint(ratio), 0, 15).astype(np.uint8)
    v_hat = ((scale[:, :, None] * codes.astype(F32)).astype(F32) + lo[:, :, None]).astype(F32)
    eta = F32(np.max(np.abs((v - v_hat).astype(F32))))
    return codes.reshape(n, d), scale, lo, v_hat.reshape(n, d), eta


def pack_int4(codes: np.ndarray) -> np.ndarray:
    """Two INT4 codes per byte: channel 2j in the low nibble, 2j+1 in the high one."""
    c = codes.astype(np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & 0x0F
    out[..., 1::2] = packed >> 4
    return out


def build_unit(K16: np.ndarray, V16: np.ndarray, fp16_meta: bool = False) -> dict:
    """Tier-1 and Tier-2 contents of one (layer, batch row, kv head) after T tokens.

    Sealed blocks are the nb = T // BLOCK complete blocks; the r = T % BLOCK
    newest tokens form the residual block, kept exact in FP16 (Delta = 0,
    eta = 0).  Each sealed block depends only on its own tokens, so the result
    is independent of how the tokens were appended.  vmin / vmax are the
    per-channel value ranges over all T tokens.  fp16_meta: scales and offsets
    stored as binary16 (quantize_keys_block, quantize_values_block).
    """
    T, d = K16.shape
    nb = T // BLOCK
    kc = np.zeros((nb, BLOCK, d), np.int8)
    ks = np.zeros((nb, d), F32)
    vc = np.zeros((nb, BLOCK, d), np.uint8)
    vs = np.zeros((nb, BLOCK, d // VGROUP), F32)
    vz = np.zeros((nb, BLOCK, d // VGROUP), F32)
    vh = np.zeros((nb, BLOCK, d), F32)
    eta = np.zeros(nb, F32)
    for j in range(nb):
        sl = slice(j * BLOCK, (j + 1) * BLOCK)
        kc[j], ks[j] = quantize_keys_block(K16[sl], fp16_meta)
        vc[j], vs[j], vz[j], vh[j], eta[j] = quantize_values_block(V16[sl], fp16_meta)
    Vf = V16.astype(F32)
    vmin = Vf.min(axis=0) if T else np.zeros(d, F32)
    vmax = Vf.max(axis=0) if T else np.zeros(d, F32)
    return dict(nb=nb, r=T - nb * BLOCK, d=d, kcodes=kc, kscale=ks, vcodes=vc,
                vscale=vs, voffset=vz, vhat=vh, eta=eta, vmin=vmin, vmax=vmax,
                K=K16, V=V16)


# ---------------------------------------------------------------------------
# Bounds (Methodology §2)
# ---------------------------------------------------------------------------

def e_key_bound(delta_tail: float, delta_all: float, m8_tail: float) -> float:
    """Total-variation bound between exact and mixed softmax (Methodology §2, E_key).

    Every tail logit is off by at most delta_tail from its exact value and
    every promoted or residual logit is exact, so
      (a) TV <= tanh(delta_tail / 2): the worst case of log-weight shifts in
          [-D, D] is +D on a set of mass 1/(1+e^D) and -D elsewhere;
      (b) TV <= m_tail * (e^(2 delta_tail) - 1): each tail weight changes by a
          factor in [e^-2D, e^2D] after renormalisation, and the promoted part
          moves by exactly the opposite total.
    m_tail is the exact tail mass, unknown before promotion; it is replaced by
    its upper bound from the INT8 estimate m8_tail, using that the scoring pass
    shifted tail logits by at most delta_tail and all others by at most
    delta_all:  m_ub = m8 e^dT / (m8 e^dT + (1 - m8) e^-dA).
    """
    if m8_tail <= 0.0 and delta_tail <= 0.0:
        return 0.0
    a = m8_tail * math.exp(delta_tail)
    m_ub = a / (a + (1.0 - m8_tail) * math.exp(-delta_all)) if a > 0 else 0.0
    return min(math.tanh(delta_tail / 2.0), m_ub * math.expm1(2.0 * delta_tail))


# ---------------------------------------------------------------------------
# Selection (Methodology §3, adaptive top-K)
# ---------------------------------------------------------------------------

def coverage_kstar(ell8: np.ndarray, m8: np.ndarray, m_res: float, tau_cov: float):
    """Smallest K such that the residual mass plus the K largest estimated block
    masses reach tau_cov (Methodology §3, adaptive top-K selection).

    Blocks are ordered by INT8 block log-mass ell8 descending, ties to the lower
    block index; the running sum is float64 in that order, starting from the
    exact residual mass.  tau_cov >= 1 promotes every block.
    Returns (kstar, order, cumulative sums cum[k] = mass covered by the first k).
    """
    nb = ell8.shape[0]
    order = np.lexsort((np.arange(nb), -ell8))
    cum = np.empty(nb + 1)
    cum[0] = m_res
    if nb:
        cum[1:] = m_res + np.cumsum(m8[order])
    if tau_cov >= 1.0:
        return nb, order, cum
    hit = np.nonzero(cum >= tau_cov)[0]
    kstar = int(hit[0]) if hit.size else nb
    return kstar, order, cum


@dataclass
class Thresholds:
    """Runtime thresholds.  tau_cov (coverage) and v_tol (value tolerance) are
    named by the method; eps_key, eps_val, rank_r, rank_tol, max_expand and
    layer_dense_frac are this implementation's readings of the ladder's
    unstated triggers."""

    tau_cov: float = 0.995
    eps_key: float = 5e-3
    eps_val: float = float("inf")
    v_tol: float = 0.05
    rank_r: int = 8
    rank_tol: int = 2
    max_expand: int = 4
    layer_dense_frac: float = 0.5
    naive: bool = False  # certification off: no promotion, no ladder


def _lse(x: np.ndarray, axis=-1):
    m = np.max(x, axis=axis, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    return (np.log(np.sum(np.exp(x - m), axis=axis, keepdims=True)) + m).squeeze(axis)


def dense_attention(q16: np.ndarray, K16: np.ndarray, V16: np.ndarray) -> np.ndarray:
    """Exact attention softmax(q K^T / sqrt(d)) V over FP16 keys and values, float64
    (the O_dense the fallback ladder returns).  q16 [G, d]; K16, V16 [T, d]."""
    d = K16.shape[1]
    s = (q16.astype(np.float64) @ K16.astype(np.float64).T) / math.sqrt(d)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ V16.astype(np.float64)


def _top_r(keys: np.ndarray, idx: np.ndarray, r: int) -> list:
    o = np.lexsort((idx, -keys))
    return [int(idx[i]) for i in o[:r]]


def rank_discordance(ell8: np.ndarray, ell16: np.ndarray, promoted: np.ndarray,
                     rank_r: int) -> int:
    """Disagreement between the INT8 and the FP16 block rankings (Methodology §3,
    rank-consistency check), as a count of discordant pairs.

    Over the promoted blocks, take the top r = min(rank_r, number promoted) by
    INT8 block log-mass and the top r by FP16 block log-mass (each ordered by
    log-mass descending, ties to the lower block index), and form their union U.
    Every promoted block has both log-masses, so both orders are defined on U;
    the result is the number of pairs of U that the two orders place the other
    way round (the Kendall distance of the two rankings restricted to U).  A
    block that one ranking puts near the top and the other far below it is in
    U and is discordant with every block it passes, so a large misranking of a
    heavy block counts many times, while a swap of two neighbours counts once.
    """
    idx = np.nonzero(promoted)[0]
    if idx.size == 0:
        return 0
    r = min(rank_r, idx.size)
    U = sorted(set(_top_r(ell8[idx], idx, r)) | set(_top_r(ell16[idx], idx, r)))
    n = 0
    for i in range(len(U)):
        for j in range(i + 1, len(U)):
            a, b = U[i], U[j]  # a < b: on equal keys the lower index a comes first
            a_first_8 = ell8[a] >= ell8[b]
            a_first_16 = ell16[a] >= ell16[b]
            n += a_first_8 != a_first_16
    return n


def rank_consistent(ell8: np.ndarray, ell16: np.ndarray, promoted: np.ndarray, rank_r: int,
                    rank_tol: int = 0) -> bool:
    """Block-ranking consistency check (Methodology §3): the rankings agree when
    at most rank_tol pairs of the union of the two top-r lists are discordant
    (rank_discordance).  The pages name the check, not its form; this is the
    reading used here, calibrated on the synthetic workloads so that single
    swaps of blocks whose masses INT8 noise cannot separate pass while a
    shuffled group of near-tied heavy blocks fails (parity unpinned beyond this
    stated rule).  rank_tol = 0 is the strict reading: the ordered top-r lists
    must be equal."""
    return rank_discordance(ell8, ell16, promoted, rank_r) <= rank_tol


def decode_group(q16: np.ndarray, u: dict, th: Thresholds) -> dict:
    """Certified decode for the G query heads sharing one kv head (one unit).

    q16: float16 [G, d].  Returns per-head arrays and the unit's trace; the
    per-head dense decision needs every unit of the (layer, batch row) and is
    taken in decode().
    """
    G, d = q16.shape
    nb, r = u["nb"], u["r"]
    sigma = 1.0 / math.sqrt(d)
    q = q16.astype(np.float64)
    K = u["K"].astype(np.float64)
    V = u["V"].astype(np.float64)
    T = nb * BLOCK + r

    # -- INT8 scoring pass (Methodology §3): block log-masses and Delta (§2) --
    khat = (u["kcodes"].astype(np.float64) * u["kscale"][:, None, :].astype(np.float64))
    logit8 = sigma * (khat.reshape(nb * BLOCK, d) @ q.T).T.reshape(G, nb, BLOCK)
    ell8 = _lse(logit8, axis=2) if nb else np.zeros((G, 0))
    # per-token score perturbation bound: |q . (k - k_hat)| <= sum_c |q_c| s_c / 2
    delta = sigma * (np.abs(q) @ u["kscale"].astype(np.float64).T) / 2.0  # [G, nb]
    exact = sigma * (q @ K.T)  # [G, T]: FP16-key logits (residual and promoted blocks)
    res_logit = exact[:, nb * BLOCK:]
    ell_res = _lse(res_logit, axis=1) if r else np.full(G, -np.inf)
    lse_all = _lse(np.concatenate([ell8, ell_res[:, None]], axis=1), axis=1)
    m8 = np.exp(ell8 - lse_all[:, None])
    m_res = np.exp(ell_res - lse_all)

    # -- coverage selection with rung 1 (widen K*) --
    kstar = np.zeros(G, np.int64)
    orders, cums = [], []
    for h in range(G):
        if th.naive:
            kstar[h], o, c = 0, np.arange(nb), np.zeros(nb + 1)
        else:
            kstar[h], o, c = coverage_kstar(ell8[h], m8[h], float(m_res[h]), th.tau_cov)
        orders.append(o)
        cums.append(c)
    kstar0 = kstar.copy()
    expanded = np.zeros(G, bool)
    delta_all = delta.max(axis=1) if nb else np.zeros(G)

    def promoted_set():
        P = np.zeros(nb, bool)
        for h in range(G):
            P[orders[h][:kstar[h]]] = True
        return P

    def e_keys(P):
        tail = ~P
        out = np.zeros(G)
        for h in range(G):
            if not tail.any():
                continue
            out[h] = e_key_bound(float(delta[h][tail].max()), float(delta_all[h]),
                                 float(m8[h][tail].sum()))
        return out

    rounds = 0
    while True:
        P = promoted_set()
        e_key = e_keys(P)
        fail = e_key > th.eps_key
        if th.naive or not fail.any() or rounds == th.max_expand:
            break
        for h in np.nonzero(fail)[0]:
            kstar[h] = min(nb, max(1, 2 * kstar[h]))
            expanded[h] = True
        rounds += 1
    key_fail = (e_key > th.eps_key) & (not th.naive)

    # -- rung 2: FP16 values where m8_b * eta_b exceeds v_tol --
    contrib = m8 * u["eta"].astype(np.float64)[None, :]  # [G, nb]
    if th.naive:
        vp_head = np.zeros((G, nb), bool)
    else:
        vp_head = contrib > th.v_tol
    VP = vp_head.any(axis=0)
    rung2 = vp_head.any(axis=1)

    # -- mixed attention: FP16 logits on promoted + residual, INT8 on the tail --
    logits = exact.copy()
    tail_tok = np.repeat(~P, BLOCK)
    if nb:
        logits[:, :nb * BLOCK][:, tail_tok] = logit8.reshape(G, nb * BLOCK)[:, tail_tok]
    mx = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - mx)
    p /= p.sum(axis=1, keepdims=True)
    Vmix = V.copy()
    int4_tok = np.repeat(~VP, BLOCK)
    if nb:
        Vmix[:nb * BLOCK][int4_tok] = u["vhat"].reshape(nb * BLOCK, d).astype(np.float64)[int4_tok]
    out = p @ Vmix
    pb = p[:, :nb * BLOCK].reshape(G, nb, BLOCK).sum(axis=2) if nb else np.zeros((G, 0))
    e_val = (pb[:, ~VP] * u["eta"].astype(np.float64)[None, ~VP]).sum(axis=1)
    ell16 = np.full((G, nb), np.nan)
    if nb:
        e16 = exact[:, :nb * BLOCK].reshape(G, nb, BLOCK)
        ell16[:, P] = _lse(e16[:, P, :], axis=2)

    # -- rank-consistency check over the promoted blocks --
    rank_fail = np.zeros(G, bool)
    if not th.naive:
        for h in range(G):
            rank_fail[h] = not rank_consistent(ell8[h], ell16[h], P, th.rank_r, th.rank_tol)

    r_v = float(np.max(u["vmax"].astype(np.float64) - u["vmin"].astype(np.float64))) if T else 0.0
    return dict(out=out, e_key=e_key, e_val=e_val, key_fail=key_fail, rank_fail=rank_fail,
                expanded=expanded, rung2=rung2, kstar=kstar, kstar0=kstar0, P=P, VP=VP,
                ell8=ell8, ell16=ell16, delta=delta, m8=m8, m_res=m_res, cum=cums,
                order=orders, contrib=contrib, p=p, r_v=r_v, rounds=rounds)


def decode(q16: np.ndarray, units: list, th: Thresholds) -> dict:
    """One certified decode step of one (layer, batch row).

    q16: float16 [H_q, d]; units: build_unit() results for the H_kv kv heads
    (query head h reads kv head h // (H_q / H_kv)).
    Returns out float64 [H_q, d], e_key, e_val float64 [H_q], rung uint8 [H_q]
    (0 certified as selected, 1 coverage widened, 2 FP16 values promoted,
    3 per-head dense, 4 whole-layer dense), layer_dense, and per-group traces.

    Rung 3 fires when a head's E_key stays above eps_key after max_expand
    widenings or when its rank check fails.  Rung 4 (whole layer dense) fires
    when at least ceil(layer_dense_frac * H_q) heads of the layer took rung 3
    that way.  Otherwise a head whose E_val exceeds eps_val also takes rung 3
    (a post-check; it does not re-count rung 4).  Dense heads return O_dense
    with E_key = E_val = 0.
    """
    Hq, d = q16.shape
    Hkv = len(units)
    G = Hq // Hkv
    groups = [decode_group(q16[g * G:(g + 1) * G], units[g], th) for g in range(Hkv)]
    out = np.concatenate([g["out"] for g in groups])
    e_key = np.concatenate([g["e_key"] for g in groups])
    e_val = np.concatenate([g["e_val"] for g in groups])
    # rungs 3 and 4 are decided before the attention pass, from the E_key and
    # rank-check failures; the E_val post-check (eps_val) then sends single
    # heads to dense attention without re-counting rung 4
    rung3 = np.concatenate([g["key_fail"] | g["rank_fail"] for g in groups])
    rung = np.zeros(Hq, np.uint8)
    rung[np.concatenate([g["expanded"] for g in groups])] = 1
    rung[np.concatenate([g["rung2"] for g in groups])] = 2
    need = math.ceil(th.layer_dense_frac * Hq)
    layer_dense = (not th.naive) and int(rung3.sum()) >= need
    if not th.naive and not layer_dense:
        rung3 = rung3 | (e_val > th.eps_val)
    dense_heads = np.ones(Hq, bool) if layer_dense else rung3
    for h in np.nonzero(dense_heads)[0]:
        u = units[h // G]
        out[h] = dense_attention(q16[h:h + 1], u["K"], u["V"])[0]
        e_key[h] = 0.0
        e_val[h] = 0.0
    rung[rung3] = 3
    if layer_dense:
        rung[:] = 4
    r_v = np.repeat([g["r_v"] for g in groups], G)
    return dict(out=out, e_key=e_key, e_val=e_val, rung=rung, layer_dense=layer_dense,
                rung3=rung3, e_out=r_v * e_key + e_val, groups=groups)
