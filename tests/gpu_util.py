"""Helpers of the GPU parity tests: fill a library cache from the seeded
generator, run the oracle on the same inputs, and compare decisions, bounds
and outputs.  Threshold ties are logged, not failed: a decision that differs
between the CUDA path and the oracle passes only when the oracle's deciding
quantity lies within TIE (relative) of its threshold or of the competing key.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

import synthetic_kv as sk

TIE = 1e-6        # relative band of a threshold tie
OUT_TOL = 2e-3    # max-abs output agreement
BOUND_RTOL = 1e-3  # relative agreement of E_key, E_val
SCORE_RTOL = 1e-5  # block log-masses and Delta (float32 vs float64)


@dataclass
class TieLog:
    entries: list = field(default_factory=list)

    def add(self, what, **kw):
        self.entries.append((what, kw))


def fill_cache(cache, w, layers, ctx, chunks=None, device="cuda"):
    """Append tokens [0, ctx) of `layers` (cache layer i <- workload layer layers[i])."""
    for i, layer in enumerate(layers):
        K, V = sk.kv_layer(w, layer, 0, ctx, device=device)
        if chunks is None:
            cache.append(i, K, V)
        else:
            t = 0
            for n in chunks:
                n = min(n, ctx - t)
                if n <= 0:
                    break
                cache.append(i, K[:, :, t:t + n].contiguous(), V[:, :, t:t + n].contiguous())
                t += n
            if t < ctx:
                cache.append(i, K[:, :, t:].contiguous(), V[:, :, t:].contiguous())
    torch.cuda.synchronize()


def oracle_units(w, layer, b, ctx, fp16_meta=False):
    from oracle import build_unit
    K, V = sk.kv_layer(w, layer, 0, ctx, device="cpu")
    return [build_unit(K[b, g].numpy(), V[b, g].numpy(), fp16_meta) for g in range(w.n_kv_heads)]


def oracle_thresholds(th):
    from oracle import Thresholds as OT
    d = th.float32_rounded()
    return OT(tau_cov=d["tau_cov"], eps_key=d["eps_key"], eps_val=d["eps_val"], v_tol=d["v_tol"],
              rank_r=d["rank_r"], rank_tol=d["rank_tol"], max_expand=d["max_expand"],
              layer_dense_frac=d["layer_dense_frac"], naive=bool(d["naive"]))


def _rel_close(a, b, rtol, atol=0.0):
    return np.abs(a - b) <= rtol * np.maximum(np.abs(a), np.abs(b)) + atol


def _kstar_tie(group, h, k_gpu, tau):
    cum = group["cum"][h]
    k_o = int(group["kstar0"][h])
    lo, hi = min(k_gpu, k_o), max(k_gpu, k_o)
    return all(abs(cum[k] - tau) <= TIE * tau for k in range(lo, hi + 1) if k < len(cum))


def _near_tie_keys(vals, idx_a, idx_b):
    a, b = vals[idx_a], vals[idx_b]
    return abs(a - b) <= TIE * max(1.0, abs(a), abs(b))


def compare_decode(gpu, ora, th, G, log: TieLog, label=""):
    """gpu: dict of numpy arrays for one batch row (out, e_key, e_val, rung, kstar,
    block_flags [Hkv][nb], ell8, ell16, delta, head_flags, ell_res); ora: oracle.decode()."""
    Hq = gpu["out"].shape[0]
    groups = ora["groups"]
    nb = groups[0]["ell8"].shape[1]
    tau = th.tau_cov
    skip_heads = set()
    # scoring pass
    e8_o = np.concatenate([g["ell8"] for g in groups])
    dl_o = np.concatenate([g["delta"] for g in groups])
    if nb:
        assert np.all(_rel_close(gpu["ell8"], e8_o, SCORE_RTOL, 1e-6)), f"{label} ell8"
        assert np.all(_rel_close(gpu["delta"], dl_o, SCORE_RTOL, 1e-7)), f"{label} delta"
    for gi, g in enumerate(groups):
        heads = range(gi * G, (gi + 1) * G)
        # K* and promoted set
        decided_same = True
        for hh, h in enumerate(heads):
            if th.naive:
                continue
            k_o = int(g["kstar"][hh])
            k_g = int(gpu["kstar"][h])
            if k_g != k_o:
                if g["rounds"] == 0 and _kstar_tie(g, hh, k_g, tau):
                    log.add("kstar", label=label, head=h, gpu=k_g, oracle=k_o)
                    decided_same = False
                else:
                    raise AssertionError(f"{label} head {h}: K* {k_g} vs oracle {k_o}")
        pf = (gpu["block_flags"][gi] & 1).astype(bool)
        vf = (gpu["block_flags"][gi] & 2).astype(bool)
        if not np.array_equal(pf, g["P"]):
            bad = np.nonzero(pf != g["P"])[0]
            ok = True
            for j in bad:
                # a block on the coverage boundary of some head within TIE of its neighbour
                near = False
                for hh in range(G):
                    o = g["order"][hh]
                    k = int(g["kstar"][hh])
                    pos = int(np.nonzero(o == j)[0][0])
                    for q_ in (k - 1, k):
                        if 0 <= q_ < nb and _near_tie_keys(g["ell8"][hh], j, o[q_]):
                            near = True
                ok &= near or not decided_same
            assert ok, f"{label} group {gi}: promoted set differs at blocks {bad[:8]}"
            log.add("promoted", label=label, group=gi, blocks=bad.tolist())
            decided_same = False
        if not np.array_equal(vf, g["VP"]):
            bad = np.nonzero(vf != g["VP"])[0]
            for j in bad:
                c = g["contrib"][:, j]
                assert np.any(np.abs(c - th.v_tol) <= 1e-5 * th.v_tol), \
                    f"{label} group {gi}: value promotion differs at block {j} ({c} vs {th.v_tol})"
            log.add("value_promoted", label=label, group=gi, blocks=bad.tolist())
            decided_same = False
        if not decided_same:
            skip_heads.update(heads)
            continue
        # bounds decided from the same sets
        for hh, h in enumerate(heads):
            if ora["rung"][h] >= 3 or gpu["rung"][h] >= 3:
                continue
            assert _rel_close(gpu["e_key"][h], g["e_key"][hh], BOUND_RTOL, 1e-9), \
                f"{label} head {h}: E_key {gpu['e_key'][h]} vs {g['e_key'][hh]}"
            if nb and g["P"].any():
                m = g["P"]
                assert np.all(_rel_close(gpu["ell16"][h][m], g["ell16"][hh][m], SCORE_RTOL, 1e-6)), \
                    f"{label} head {h}: ell16"
    # rungs
    for h in range(Hq):
        if h in skip_heads:
            continue
        rg, ro = int(gpu["rung"][h]), int(ora["rung"][h])
        if rg != ro:
            # rank-check near-ties or the layer count moved by a logged tie
            gi, hh = h // G, h % G
            g = groups[gi]
            # a rank-check difference is excused only when the oracle's discordant
            # pair count is one pair from the tolerance and two blocks near the
            # top of either ranking are tied within TIE (float32 against
            # float64 can then order them either way)
            from oracle import rank_discordance
            P = np.nonzero(g["P"])[0]
            r = min(th.rank_r, P.size)
            tie = False
            if r and abs(rank_discordance(g["ell8"][hh], g["ell16"][hh], g["P"], th.rank_r)
                         - th.rank_tol - 0.5) <= 0.5:
                near = set()
                for key in (g["ell8"][hh], g["ell16"][hh]):
                    near |= {int(P[i]) for i in np.lexsort((P, -key[P]))[: r + 1]}
                near = sorted(near)
                for key in (g["ell8"][hh], g["ell16"][hh]):
                    for i, a in enumerate(near):
                        for b in near[i + 1:]:
                            if _near_tie_keys(key, a, b):
                                tie = True
            # a whole-layer (rung 4) difference is excused only when a tie was
            # logged for this same (layer, batch row) and the oracle's count of
            # rung-3 heads sits within one head of the trigger, so that one
            # tied head could have moved it across
            n3 = int(sum(int(np.sum(gg["key_fail"] | gg["rank_fail"])) for gg in groups))
            need = math.ceil(th.layer_dense_frac * Hq)
            layer_level = ((rg == 4) != (ro == 4) and abs(n3 - need) <= 1 and any(
                e[1].get("label") == label for e in log.entries))
            if not tie and not layer_level:
                raise AssertionError(f"{label} head {h}: rung {rg} vs oracle {ro}")
            log.add("rung", label=label, head=h, gpu=rg, oracle=ro)
            skip_heads.add(h)
    # outputs and E_val
    for h in range(Hq):
        if h in skip_heads:
            continue
        err = float(np.abs(gpu["out"][h] - ora["out"][h]).max())
        assert err <= OUT_TOL, f"{label} head {h}: max-abs output error {err}"
        assert _rel_close(gpu["e_val"][h], ora["e_val"][h], BOUND_RTOL, 1e-9), \
            f"{label} head {h}: E_val {gpu['e_val'][h]} vs {ora['e_val'][h]}"
        if ora["rung"][h] < 3:
            assert _rel_close(gpu["e_key"][h], ora["e_key"][h], BOUND_RTOL, 1e-9)
    return skip_heads


def run_decode(cache, layer, q, th, stream=None):
    outs = cache.alloc_outputs()
    trace = cache.alloc_trace(layer)
    cache.decode(layer, q, th, outputs=outs, trace=trace, stream=stream)
    torch.cuda.synchronize()
    assert cache.device_status() == 0, "a device wait gave up"
    res = dict(out=outs[0], e_key=outs[1], e_val=outs[2], rung=outs[3], **trace)
    return {k: v.cpu().numpy() for k, v in res.items()}


_BLOCK_AXIS = ("block_flags", "ell8", "ell16", "delta")


def row(res, b, nb=None):
    """Batch row b of run_decode's result; with nb, the per-block trace arrays are
    cut to the row's own nb sealed blocks (a ragged batch sizes them for its
    longest row)."""
    out = {k: v[b] for k, v in res.items()}
    if nb is not None:
        for k in _BLOCK_AXIS:
            out[k] = out[k][:, :nb]
    return out
