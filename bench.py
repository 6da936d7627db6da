#!/usr/bin/env python
"""Decode-step benchmark of certified quantized KV-cache attention on B200.

One step = one decode step of the whole layer stack of the workload: for every
layer, append the step's new token (workloads that append) and run the
certified decode (INT8 scoring, coverage selection, fused FP16 promotion from
pinned Tier 2, split-K attention with the value bound, combine, rank check,
fallback ladder).  The line printed on rank 0 reports:

  value        decode steps/s of the whole job (inputs resident on the device)
  e2e          the same through the public API with the step's inputs copied
               from pinned host buffers and its outputs read back every step
  int8_int4_path  the same stack with certification off (no promotion, no
               ladder): Tier-1 bytes per step / step time = effective KV GB/s
  roofline     the dominant kernel of the certified step against its bound
  roofline_hbm the INT8 scoring kernel against the measured HBM peak
  cpu_baseline the CPU oracle on a bounded sample of the same workload

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
       python bench.py --impl reference ...   (the CPU oracle arm)
Multi-GPU: torchrun --nproc-per-node N bench.py --gpus N: every rank runs an
independent replica (its own sequences, seed = rank); no collective is on the
data path, timing is the max over ranks.
"""

from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synthetic_kv as sk  # noqa: E402

METRIC = "decode-attn steps/s and effective KV GB/s vs HBM peak at 8K–128K ctx"
DEFAULT_WORKLOAD = "llama8b_32k_32layer_append"
BLOCK = 64


# ---------------------------------------------------------------- helpers ----

def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def tier1_bytes_per_block(d: int, meta_fp16: bool = False) -> int:
    """INT8 key codes + key scales + INT4 value codes + value scale/offset + eta_b
    (scales and offsets 2 bytes each with binary16 metadata, else 4)."""
    m = 2 if meta_fp16 else 4
    return BLOCK * d + m * d + BLOCK * d // 2 + BLOCK * (d // 32) * 2 * m + 4


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(ws: int, backend: str, timeout_s: float = 120.0):
    if ws <= 1:
        return None
    import datetime

    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def max_over_ranks(x: float, dist, device) -> float:
    """Max of a host float over all ranks (the timing reduction)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device):
    if dist is None:
        return
    if device.type == "cuda":
        dist.barrier(device_ids=[device.index])
    else:
        dist.barrier()


def weak_scaling_value(steps_per_rank: int, n_ranks: int, max_elapsed_s: float) -> float:
    """Whole-job steps/s: the steps all ranks ran over the slowest rank's time."""
    return steps_per_rank * n_ranks / max_elapsed_s


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, path: str | None = None):
        import tempfile
        self.index = index
        self.proc = None
        if path is None:
            fd, path = tempfile.mkstemp(prefix=f"cqa_clocks{index}_", suffix=".csv")
            os.close(fd)
        self.path = path

    def start(self):
        d = os.path.dirname(self.path)
        if d:
            os.makedirs(d, exist_ok=True)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv",
                 "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9 or not parts[1].split()[0].isdigit():
                    continue
                sm.append(float(parts[1].split()[0]))
                smax.append(float(parts[2].split()[0]))
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
                "reasons": sorted(reasons)}


def h2d_probe_gbs(device, nbytes: int = 1 << 30) -> float:
    """Pinned host -> device copy rate (the host-link peak used for promotion)."""
    h = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    d = torch.empty(nbytes, dtype=torch.uint8, device=device)
    s = torch.cuda.current_stream(device)
    best = 0.0
    for _ in range(4):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        d.copy_(h, non_blocking=True)
        b.record(s)
        b.synchronize()
        best = max(best, nbytes / (a.elapsed_time(b) * 1e-3) / 1e9)
    del h, d
    return best


def traffic_record(kernel: str):
    """DRAM bytes per unit from a committed ncu summary, if the kernel source is unchanged."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(kernel)
    if not rec:
        return None
    src = os.path.join(ROOT, "certified_quantized_kv_int8_b200", "csrc", rec["source"])
    if not os.path.exists(src):
        return None
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != rec["sha256"]:
            return None
    return rec


TIE_REL = 1e-6  # relative band of a threshold tie


def l2_policy(w: sk.Workload, meta_fp16: bool, l2_bytes: int) -> tuple[bool, str]:
    """Whether the timed steps flush the L2 between them (a step's Tier 1, at the
    workload's starting lengths, below twice the L2) and the config's words for it."""
    step_t1 = (sum(n // BLOCK for n in sk.row_lengths(w)) * w.n_layers * w.n_kv_heads
               * tier1_bytes_per_block(w.head_dim, meta_fp16))
    if step_t1 < 2 * l2_bytes:
        return True, ("L2 flushed before each timed step (Tier 1 %.1f MiB per replica, below "
                      "twice the %.0f MiB L2)" % (step_t1 / 2 ** 20, l2_bytes / 2 ** 20))
    return False, "inputs larger than L2 (Tier 1 %.2f GiB per replica)" % (step_t1 / 2 ** 30)


def run_config(w: sk.Workload, ws: int, meta_fp16: bool, l2_words: str, th) -> dict:
    """The JSON line's config, the same for both arms."""
    appends = w.appends > 0
    return {
        "workload": w.name, "layers": w.n_layers, "global_batch": w.batch * ws,
        "batch_per_gpu": w.batch, "ctx": w.ctx, "q_heads": w.n_q_heads,
        "kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
        **({"row_ctx": list(w.row_ctx)} if w.row_ctx else {}),
        "appends_per_step": 1 if appends else 0, "parallelism": f"replicas{ws}",
        "meta_fp16": bool(meta_fp16), "l2": l2_words,
        "thresholds": dataclasses.asdict(th),
    }


def l2_size_bytes(device=None) -> int:
    """The GPU's L2 size (126 MiB on a B200 when no GPU is visible)."""
    if torch.cuda.is_available():
        return torch.cuda.get_device_properties(device or 0).L2_cache_size
    return 126 << 20


def tie_counts(e_key, ell8, ell_res, rung, eta_rows, nb_row, th, G) -> dict:
    """Decisions of one decode that sat within TIE_REL (relative) of their
    threshold, where float32 rounding could have taken either side: heads whose
    INT8 coverage sum at some rank (residual mass plus the largest block masses)
    or whose E_key lies that close to tau_cov or eps_key, and (kv head, block)
    pairs whose estimated value contribution m_b * eta_b does so for some head
    of the group against v_tol.  e_key, rung: [B][Hq]; ell8: [B][Hq][>= nb];
    ell_res: [B][Hq]; eta_rows[b]: [Hkv][>= nb_b]; nb_row[b]: sealed blocks."""
    out = dict(coverage=0, e_key=0, value_promotion=0)
    cert = rung < 3  # dense heads report 0 for both bounds
    out["e_key"] = int((cert & (np.abs(e_key - th.eps_key) <= TIE_REL * abs(th.eps_key))).sum())
    for b in range(len(nb_row)):
        n = int(nb_row[b])
        if n == 0:
            continue
        x = ell8[b, :, :n].astype(np.float64)  # [Hq][n]
        er = ell_res[b].astype(np.float64)
        mx = np.maximum(x.max(axis=1), er)
        with np.errstate(invalid="ignore"):
            res = np.where(np.isfinite(er), np.exp(er - mx), 0.0)
        tot = np.exp(x - mx[:, None]).sum(axis=1) + res
        m8 = np.exp(x - mx[:, None]) / tot[:, None]
        cum = (res / tot)[:, None] + np.cumsum(-np.sort(-m8, axis=1), axis=1)
        near = np.abs(cum - th.tau_cov) <= TIE_REL * th.tau_cov
        out["coverage"] += int((near.any(axis=1) & cert[b]).sum())
        eb = np.asarray(eta_rows[b])[:, :n]  # [Hkv][n]
        contrib = m8.reshape(eb.shape[0], G, n) * eb[:, None, :]
        out["value_promotion"] += int(
            (np.abs(contrib - th.v_tol) <= TIE_REL * th.v_tol).any(axis=1).sum())
    return out


def decision_census(cache, qs_steps, th, w, device) -> dict:
    """Decode every layer once more with a trace, for the queries of each step in
    qs_steps (a list of per-layer query lists), and count the decisions; counts are
    summed over all those decodes (c["decodes"] of them)."""
    L, B, Hkv, G = w.n_layers, w.batch, w.n_kv_heads, w.group
    c = dict(blocks=0, key_promoted=0, value_promoted=0, heads=0, rungs=[0] * 5, units=0,
             dense_units=0, dense_unit_blocks=0, dense_unit_nonpromoted=0,
             vp_or_dense_blocks=0, int4_blocks=0, blocks_per_layer=0, rank_fail=0, key_fail=0,
             decodes=0, ties=dict(coverage=0, e_key=0, value_promotion=0))
    e_key, e_val = [], []
    for qs, layer in ((qs, layer) for qs in qs_steps for layer in range(L)):
        c["decodes"] += 1
        tr = cache.alloc_trace(layer)
        o = cache.alloc_outputs()
        cache.decode(layer, qs[layer], th, outputs=o, trace=tr)
        torch.cuda.synchronize(device)
        nb = cache.length(layer) // BLOCK
        nb_row = np.array([n // BLOCK for n in cache.row_lengths(layer)])  # ragged rows
        own = (np.arange(nb)[None, :] < nb_row[:, None])[:, None, :]  # [B][1][nb]
        bf = tr["block_flags"].cpu().numpy()[..., :nb]  # [B][Hkv][nb]
        rg = o[3].cpu().numpy()  # [B][Hq]
        dense_h = rg.reshape(B, Hkv, G) >= 3
        unit_dense = dense_h.any(axis=2)  # [B][Hkv]
        unit_mixed = (~dense_h).any(axis=2)
        kp = (bf & 1).astype(bool) & own
        vp = (bf & 2).astype(bool) & own
        c["blocks"] += int(nb_row.sum()) * Hkv
        c["blocks_per_layer"] = int(nb_row.sum()) * Hkv
        c["key_promoted"] += int(kp.sum())
        c["value_promoted"] += int(vp.sum())
        c["units"] += B * Hkv
        c["dense_units"] += int(unit_dense.sum())
        c["dense_unit_blocks"] += int((unit_dense * nb_row[:, None]).sum())
        c["dense_unit_nonpromoted"] += int((~kp & own & unit_dense[..., None]).sum())
        c["vp_or_dense_blocks"] += int(((vp | unit_dense[..., None]) & own).sum())
        c["int4_blocks"] += int((~vp & own & unit_mixed[..., None]).sum())
        c["heads"] += int(rg.size)
        for r in range(5):
            c["rungs"][r] += int((rg == r).sum())
        hf = tr["head_flags"].cpu().numpy()
        c["rank_fail"] += int(((hf & 8) != 0).sum())
        c["key_fail"] += int(((hf & 4) != 0).sum())
        cert = rg < 3  # dense heads report 0 for both bounds
        e_key.append(o[1].cpu().numpy()[cert])
        e_val.append(o[2].cpu().numpy()[cert])
        eta = cache.export(layer, 4)  # EXPORT_ETA: [B][Hkv][nb], or per-row arrays
        t = tie_counts(o[1].cpu().numpy(), tr["ell8"].cpu().numpy(), tr["ell_res"].cpu().numpy(),
                       rg, [np.asarray(eta[b]) for b in range(B)], nb_row, th, G)
        for k in c["ties"]:
            c["ties"][k] += t[k]
    ek, ev = np.concatenate(e_key), np.concatenate(e_val)
    pct = (50, 90, 99, 100)
    c["e_key_pct"] = {f"p{q}": float(np.percentile(ek, q)) for q in pct} if ek.size else None
    c["e_val_pct"] = {f"p{q}": float(np.percentile(ev, q)) for q in pct} if ev.size else None
    return c


def phase_bytes(c: dict, w: sk.Workload, staged_frac: float = 0.0) -> dict:
    """Algorithmic bytes per launch of each decode phase: (host link, HBM).
    staged_frac: share of promote launches whose keys came from the device copy
    made by the whole-layer key prefetch (read from HBM instead of Tier 2)."""
    d, G = w.head_dim, w.group
    kblk = BLOCK * d * 2  # FP16 keys (or values) of one block and kv head
    per = lambda x: x / c["decodes"]  # noqa: E731  (census counts are over all its decodes)
    nblk = per(c["blocks"])
    kp = per(c["key_promoted"]) * kblk
    return {
        "score": (0.0, nblk * (BLOCK * d + 4 * d + G * BLOCK * 4 + 8 * G)),
        "select": (0.0, nblk * (G * 12 + 5)),
        "promote": ((1 - staged_frac) * kp,
                    staged_frac * kp + per(c["key_promoted"]) * G * (BLOCK * 4 + 4)),
        "prefetch": (nblk * kblk, nblk * kblk),
        "dense_keys": (per(c["dense_unit_nonpromoted"]) * kblk,
                       per(c["dense_unit_nonpromoted"]) * G * BLOCK * 4),
        "attend": (per(c["vp_or_dense_blocks"]) * kblk,
                   per(c["int4_blocks"]) * (BLOCK * d // 2 + BLOCK * (d // 32) * 8 + 4)
                   + nblk * G * BLOCK * 4),
    }


def accuracy_on_layer(cache, layer, q, thr_list, dense):
    """Max-abs error against exact attention and the certified bound per threshold set
    (untimed).  The bound is R_V * E_key + E_val per head, R_V = max_c (vmax_c - vmin_c)
    of the head's kv head (Methodology §2)."""
    B, Hq, Hkv = cache.batch, cache.n_q_heads, cache.n_kv_heads
    vr = torch.from_numpy(cache.export(layer, 5)).double()  # [B][Hkv][2][d]
    r_v = (vr[:, :, 1] - vr[:, :, 0]).amax(dim=-1)          # [B][Hkv]
    r_v = r_v.repeat_interleave(Hq // Hkv, dim=1)           # [B][Hq]
    rows = []
    for thr in thr_list:
        trace = cache.alloc_trace(layer)
        o, ek, ev, rg = cache.decode(layer, q, thr, trace=trace)
        torch.cuda.synchronize()
        err = (o.double() - dense.double()).abs().amax(dim=-1).cpu()  # [B][Hq]
        bound = r_v * ek.double().cpu() + ev.double().cpu()
        bf = trace["block_flags"]
        rows.append({
            "max_abs_err": float(err.max()),
            "max_bound": float(bound.max()),
            "bound_holds": bool((err <= bound * (1 + 1e-3) + 1e-5).all()),  # + fp32 noise
            "value_promoted_frac": float(((bf & 2) != 0).float().mean()),
            "max_e_val": float(ev.max()),
            "rung_histogram": [int((rg == k).sum()) for k in range(5)],
        })
    return rows


# --------------------------------------------------------------- our arm ----

def run_ours(args, w: sk.Workload, ws: int, rank: int, dist, device) -> dict | None:
    import certified_quantized_kv_int8_b200 as cqa

    torch.cuda.set_device(device)
    th = cqa.Thresholds(**sk.default_thresholds(w))
    th_naive = dataclasses.replace(th, naive=True)
    L, B, Hq, Hkv, d = w.n_layers, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim
    appends = w.appends > 0
    n_e2e = args.e2e_steps
    n_naive = args.steps
    # headline loops run without per-kernel events; a second, profiled pass of
    # each supplies the per-kernel times (events between kernels add gaps)
    total_steps = args.warmup + 2 * args.steps + n_e2e + args.warmup + 2 * n_naive
    max_ctx = w.ctx + (total_steps if appends else 0)
    wr = dataclasses.replace(w, seed=w.seed + rank)  # independent replica per rank

    cache = cqa.Cache(L, B, Hq, Hkv, d, max_ctx, device=device.index, meta_fp16=args.meta_fp16)
    lens0 = sk.row_lengths(w)
    for layer in range(L):
        if w.row_ctx:  # a ragged batch: each row appended on its own
            for b, n in enumerate(lens0):
                K, V = sk.kv_row(wr, layer, b, 0, n, device=device)
                cache.append_row(layer, b, K, V)
        else:
            K, V = sk.kv_layer(wr, layer, 0, w.ctx, device=device)
            cache.append(layer, K, V)
        del K, V
    torch.cuda.synchronize(device)

    # per-step inputs, resident on the device
    def step_kv(layer, step):
        if not w.row_ctx:
            t = w.ctx + step
            return sk.kv_layer(wr, layer, t, t + 1, device)
        rows = [sk.kv_row(wr, layer, b, n + step, n + step + 1, device)
                for b, n in enumerate(lens0)]
        return (torch.stack([k for k, _ in rows]).contiguous(),
                torch.stack([v for _, v in rows]).contiguous())

    def step_inputs(step):
        qs = [sk.queries(wr, layer, step, device) for layer in range(L)]
        kv = [step_kv(layer, step) for layer in range(L)] if appends else []
        return qs, kv

    inputs = [step_inputs(s) for s in range(total_steps)]
    outs = cache.alloc_outputs()
    stream = torch.cuda.current_stream(device)
    # Tier 1 of a whole step below twice the L2: flush the L2 between steps
    l2_bytes = l2_size_bytes(device)
    do_flush, l2_words = l2_policy(w, args.meta_fp16, l2_bytes)
    flush = torch.empty(2 * l2_bytes, dtype=torch.uint8, device=device) if do_flush else None

    # the timed loops call the C entry points with marshalled arguments prepared
    # once, so the host enqueues a layer in a few microseconds (the e2e pass below
    # goes through the Python API instead)
    import ctypes
    lib = cqa.load_library()
    c_stream = ctypes.c_void_p(stream.cuda_stream)
    c_outs = [ctypes.c_void_p(t.data_ptr()) for t in outs]
    c_th_keep = [th.as_c(), th_naive.as_c()]
    c_th = {id(th): ctypes.byref(c_th_keep[0]), id(th_naive): ctypes.byref(c_th_keep[1])}
    c_in = []
    for qs_, kv_ in inputs:
        c_in.append(([ctypes.c_void_p(x.data_ptr()) for x in qs_],
                     [(ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr())) for k, v in kv_]))

    def run_step(s, thr):
        cq, ckv = c_in[s]
        cth = c_th[id(thr)]
        h = cache.handle
        for layer in range(L):
            if appends:
                rc = lib.cqa_quantize_append(h, layer, ckv[layer][0], ckv[layer][1], 1, c_stream)
                if rc:
                    raise cqa.CqaError(rc, "cqa_quantize_append")
            rc = lib.cqa_decode(h, layer, cq[layer], cth, c_outs[0], c_outs[1], c_outs[2],
                                c_outs[3], None, c_stream)
            if rc:
                raise cqa.CqaError(rc, "cqa_decode")

    def timed(first, n, thr, profile=False, label="timed"):
        barrier(dist, device)
        torch.cuda.synchronize(device)
        if profile:
            cache.profile_begin(1 << 20)
        torch.cuda.nvtx.range_push(label)  # lets a profiler select the timed steps
        if flush is None:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for s in range(first, first + n):
                run_step(s, thr)
            b.record(stream)
            evs = [(a, b)]
        else:
            # a step whose data fits in L2: the L2 is flushed before each step,
            # outside that step's events (the flush also keeps the GPU busy
            # while the host enqueues the step)
            evs = []
            for s in range(first, first + n):
                flush.fill_(s & 0xFF)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                run_step(s, thr)
                b.record(stream)
                evs.append((a, b))
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize(device)
        prof = cache.profile_end() if profile else None
        barrier(dist, device)
        return sum(a.elapsed_time(b) for a, b in evs) * 1e-3, prof

    for s in range(args.warmup):
        run_step(s, th)
    torch.cuda.synchronize(device)

    clocks = ClockSampler(device.index, args.clocks_csv)
    clocks.start()
    elapsed, _ = timed(args.warmup, args.steps, th)
    clk = clocks.stop()
    t_max = max_over_ranks(elapsed, dist, device)
    value = weak_scaling_value(args.steps, ws, t_max)
    # the same steps again with every kernel bracketed by events: per-kernel times
    p_el, prof = timed(args.warmup + args.steps, args.steps, th, profile=True, label="profiled")
    p_max = max_over_ranks(p_el, dist, device)
    phase_ms, phase_n, untimed = prof

    # census of the decisions (untimed, on the state after the timed steps)
    # (several steps' queries when a step has few layers, so that one step's
    # decisions do not stand for all of them)
    n_census = max(1, min(16, 64 // L))
    census = decision_census(
        cache, [inputs[args.warmup + args.steps - 1 - k][0] for k in range(n_census)], th, w,
        device)

    # every layer once more with no copy in flight: in the step, the key
    # prefetch's host-to-device copy delays each kernel launch by about 20 us,
    # which the in-step event times above include
    cache.set_key_prefetch(0)
    torch.cuda.synchronize(device)
    cache.profile_begin(1 << 20)
    cq_last = c_in[args.warmup + args.steps - 1][0]
    for layer in range(L):
        rc = lib.cqa_decode(cache.handle, layer, cq_last[layer], c_th[id(th)], c_outs[0], c_outs[1],
                            c_outs[2], c_outs[3], None, c_stream)
        if rc:
            raise cqa.CqaError(rc, "cqa_decode")
    torch.cuda.synchronize(device)
    iso_ms, iso_n, _ = cache.profile_end()
    cache.set_key_prefetch(1)

    # end to end through the public API: host inputs in, host results out, every step
    e2e = None
    if n_e2e > 0:
        first = args.warmup + 2 * args.steps
        hq = [[x.cpu().pin_memory() for x in inputs[s][0]] for s in range(first, first + n_e2e)]
        hkv = [[(k.cpu().pin_memory(), v.cpu().pin_memory()) for k, v in inputs[s][1]]
               for s in range(first, first + n_e2e)]
        dq = [torch.empty_like(x) for x in inputs[0][0]]
        dkv = [(torch.empty_like(k), torch.empty_like(v)) for k, v in inputs[0][1]]
        ho = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
        h2d = sum(x.numel() * x.element_size() for x in hq[0])
        h2d += sum(k.numel() * k.element_size() * 2 for k, _ in hkv[0])
        d2h = L * sum(t.numel() * t.element_size() for t in outs)
        barrier(dist, device)
        torch.cuda.synchronize(device)
        # one pair of events around all steps (host gaps between steps included);
        # with an L2 flush, one pair per step with the flush between them
        evs = []
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(n_e2e):
            if flush is not None:
                if i:
                    b.record(stream)
                    evs.append((a, b))
                flush.fill_(i & 0xFF)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
            for layer in range(L):
                dq[layer].copy_(hq[i][layer], non_blocking=True)
                if appends:
                    dkv[layer][0].copy_(hkv[i][layer][0], non_blocking=True)
                    dkv[layer][1].copy_(hkv[i][layer][1], non_blocking=True)
                    cache.append(layer, dkv[layer][0], dkv[layer][1], stream)
                cache.decode(layer, dq[layer], th, outputs=outs, stream=stream)
                for h_, d_ in zip(ho, outs):
                    h_.copy_(d_, non_blocking=True)
            stream.synchronize()  # the step's results are on the host
        b.record(stream)
        evs.append((a, b))
        torch.cuda.synchronize(device)
        e_el = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) * 1e-3, dist, device)
        e2e = {"value": weak_scaling_value(n_e2e, ws, e_el), "unit": "steps/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": n_e2e}

    # the INT8/INT4 path alone (certification off): effective KV GB/s, after its
    # own warm-up steps (its kernels' first launches load their code)
    first = args.warmup + 2 * args.steps + n_e2e
    for s in range(first, first + args.warmup):
        run_step(s, th_naive)
    first += args.warmup
    n_el, _ = timed(first, n_naive, th_naive, label="int8_int4")
    n_max = max_over_ranks(n_el, dist, device)
    _, nprof = timed(first + n_naive, n_naive, th_naive, profile=True, label="int8_int4_profiled")

    # accuracy against exact attention on one layer (untimed): the certified path
    # against the INT8/INT4 path; on the needle workload the layer with ties planted
    # in every kv group
    acc_layer = min(w.tie_layer_all, L - 1) if w.needle else 0
    q_acc = inputs[first + 2 * n_naive - 1][0][acc_layer]
    dense = cache.dense_reference(acc_layer, q_acc)
    a_c, a_n = accuracy_on_layer(cache, acc_layer, q_acc, [th, th_naive], dense)
    accuracy = {"layer": acc_layer, "certified": a_c, "int8_int4": a_n}
    vtol_sweep = None
    if args.vtol_sweep:
        # the value-side ablation: value promotion from none to every block (all FP16 values)
        # on layer 0 (on the needle workload layer 17 goes whole-layer dense at any v_tol)
        q0 = inputs[first + 2 * n_naive - 1][0][0]
        dense0 = cache.dense_reference(0, q0)
        tols = [float("inf"), th.v_tol, th.v_tol / 10, th.v_tol / 100, 0.0]
        thrs = [dataclasses.replace(th, v_tol=v) for v in tols]
        rows = accuracy_on_layer(cache, 0, q0, thrs, dense0)
        for v, thr, row in zip(tols, thrs, rows):
            torch.cuda.synchronize(device)
            ta, tb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ta.record(stream)
            for _ in range(5):
                cache.decode(0, q0, thr, outputs=outs, stream=stream)
            tb.record(stream)
            torch.cuda.synchronize(device)
            row["layer"] = 0
            row["v_tol"] = v if v != float("inf") else "inf"
            row["decode_ms"] = ta.elapsed_time(tb) / 5
        vtol_sweep = rows
    # sealed blocks of all (layer, batch row) units per kv head, lengths at the end
    blk_units = sum(n // BLOCK for layer in range(L) for n in cache.row_lengths(layer))
    t1_bytes = blk_units * Hkv * tier1_bytes_per_block(d, args.meta_fp16)  # per step
    peaks = measured_peaks()
    kv_gbs = t1_bytes * n_naive / n_max / 1e9 * ws

    h2d_peak = h2d_probe_gbs(device)

    # per-phase algorithmic bytes per launch, from the decisions of the census
    staged = phase_n["promote_staged"] / max(1, phase_n["promote"])
    pb = phase_bytes(census, w, staged_frac=min(1.0, staged))
    phases = {}
    for p_, ms in phase_ms.items():
        n = phase_n[p_]
        if n == 0 or p_ not in pb:
            continue
        host_b, hbm_b = pb[p_]
        avg = ms / n
        t_host = host_b / (h2d_peak * 1e9)
        t_hbm = hbm_b / (peaks["hbm_gbs"] * 1e9)
        bound = "h2d" if t_host >= t_hbm else "hbm"
        ach = (host_b if bound == "h2d" else hbm_b) / (avg * 1e-3) / 1e9
        pk = h2d_peak if bound == "h2d" else peaks["hbm_gbs"]
        phases[p_] = {"ms_per_step": ms / args.steps, "launches": n, "avg_launch_ms": avg,
                      "host_link_bytes": host_b, "hbm_bytes": hbm_b, "bound": bound,
                      "achieved_gbs": ach, "frac": ach / pk}
        if iso_n.get(p_):
            phases[p_]["isolated_avg_launch_ms"] = iso_ms[p_] / iso_n[p_]
    # the dominant kernel of the step (the key prefetch is a copy-engine
    # transfer, reported on its own below)
    dom = max((k for k in phases if k != "prefetch"), key=lambda k: phases[k]["ms_per_step"])

    def roofline_of(name):
        dp = phases[name]
        rec = traffic_record(name)
        r = {
            "kernel": name, "bound": dp["bound"], "achieved": dp["achieved_gbs"],
            "peak": h2d_peak if dp["bound"] == "h2d" else peaks["hbm_gbs"], "unit": "GB/s",
            "frac": dp["frac"],
            "peak_source": ("pinned 1 GiB cudaMemcpyAsync H2D probe, this run"
                            if dp["bound"] == "h2d"
                            else f"MEASURED_PEAKS.json hbm_gbs, of {peaks['source']}"),
            "avg_launch_ms": dp["avg_launch_ms"],
            "algorithmic_bytes_per_launch": {"host_link": dp["host_link_bytes"],
                                             "hbm": dp["hbm_bytes"]},
            "traffic": (rec["dram_bytes_per_block"] * census["blocks_per_layer"]
                        if rec and name != "prefetch" else None),
        }
        if dp["bound"] == "h2d" and name != "prefetch" and phase_n.get("prefetch"):
            r["note"] = ("the link is shared with the copy-engine key prefetch running beside "
                         "this kernel; step_roofline has the link over the whole step")
        return r

    roofline_kernel = roofline_of(dom)
    # the operation that bounds the step: the key prefetch when it takes the most
    # device time (it is a copy-engine transfer, timed by events on its stream)
    if phases.get("prefetch") and phases["prefetch"]["ms_per_step"] > phases[dom]["ms_per_step"]:
        roofline = roofline_of("prefetch")
        roofline["kernel"] = "prefetch"
        roofline["note"] = ("the step's dominant device operation is the copy-engine transfer of "
                            "each layer's sealed FP16 keys (one cudaMemcpy2DAsync per layer), not "
                            "a kernel; roofline_kernel has the dominant kernel")
    else:
        roofline = roofline_kernel
    # the host link over the whole certified step: key copies by the copy engine
    # plus every kernel's host-link reads, against the pinned-copy rate
    link_bytes = sum(p["host_link_bytes"] * p["launches"] for p in phases.values()) / args.steps
    step_roofline = {
        "bound": "h2d", "bytes_per_step": link_bytes,
        "achieved": link_bytes / (t_max / args.steps) / 1e9, "peak": h2d_peak, "unit": "GB/s",
        "profiled_pass_ms_per_step": p_max / args.steps * 1e3,
        "peak_source": "pinned 1 GiB cudaMemcpyAsync H2D probe, this run",
    }
    step_roofline["frac"] = step_roofline["achieved"] / h2d_peak
    sp = phases["score"]
    rec_sc = traffic_record("score")
    roofline_hbm = {
        "kernel": "score", "bound": "hbm", "achieved": sp["hbm_bytes"] / (sp["avg_launch_ms"] * 1e-3) / 1e9,
        "peak": peaks["hbm_gbs"], "unit": "GB/s",
        "peak_source": f"MEASURED_PEAKS.json hbm_gbs, of {peaks['source']}",
        "avg_launch_ms": sp["avg_launch_ms"], "algorithmic_bytes_per_launch": sp["hbm_bytes"],
        "traffic": (rec_sc["dram_bytes_per_block"] * census["blocks_per_layer"] if rec_sc else None),
    }
    roofline_hbm["frac"] = roofline_hbm["achieved"] / roofline_hbm["peak"]
    if sp.get("isolated_avg_launch_ms"):
        # the same kernel and bytes, timed with no host-to-device copy beside it
        iso = sp["isolated_avg_launch_ms"]
        roofline_hbm["isolated_avg_launch_ms"] = iso
        roofline_hbm["isolated_achieved"] = sp["hbm_bytes"] / (iso * 1e-3) / 1e9
        roofline_hbm["isolated_frac"] = roofline_hbm["isolated_achieved"] / roofline_hbm["peak"]
    # the certified step's quantized path without the promotion: the scoring,
    # selection, rank-check, attention and combine kernels of every layer, each
    # at its isolated time (one pass over the layers with no copy in flight)
    qp = ("score", "select", "decide", "attend", "combine")
    if all(iso_n.get(k) for k in qp):
        qp_ms = sum(iso_ms[k] / iso_n[k] for k in qp) * L
        quant_path = {"kernels": list(qp), "ms_per_step": qp_ms,
                      "effective_kv_gbs": t1_bytes / (qp_ms * 1e-3) / 1e9,
                      "frac_of_hbm_peak": t1_bytes / (qp_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                      "note": "each kernel's isolated CUDA-event time per launch, times the "
                              "layers; the key promotion is excluded, the attention pass "
                              "includes the FP16 values that dense heads read over the host "
                              "link"}
    else:
        quant_path = None
    frac_k = census["key_promoted"] / max(1, census["blocks"])
    frac_v = census["value_promoted"] / max(1, census["blocks"])

    nphase_ms, nphase_n, _ = nprof
    quant_ms = sum(v for k, v in nphase_ms.items() if not k.startswith("append")) / n_naive
    # the streaming pass's own roofline: Tier-1 bytes of a layer per launch
    naive_roof = None
    if nphase_n.get("naive"):
        avg = nphase_ms["naive"] / nphase_n["naive"]
        per_launch = t1_bytes / L
        rec_nv = traffic_record("naive")
        naive_roof = {
            "kernel": "naive", "bound": "hbm", "achieved": per_launch / (avg * 1e-3) / 1e9,
            "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "peak_source": f"MEASURED_PEAKS.json hbm_gbs, of {peaks['source']}",
            "avg_launch_ms": avg, "algorithmic_bytes_per_launch": per_launch,
            "traffic": (rec_nv["dram_bytes_per_block"] * blk_units * Hkv / L if rec_nv else None),
        }
        naive_roof["frac"] = naive_roof["achieved"] / naive_roof["peak"]
    res = {
        "metric": METRIC,
        "value": value,
        "unit": "steps/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": t_max / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": run_config(w, ws, args.meta_fp16, l2_words, th),
        "roofline": roofline,
        "roofline_kernel": roofline_kernel,
        "roofline_hbm": roofline_hbm,
        "step_roofline": step_roofline,
        "certified_quantized_path": quant_path,
        "int8_int4_path": {
            "steps_per_s": n_naive * ws / n_max,
            "effective_kv_gbs": kv_gbs,
            "frac_of_hbm_peak": kv_gbs / ws / peaks["hbm_gbs"],
            "tier1_bytes_per_step": t1_bytes,
            "kernel_ms_per_step": quant_ms,
            "kernel_kv_gbs": t1_bytes / (quant_ms * 1e-3) / 1e9,
            "phases_ms_per_step": {k: v / n_naive for k, v in nphase_ms.items() if nphase_n[k]},
            "launches_per_step": {k: v / n_naive for k, v in nphase_n.items() if v},
            "roofline": naive_roof,
        },
        "promotion": {
            "key_promoted_frac": frac_k, "value_promoted_frac": frac_v,
            "dense_unit_frac": census["dense_units"] / max(1, census["units"]),
            "h2d_peak_gbs": h2d_peak,
            "staged_layer_frac": staged,
            "prefetch_copy_gbs": phases.get("prefetch", {}).get("achieved_gbs"),
            "rung_histogram": census["rungs"],
            "rank_fail_heads": census["rank_fail"],
            "key_fail_heads": census["key_fail"],
            "heads": census["heads"],
            "census_decodes": census["decodes"],
            "threshold_ties": census["ties"],
            "e_key_percentiles": census["e_key_pct"],
            "e_val_percentiles": census["e_val_pct"],
        },
        "accuracy": accuracy,
        "phases": phases,
        "gpu_launches": int(sum(v for k, v in phase_n.items()
                                if k not in ("prefetch", "promote_staged"))),
        "clocks": clk,
    }
    if e2e:
        res["e2e"] = e2e
    if vtol_sweep:
        res["vtol_sweep"] = vtol_sweep
    cache.close()
    return res


# ------------------------------------------------ the larger workloads ----

EXTRA_WORKLOADS = ("llama8b_64k_b4_t3values", "llama8b_128k_needle")


def run_extra_workload(name: str, device, cert_steps: int = 5, naive_steps: int = 10,
                       warmup: int = 3, meta_fp16: bool = False) -> dict:
    """A few timed steps of a larger workload on one GPU: certified steps/s, the
    INT8/INT4 path's effective KV GB/s and the streaming kernel's per-launch
    roofline (CUDA events on the launch stream, in a second, profiled pass)."""
    import certified_quantized_kv_int8_b200 as cqa
    w = sk.WORKLOADS[name]
    th = cqa.Thresholds(**sk.default_thresholds(w))
    th_naive = dataclasses.replace(th, naive=True)
    L, B, Hq, Hkv, d = w.n_layers, w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim
    t_setup = time.perf_counter()
    cache = cqa.Cache(L, B, Hq, Hkv, d, w.ctx, device=device.index, meta_fp16=meta_fp16)
    for layer in range(L):
        K, V = sk.kv_layer(w, layer, 0, w.ctx, device=device)
        cache.append(layer, K, V)
        del K, V
    torch.cuda.synchronize(device)
    t_setup = time.perf_counter() - t_setup
    n_q = warmup + cert_steps + 2 * naive_steps + 1
    qs = [[sk.queries(w, layer, s, device) for layer in range(L)] for s in range(n_q)]
    outs = cache.alloc_outputs()
    stream = torch.cuda.current_stream(device)

    def run(first, n, thr):
        torch.cuda.synchronize(device)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for s in range(first, first + n):
            for layer in range(L):
                cache.decode(layer, qs[s][layer], thr, outputs=outs, stream=stream)
        b.record(stream)
        torch.cuda.synchronize(device)
        return a.elapsed_time(b) * 1e-3

    for s in range(warmup):
        run(s, 1, th)
    clocks = ClockSampler(device.index)
    clocks.start()
    t_cert = run(warmup, cert_steps, th)
    first = warmup + cert_steps
    run(first, 1, th_naive)  # the INT8/INT4 path's own warm-up
    t_naive = run(first, naive_steps, th_naive)
    clk = clocks.stop()
    cache.profile_begin(1 << 20)
    run(first + naive_steps, naive_steps, th_naive)
    nms, nn, _ = cache.profile_end()
    census = decision_census(cache, [qs[warmup + cert_steps - 1]], th, w, device)
    blk_units = sum(n // BLOCK for layer in range(L) for n in cache.row_lengths(layer))
    t1_bytes = blk_units * Hkv * tier1_bytes_per_block(d, meta_fp16)
    peaks = measured_peaks()
    kv_gbs = t1_bytes * naive_steps / t_naive / 1e9
    avg = nms["naive"] / nn["naive"]
    per_launch = t1_bytes / L
    rec = traffic_record("naive")
    cache.close()
    return {
        "config": {"workload": name, "layers": L, "batch": B, "ctx": w.ctx, "q_heads": Hq,
                   "kv_heads": Hkv, "head_dim": d, "meta_fp16": meta_fp16},
        "certified_steps_per_s": cert_steps / t_cert, "certified_steps": cert_steps,
        "int8_int4_path": {
            "steps_per_s": naive_steps / t_naive, "steps": naive_steps,
            "effective_kv_gbs": kv_gbs, "frac_of_hbm_peak": kv_gbs / peaks["hbm_gbs"],
            "tier1_bytes_per_step": t1_bytes,
            "roofline": {
                "kernel": "naive", "bound": "hbm", "achieved": per_launch / (avg * 1e-3) / 1e9,
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": per_launch / (avg * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "peak_source": f"MEASURED_PEAKS.json hbm_gbs, of {peaks['source']}",
                "avg_launch_ms": avg, "algorithmic_bytes_per_launch": per_launch,
                "traffic": (rec["dram_bytes_per_block"] * blk_units * Hkv / L if rec else None),
            },
        },
        "promotion": {
            "key_promoted_frac": census["key_promoted"] / max(1, census["blocks"]),
            "value_promoted_frac": census["value_promoted"] / max(1, census["blocks"]),
            "dense_unit_frac": census["dense_units"] / max(1, census["units"]),
            "rung_histogram": census["rungs"], "rank_fail_heads": census["rank_fail"],
            "heads": census["heads"], "threshold_ties": census["ties"],
            "e_key_percentiles": census["e_key_pct"], "e_val_percentiles": census["e_val_pct"],
        },
        "clocks": clk,
        "setup_s": t_setup,
    }


# --------------------------------------------------------- oracle timing ----

def oracle_sample_seconds(w: sk.Workload, layer: int, b: int, th) -> tuple[float, dict]:
    """Time the CPU oracle's decode of one (layer, batch row) of the workload."""
    from oracle import Thresholds as OT
    from oracle import build_unit, decode
    K, V = sk.kv_row(w, layer, b, 0, sk.row_lengths(w)[b], device="cpu")
    units = [build_unit(K[g].numpy(), V[g].numpy()) for g in range(w.n_kv_heads)]
    q = sk.queries(w, layer, 0, "cpu")[b].numpy()
    d = th.float32_rounded()
    oth = OT(tau_cov=d["tau_cov"], eps_key=d["eps_key"], eps_val=d["eps_val"], v_tol=d["v_tol"],
             rank_r=d["rank_r"], rank_tol=d["rank_tol"], max_expand=d["max_expand"],
             layer_dense_frac=d["layer_dense_frac"])
    t0 = time.perf_counter()
    decode(q, units, oth)
    return time.perf_counter() - t0, units


def rows_per_sample(w: sk.Workload) -> float:
    """Batch rows of a step in units of row 0 (the sampled row), by length: the
    oracle's decode time grows with the row's length."""
    lens = sk.row_lengths(w)
    return sum(lens) / lens[0]


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(w: sk.Workload, th, budget_s: float = 20.0) -> dict:
    """The oracle as it stands, on one (layer, batch row) at a time, scaled to steps/s."""
    secs, n = [], 0
    t_start = time.perf_counter()
    layer = 0
    while n < 1 or (time.perf_counter() - t_start < budget_s and n < 3):
        s, _ = oracle_sample_seconds(w, layer % w.n_layers, 0, th)
        secs.append(s)
        n += 1
        layer += 1
    per = statistics.mean(secs)
    scale = w.n_layers * rows_per_sample(w)
    step_s = per * scale
    res = {"value": 1.0 / step_s, "unit": "steps/s", "cores": blas_threads(), "kind": "oracle",
           "sample": f"{n} of {w.n_layers * w.batch} (layer, batch row) decodes of one step, "
                     f"{per:.2f} s each, scaled to the full step (appends not included"
                     + (", rows scaled by length)" if w.row_ctx else ")")}
    # the same oracle on one thread (one (layer, batch row) decode)
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            s1, _ = oracle_sample_seconds(w, 0, 0, th)
        res["single_thread_value"] = 1.0 / (s1 * scale)
        res["single_thread_sample"] = f"1 (layer, batch row) decode, {s1:.2f} s, scaled"
    except ImportError:
        pass
    return res


def run_reference(args, w: sk.Workload, ws: int, rank: int) -> dict | None:
    import certified_quantized_kv_int8_b200 as cqa_py  # Thresholds only; no library call
    if rank != 0:
        return None
    th = cqa_py.Thresholds(**sk.default_thresholds(w))
    K, V = sk.kv_row(w, 0, 0, 0, sk.row_lengths(w)[0], device="cpu")
    from oracle import Thresholds as OT
    from oracle import build_unit, decode
    units = [build_unit(K[g].numpy(), V[g].numpy()) for g in range(w.n_kv_heads)]
    d = th.float32_rounded()
    oth = OT(tau_cov=d["tau_cov"], eps_key=d["eps_key"], eps_val=d["eps_val"], v_tol=d["v_tol"],
             rank_r=d["rank_r"], rank_tol=d["rank_tol"], max_expand=d["max_expand"],
             layer_dense_frac=d["layer_dense_frac"])
    qs = [sk.queries(w, 0, s, "cpu")[0].numpy() for s in range(args.warmup + args.steps)]
    for s in range(args.warmup):
        decode(qs[s], units, oth)
    t0 = time.perf_counter()
    for s in range(args.warmup, args.warmup + args.steps):
        decode(qs[s], units, oth)
    el = time.perf_counter() - t0
    per = el / args.steps
    scale = w.n_layers * rows_per_sample(w)
    value = 1.0 / (per * scale)
    sample = (f"each step decodes one (layer 0, batch row 0) of the {w.n_layers}-layer, "
              f"batch-{w.batch} step ({per:.2f} s) and is scaled by {scale:g}"
              + (" (rows scaled by length)" if w.row_ctx else ""))
    return {
        "metric": METRIC, "impl": "reference", "value": value, "unit": "steps/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per * scale * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": run_config(w, ws, args.meta_fp16, l2_policy(w, args.meta_fp16, l2_size_bytes())[1],
                             th),
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 64, the 32K workload's append-and-decode "
                         "steps; 2048 for a single-layer workload, whose steps are short)")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(sk.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--vtol-sweep", action="store_true",
                    help="add the value-side ablation: one layer decoded at v_tol = inf, the "
                         "default, /10, /100 and 0 (every block's FP16 values)")
    ap.add_argument("--layers", type=int, default=None,
                    help="decode only the first N layers (profiling captures; the reported "
                         "line then covers N layers, not the workload's step)")
    ap.add_argument("--meta-fp16", action="store_true",
                    help="caches store Tier-1 scales and offsets as binary16 (212 instead of "
                         "232 bytes per token and kv head)")
    ap.add_argument("--no-extra-workloads", action="store_true",
                    help="skip the few timed steps of the 64K x B4 and 128K workloads that the "
                         "default single-GPU line adds under `workloads`")
    ap.add_argument("--clocks-csv", default=None,
                    help="keep the nvidia-smi samples of the timed region in this file")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    w = sk.WORKLOADS[args.workload]
    if args.layers is not None:
        w = dataclasses.replace(w, n_layers=max(1, min(args.layers, w.n_layers)))
    ws, rank, local = dist_env()

    if args.impl == "reference":
        if args.steps is None:
            args.steps = 64
        res = run_reference(args, w, ws, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0

    from certified_quantized_kv_int8_b200.build import build
    if rank == 0:
        build()
    dist = init_dist(ws, "nccl")
    if dist is not None:
        barrier(dist, torch.device("cuda", local))
        build()  # no-op once rank 0 built it
    device = torch.device("cuda", local)
    if args.steps is None:
        args.steps = 64 if w.n_layers > 1 else 2048
    res = run_ours(args, w, ws, rank, dist, device)
    if (res is not None and ws == 1 and args.layers is None and not args.no_extra_workloads
            and w.name == DEFAULT_WORKLOAD):
        # the larger single-GPU workloads, a few steps each (one GPU only: the
        # 64K x B4 workload holds 32 GiB of pinned host memory)
        res["workloads"] = {n: run_extra_workload(n, device, meta_fp16=args.meta_fp16)
                            for n in EXTRA_WORKLOADS}
    if rank == 0 and res is not None:
        if ws == 1 and not args.no_cpu_baseline:
            import certified_quantized_kv_int8_b200 as cqa
            res["cpu_baseline"] = cpu_baseline(w, cqa.Thresholds(**sk.default_thresholds(w)))
        print(json.dumps(res), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
