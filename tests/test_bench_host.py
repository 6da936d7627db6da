"""Host-side logic of bench.py: the max-over-ranks timing and the weak-scaling
value, run as two gloo ranks on the CPU; and the reference (oracle) arm."""

import json
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, ws, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(ws),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    dist = bench.init_dist(ws, "gloo", timeout_s=30)
    dev = torch.device("cpu")
    elapsed = 1.0 + rank  # rank 1 is the slowest
    bench.barrier(dist, dev)
    t = bench.max_over_ranks(elapsed, dist, dev)
    v = bench.weak_scaling_value(10, ws, t)
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump({"t": t, "v": v}, f)
    dist.destroy_process_group()


def test_two_rank_timing_is_max_and_value_is_weak_scaling(tmp_path):
    ws = 2
    mp.start_processes(_rank_main, args=(ws, _free_port(), str(tmp_path)), nprocs=ws,
                       join=True, start_method="spawn")
    for r in range(ws):
        d = json.load(open(tmp_path / f"r{r}.json"))
        assert d["t"] == 2.0
        assert d["v"] == pytest.approx(10 * 2 / 2.0)


def test_single_process_helpers():
    dev = torch.device("cpu")
    assert bench.max_over_ranks(3.5, None, dev) == 3.5
    assert bench.weak_scaling_value(20, 1, 2.0) == 10.0
    assert bench.tier1_bytes_per_block(128) == 64 * 128 + 512 + 64 * 64 + 64 * 4 * 8 + 4


def test_reference_arm_prints_one_line(capsys):
    """--impl reference times the CPU oracle on a bounded sample (tiny workload)."""
    rc = bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3"])
    assert rc == 0
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_cpu_baseline_reports_threads_and_single_thread():
    """The oracle timing beside the GPU numbers: its BLAS threads, and one thread."""
    import certified_quantized_kv_int8_b200 as cqa
    import synthetic_kv as sk
    w = sk.WORKLOADS["tiny"]
    th = cqa.Thresholds(**sk.default_thresholds(w))
    d = bench.cpu_baseline(w, th, budget_s=1.0)
    assert d["kind"] == "oracle" and d["value"] > 0 and d["cores"] >= 1
    assert d["single_thread_value"] > 0


def test_ragged_oracle_scaling():
    """The oracle's sampled row stands for the step's rows in proportion to length."""
    import dataclasses
    import synthetic_kv as sk
    w = sk.WORKLOADS["llama8b_ragged_b4"]
    assert bench.rows_per_sample(w) == pytest.approx(sum(w.row_ctx) / w.row_ctx[0])
    u = dataclasses.replace(sk.WORKLOADS["tiny"], batch=3)
    assert bench.rows_per_sample(u) == 3


def test_reference_arm_on_a_ragged_batch(capsys):
    import dataclasses
    import synthetic_kv as sk
    w = dataclasses.replace(sk.WORKLOADS["tiny"], batch=2, row_ctx=(1024, 300))
    sk.WORKLOADS["tiny_ragged_test"] = dataclasses.replace(w, name="tiny_ragged_test")
    try:
        rc = bench.main(["--impl", "reference", "--workload", "tiny_ragged_test", "--steps", "1",
                         "--warmup", "3"])
    finally:
        del sk.WORKLOADS["tiny_ragged_test"]
    assert rc == 0
    d = json.loads([l for l in capsys.readouterr().out.splitlines() if l.strip()][0])
    assert d["config"]["row_ctx"] == [1024, 300] and d["value"] > 0


def test_l2_policy_and_one_config_for_both_arms(capsys):
    """A step whose Tier 1 is below twice the L2 is timed with the L2 flushed
    between steps; the reference arm reports the config our arm builds."""
    import synthetic_kv as sk
    import certified_quantized_kv_int8_b200 as cqa
    l2 = 126 << 20
    flush8, words8 = bench.l2_policy(sk.WORKLOADS["llama8b_8k_1layer"], False, l2)
    flush32, words32 = bench.l2_policy(sk.WORKLOADS["llama8b_32k_32layer_append"], False, l2)
    assert flush8 and "flushed" in words8
    assert not flush32 and "larger than L2" in words32
    w = sk.WORKLOADS["tiny"]
    rc = bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3"])
    assert rc == 0
    line = [l for l in capsys.readouterr().out.splitlines() if l.strip()][-1]
    got = json.loads(line)["config"]
    th = cqa.Thresholds(**sk.default_thresholds(w))
    want = bench.run_config(w, 1, False, bench.l2_policy(w, False, bench.l2_size_bytes())[1], th)
    assert got == json.loads(json.dumps(want))


def test_tie_counts_hand_case():
    """Residual mass 0.05 and block masses 0.5, 0.3, 0.15: the coverage sums are
    0.55, 0.85, 1.0, so tau_cov = 0.85 is a tie for every certified head; E_key
    equal to eps_key on one head; m_b * eta_b equal to v_tol on one block."""
    import numpy as np
    import certified_quantized_kv_int8_b200 as cqa
    th = cqa.Thresholds(tau_cov=0.85, eps_key=5e-3, v_tol=0.05)
    m = np.array([0.5, 0.3, 0.15])
    ell8 = np.log(np.tile(m, (1, 2, 1)))           # [B=1][Hq=2][nb=3]
    ell_res = np.log(np.full((1, 2), 0.05))
    rung = np.array([[0, 3]])                      # head 1 went dense
    e_key = np.array([[5e-3, 1e-2]])
    eta = [np.array([[0.05 / 0.5, 0.0, 0.0]])]     # [Hkv=1][nb]
    t = bench.tie_counts(e_key, ell8, ell_res, rung, eta, [3], th, G=2)
    assert t == {"coverage": 1, "e_key": 1, "value_promotion": 1}
    th2 = cqa.Thresholds(tau_cov=0.9, eps_key=1e-3, v_tol=0.2)
    assert bench.tie_counts(e_key, ell8, ell_res, rung, eta, [3], th2, G=2) == \
        {"coverage": 0, "e_key": 0, "value_promotion": 0}
