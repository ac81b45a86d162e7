"""Multi-process plumbing of bench.py on CPU (gloo, world size 2).

The layer has no cross-GPU exchange: each rank runs a replica on its own batch.
What multi-GPU runs rely on is the host-side plumbing: the barrier, the max
over ranks of the device time, and the reference arm running on rank 0 only.
"""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    import torch.distributed as dist
    bench.dist_init("gloo")
    assert dist.get_world_size() == world
    # each rank "measures" a different time; every rank must see the maximum
    got = bench.max_over_ranks(10.0 + 5.0 * rank)
    bench.barrier()
    # the reference arm prints on rank 0 only; other ranks return 0 without work
    ref_rc = bench.run_reference(type("A", (), {"steps": 1, "warmup": 0, "workload": "mixtral",
                                                "experts": None, "tokens": None})()) if rank else 0
    with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
        f.write(f"{got} {ref_rc}")
    dist.destroy_process_group()


def test_max_over_ranks_and_rank0_only_reference(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.spawn(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        got, rc = open(tmp_path / f"r{r}.txt").read().split()
        assert float(got) == 15.0
        assert int(rc) == 0


def test_single_process_max_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.dist_env()[2] >= 1


def test_quantiser_reference_arm_line(capsys):
    """The quantiser's reference arm (the oracle on row slices of w1) prints
    one JSON line carrying the contract's keys."""
    sys.path.insert(0, ROOT)
    import json
    import bench
    args = type("A", (), {"steps": 1, "warmup": 0, "quant_rank": 8, "quant_rounds": 1})()
    assert bench.run_quantize_reference(args, rows=64) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.QUANT_METRIC
    assert line["value"] > 0 and line["unit"] == "weights/s" and line["steps"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "weights/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert "[64, 4096]" in line["config"]["sample"]


def test_quantiser_launch_count_matches_the_launch_list():
    """The quantise line's gpu_launches: one Mixtral-shaped expert at rank 32,
    3 refinement rounds, sketch 64, 2 power steps launched 536 kernels per step
    in the ncu launch list (144 + 24 GEMMs, 168 Gram, 72 Cholesky, 12 each of
    HQQ, eigen, apply, error sum and copy, 68 slice sums)."""
    sys.path.insert(0, ROOT)
    import bench
    shapes = [(14336, 4096), (14336, 4096), (4096, 14336)]
    assert bench.quant_launches(shapes, 32, 3, 64, 2) == 536
    assert bench.quant_launches(shapes, 0, 3, 0, 2) == 12


def test_sweep_cost_counts_active_experts_only():
    """Bytes and FLOPs of one grouped w1 call, worked by hand: codes 3/8 B,
    fp16 scale and zero per 64 weights, fp16 U and V of each active expert,
    bf16 x in and fp32 y out."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    P = type("P", (), {"rank": 32})()
    wk = type("W", (), {"hidden": 4096, "inter": 14336, "T": 3, "n_routed": 8,
                        "experts": [{"w1": P} for _ in range(8)]})()
    counts = np.array([2, 0, 1, 0, 0, 0, 0, 0])
    c = bench.sweep_cost(wk, counts)
    per_expert = 14336 * 4096 * 3 // 8 + 4 * 64 * 14336 + 2 * 32 * (14336 + 4096)
    assert c["bytes"] == 2 * per_expert + 3 * 4096 * 2 + 3 * 14336 * 4
    assert c["flops"] == 3 * 2 * (14336 * 4096 + 32 * (14336 + 4096))
    assert c["active_experts"] == 2


def test_layer_line_carries_the_contract_keys(capsys):
    """The layer line that finish() prints holds every key of the bench
    contract, with the roofline, e2e and clock objects complete (fed with
    made-up timings; no GPU)."""
    sys.path.insert(0, ROOT)
    import json
    import numpy as np
    import torch
    import bench
    import workloads as wl
    wk = wl.small_moe()
    counts = np.full(wk.n_routed, 2)
    bytes_ = bench.layer_bytes(wk, counts)
    args = type("A", (), {"steps": 4, "warmup": 3, "lorc": "fp16", "workload": "mixtral", "tokens": None,
                          "no_cpu_baseline": True})()
    x = torch.zeros(wk.T, wk.hidden, dtype=torch.bfloat16)
    logits = torch.zeros(wk.T, wk.n_routed, dtype=torch.float16)
    y = torch.zeros(wk.T, wk.hidden, dtype=torch.bfloat16)
    clocks = {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": []}
    spread = {"median": 0.18, "p10": 0.179, "p90": 0.182, "steps": 4}
    assert bench.finish(args, wk, 0, 1, wk.T, 0.18, 88000.0, 0.11, 0.05, bytes_, x, logits, y, 76000.0, 8,
                        clocks, spread) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in line, key
    assert line["n_gpus"] == 1 and line["steps"] == 4 and line["gpu_launches"] == 32
    assert line["scaling"] == "weak" and line["higher_is_better"] is True
    rf = line["roofline"]
    assert rf["bound"] in ("hbm", "tensor") and rf["frac"] == rf["achieved"] / rf["peak"]
    assert "traffic" in rf and (rf["traffic"] is None or rf["traffic"] > 0)
    e2e = line["e2e"]
    assert e2e["value"] == 76000.0 and e2e["unit"] == "tokens/s"
    assert e2e["h2d_bytes_per_step"] == wk.T * wk.hidden * 2 + wk.T * wk.n_routed * 2
    assert e2e["d2h_bytes_per_step"] == wk.T * wk.hidden * 2
    assert line["clocks"] == clocks and "workload" in line["config"]
    assert line["step_ms"] == spread


def test_step_quantiles_nearest_rank():
    """The step-time spread takes the nearest-rank quantiles: of 1..10 ms the
    median is 5, p10 1 and p90 9; one step gives itself for every quantile."""
    import bench
    d = [float(v) for v in range(1, 11)]
    assert (bench.nearest_rank(d, 0.5), bench.nearest_rank(d, 0.1), bench.nearest_rank(d, 0.9)) == (5.0, 1.0, 9.0)
    assert bench.nearest_rank([2.5], 0.1) == bench.nearest_rank([2.5], 0.9) == 2.5
    assert bench.nearest_rank(list(range(200)), 0.9) == 179


def test_traffic_hash_ignores_comments_only():
    """The captured traffic stays valid across comment edits of a profiled
    kernel's sources, and only then: the hash covers the code."""
    import bench
    a = "int f(int x) {  // one\n    /* two\n       lines */\n    return x + 1;\n}\n"
    b = "// header\nint f(int x) {\n\n    return x + 1;   // changed comment\n}\n"
    c = "int f(int x) {\n    return x + 2;\n}\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)
    assert len(bench.kernel_source_hash(False)) == 16 and len(bench.kernel_source_hash(True)) == 16

