#!/usr/bin/env python
"""Benchmark: MoE layer tokens/s and achieved HBM bandwidth of the int3 +
low-rank-compensator forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl milo|reference]
                    [--workload mixtral|deepseek|prefill|single|quantize|sweep] [--lorc fp16|int3]

One step = one pass of the whole hot path over one batch of synthetic tokens:
router (top-k + grouping) -> activation preparation -> compensator
down-projection -> grouped int3 GEMM w1|w3 + SwiGLU -> preparation of h ->
compensator down-projection -> grouped int3 GEMM w2 -> weighted combine.
Weight packing is offline and not timed.

Default workload: the Mixtral-8x7B-shaped decode layer (H 4096, I 14336, 8
experts, top-2, ranks drawn from {0,16,32,64}, 16 bf16 tokens).  Its packed
weights (~0.6 GB) are larger than the 126 MB L2, so every step streams them
from HBM; no flush is needed.

Multi-GPU: each rank runs its own replica on its own batch (the layer has no
cross-GPU exchange on one node), the time is the max over ranks and `value`
counts the tokens of all ranks ("weak" scaling).

--impl reference times the CPU oracle (plain C, fp64) on the host cores, each
step a bounded sample of tokens of the same workload (with --workload
quantize: the oracle's quantiser on a row slice of the same weight).

More lines of their own: --workload single times the single-expert decode
call (1 x 1024 -> 1024, rank 16) over rotated weight copies; --workload
quantize times the offline quantiser on one Mixtral-shaped expert;
--workload sweep times the w1 projection alone over 1 ... 1024 Zipf-routed
tokens (L2 flushed before each call).
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "MoE layer tokens/s and achieved HBM TB/s (% roofline) for int3+LoRC forward"
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------------------
# distributed plumbing (also exercised by the gloo tests on CPU)
# ---------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def dist_init(backend: str):
    import datetime

    import torch.distributed as dist
    rank, local, world = dist_env()
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, local, world


def max_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.out = open(f"/tmp/milo_clocks_{os.getpid()}.csv", "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "100"], stdout=self.out,
                                         stderr=subprocess.DEVNULL)
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
        self.out.close()
        rows = []
        with open(self.out.name) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 9:
                    rows.append(p)
        os.unlink(self.out.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        power = [num(r[3]) or 0.0 for r in rows]
        pmax = max(power) if power else 0.0
        load = [num(r[1]) for r, pw in zip(rows, power) if pw >= 0.5 * pmax and num(r[1]) is not None]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip().lower() == "active"})
        return {"sm_mhz": statistics.median(load or sm) if (load or sm) else None,
                "sm_max_mhz": num(rows[0][2]), "reasons": reasons, "samples": len(rows),
                "power_w_max": pmax}


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------

def make_workload(name: str, experts: int | None = None, tokens: int | None = None):
    """The named workload; `experts` / `tokens` shrink it for profiler captures."""
    if name == "mixtral":
        return wl.mixtral(T=tokens or 16, n_experts=experts or 8)
    if name == "deepseek":
        return wl.deepseek(T=tokens or 64)
    if name == "prefill":
        return wl.prefill(T=tokens or 8192, n_experts=experts or 8)
    raise ValueError(name)


def describe(wk) -> str:
    return (f"{wk.name}: H{wk.hidden} I{wk.inter} E{wk.n_routed}+{wk.n_shared}shared top{wk.top_k} "
            f"T{wk.T} int3 g64 ranks={list(map(int, wk.ranks))}")


def gpu_layer(milo, wk, torch, lorc_int3: bool = False):
    experts = []
    for e in range(wk.n_experts):
        d = {}
        for n in ("w1", "w3", "w2"):
            P = wk.experts[e][n]

            def dev(a):
                return torch.from_numpy(a.view(np.int16)).view(torch.float16).cuda()
            d[n] = milo.QWeight.quantize(dev(P.W), dev(P.U) if P.rank else None,
                                         dev(P.V) if P.rank else None, lorc_int3=lorc_int3)
        experts.append(d)
    torch.cuda.synchronize()
    return milo.MoELayer(experts, wk.n_routed, wk.n_shared, wk.top_k)


def layer_bytes(wk, counts, lorc_int3: bool = False) -> dict:
    """Algorithmic HBM bytes of one step: every active expert's packed codes
    (3/8 B per weight), fp16 scale and zero (4/64 B per weight), compensator U
    and V (fp16), plus activations in and out, for each kernel."""
    H, I = wk.hidden, wk.inter
    active = [e for e in range(wk.n_routed) if counts[e] > 0] + list(range(wk.n_routed, wk.n_experts))
    rows = int(sum(counts[:wk.n_routed])) + wk.n_shared * wk.T
    qz = lambda n, k: n * k * 3 // 8 + 2 * (k // 64) * n * 2   # codes + scale + zero
    glu = dict(weights=0, lorc_u=0, lorc_v=0)
    w2 = dict(weights=0, lorc_u=0, lorc_v=0)
    cb = 7 / 16 if lorc_int3 else 2      # compensator bytes per element: int3 codes + s, z, or fp16
    for e in active:
        r1, r3, r2 = (wk.experts[e][n].rank for n in ("w1", "w3", "w2"))
        glu["weights"] += 2 * qz(I, H)
        glu["lorc_u"] += (r1 + r3) * I * cb
        glu["lorc_v"] += (r1 + r3) * H * cb
        w2["weights"] += qz(H, I)
        w2["lorc_u"] += r2 * H * cb
        w2["lorc_v"] += r2 * I * cb
    act_x = rows * H * 2
    act_h = rows * I * 2
    glu_kernel = glu["weights"] + glu["lorc_u"] + act_x + act_h + rows * 2 * 64 * 2
    w2_kernel = w2["weights"] + w2["lorc_u"] + act_h + rows * H * 4
    step = (glu["weights"] + glu["lorc_u"] + glu["lorc_v"] + w2["weights"] + w2["lorc_u"] + w2["lorc_v"]
            + wk.T * H * 2 + act_x + 2 * act_h + wk.T * H * 2)
    # tensor work of the two GEMM launches: the int3 contraction plus the
    # compensator's up-projection t U^T (the down-projection x V^T runs
    # in its own kernel)
    r_glu = sum(int(counts[e]) * (wk.experts[e]["w1"].rank + wk.experts[e]["w3"].rank)
                for e in range(wk.n_routed) if counts[e] > 0)
    r_glu += sum(wk.T * (wk.experts[e]["w1"].rank + wk.experts[e]["w3"].rank)
                 for e in range(wk.n_routed, wk.n_experts))
    r_w2 = sum(int(counts[e]) * wk.experts[e]["w2"].rank for e in range(wk.n_routed) if counts[e] > 0)
    r_w2 += sum(wk.T * wk.experts[e]["w2"].rank for e in range(wk.n_routed, wk.n_experts))
    glu_flops = 2 * rows * (2 * I) * H + 2 * r_glu * I
    w2_flops = 2 * rows * H * I + 2 * r_w2 * H
    return {"glu_kernel": glu_kernel, "w2_kernel": w2_kernel, "step": step,
            "weights_only": glu["weights"] + w2["weights"], "active_experts": len(active), "rows": rows,
            "glu_flops": glu_flops, "w2_flops": w2_flops,
            "routed_rows": int(sum(counts[:wk.n_routed])), "n_routed": wk.n_routed}


def uses_tensor_path(bytes_) -> bool:
    """The library's choice of grouped GEMM: the tcgen05 kernel once the
    routed rows reach 64 per routed expert on average (MILO_GEMM=mma|tc
    overrides it), else the mma.sync kernel."""
    forced = os.environ.get("MILO_GEMM", "")
    if forced in ("mma", "tc"):
        return forced == "tc"
    return bytes_["routed_rows"] >= 64 * bytes_["n_routed"]


def peaks() -> dict:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def _code_only(text: str) -> str:
    """Source text without its comments and blank lines (comment edits leave
    the kernel, and so its captured traffic, unchanged)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_source_hash(tensor: bool = False) -> str:
    """Hash of the code (comments stripped) of the sources the profiled GEMM
    kernel is built from."""
    h = hashlib.sha256()
    files = ("int3_gemm_rank_b200/csrc/gemm_tc.cu", "int3_gemm_rank_b200/csrc/milo_tc.cuh") if tensor else \
        ("int3_gemm_rank_b200/csrc/gemv.cu",)
    for rel in files + ("int3_gemm_rank_b200/csrc/milo_device.cuh", "int3_gemm_rank_b200/csrc/milo_kernels.h"):
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(name: str, tensor: bool = False):
    """DRAM bytes per launch of the GEMM kernel from the committed ncu summary,
    or None when the summary is missing or the kernel source changed since."""
    path = os.path.join(ROOT, "profiles", name)
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                if ":" in line and line.startswith("- "):
                    k, v = line[2:].split(":", 1)
                    kv[k.strip()] = v.strip()
        if kv.get("kernel_source_sha256_16") != kernel_source_hash(tensor):
            return None
        return float(kv["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


# ---------------------------------------------------------------------------
# CPU oracle legs
# ---------------------------------------------------------------------------

def oracle_sample_step(wk, tokens, ref_cache, nthreads):
    """Run the oracle's full layer on `tokens` (routing included); returns seconds."""
    import oracle
    L = wk.logits[tokens]
    t0 = time.perf_counter()
    ids, w, *_ = oracle.route(L, wk.top_k, wk.renorm)
    need = sorted(set(int(e) for e in ids.ravel())) + list(range(wk.n_routed, wk.n_experts))
    for e in need:
        if e not in ref_cache:
            raise RuntimeError("expert not prepared")
    experts = [ref_cache.get(e) or ref_cache[need[0]] for e in range(wk.n_experts)]
    oracle.moe_forward(wk.x[tokens], wk.x_dtype == "bf16", ids, w, experts, wk.n_routed, wk.n_shared,
                       wk.hidden, wk.inter, nthreads=nthreads)
    return time.perf_counter() - t0


def prepare_oracle_experts(wk, experts_needed):
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    jobs = [(e, n) for e in experts_needed for n in ("w1", "w3", "w2")]
    with ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1))) as ex:
        res = list(ex.map(lambda j: oracle.quantize_projection(wk.experts[j[0]][j[1]].W,
                                                               wk.experts[j[0]][j[1]].U,
                                                               wk.experts[j[0]][j[1]].V), jobs))
    cache = {}
    for (e, n), p in zip(jobs, res):
        cache.setdefault(e, {})[n] = p
    return cache


def cpu_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def sample_tokens(wk, n: int, seed: int) -> np.ndarray:
    return np.sort(np.random.default_rng(seed).choice(wk.T, size=min(n, wk.T), replace=False))


def cpu_baseline(wk, n_tokens: int = 4, passes: int = 7, budget_s: float = 25.0) -> dict:
    """The oracle, as it stands, on the host cores: `passes` full-layer passes
    over `n_tokens` sampled tokens each (bounded by `budget_s`)."""
    import oracle
    nthreads = cpu_threads()
    samples = [sample_tokens(wk, n_tokens, s) for s in range(1, passes + 1)]
    need = set(range(wk.n_routed, wk.n_experts))
    for tok in samples:
        ids, *_ = oracle.route(wk.logits[tok], wk.top_k, wk.renorm)
        need |= set(int(e) for e in ids.ravel())
    cache = prepare_oracle_experts(wk, sorted(need))
    times = []
    for tok in samples:
        times.append(oracle_sample_step(wk, tok, cache, nthreads))
        if sum(times) > budget_s:
            break
    total = sum(times)
    return {"value": len(times) * n_tokens / total, "unit": "tokens/s", "cores": nthreads,
            "kind": "oracle",
            "sample": f"{len(times)} oracle passes over {n_tokens} of the {wk.T} tokens each "
                      f"(full layer for those tokens, routing included), {total:.1f} s of CPU work"}


def run_reference(args):
    """--impl reference: the oracle as the reference arm (rank 0 only)."""
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    wk = make_workload(args.workload, args.experts, args.tokens)
    n_tok = 2
    nthreads = cpu_threads()
    steps = max(1, args.steps)
    warm = max(0, args.warmup)
    # prepare every expert the sampled steps will touch
    seeds = list(range(100, 100 + warm + steps))
    import oracle
    need = set(range(wk.n_routed, wk.n_experts))
    for s in seeds:
        ids, *_ = oracle.route(wk.logits[sample_tokens(wk, n_tok, s)], wk.top_k, wk.renorm)
        need |= set(int(e) for e in ids.ravel())
    cache = prepare_oracle_experts(wk, sorted(need))
    for s in seeds[:warm]:
        oracle_sample_step(wk, sample_tokens(wk, n_tok, s), cache, nthreads)
    times = [oracle_sample_step(wk, sample_tokens(wk, n_tok, s), cache, nthreads) for s in seeds[warm:]]
    total = sum(times)
    value = steps * n_tok / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": steps, "warmup": warm, "ms_per_step": 1e3 * total / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": describe(wk), "tokens_per_step": n_tok,
                       "sample": f"{n_tok} of {wk.T} tokens per step"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                             "sample": f"{n_tok} of {wk.T} tokens per step, full layer for those tokens"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_milo(args):
    import torch

    import int3_gemm_rank_b200 as milo
    from int3_gemm_rank_b200 import build as milo_build

    rank, local, world = dist_env()
    if not os.path.exists(milo.LIB_PATH):
        milo_build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init("nccl")

    wk = make_workload(args.workload, args.experts, args.tokens)
    layer = gpu_layer(milo, wk, torch, args.lorc == "int3")

    def to_dev(a, dt):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(dt).to(dev)

    x = to_dev(wk.x, torch.bfloat16 if wk.x_dtype == "bf16" else torch.float16)
    logits = to_dev(wk.logits, torch.float16)
    out_dt = torch.bfloat16
    T, k, E = wk.T, wk.top_k, wk.n_routed
    st = milo.new_status(dev)
    ws = layer.workspace(T, dev)
    y = torch.empty((T, wk.hidden), dtype=out_dt, device=dev)
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    wts = torch.empty((T, k), dtype=torch.float32, device=dev)
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty(T * k, dtype=torch.int32, device=dev)
    route = {"w": wts, "offsets": off, "perm": perm, "inv_perm": inv}
    L = milo.lib()
    import ctypes as C
    flags = milo.MILO_ROUTE_RENORM if wk.renorm else 0
    stream = torch.cuda.current_stream(dev)
    sp = C.c_void_p(stream.cuda_stream)

    def step(xin, lin):
        cur = C.c_void_p(torch.cuda.current_stream(dev).cuda_stream)   # the capture stream while capturing
        s = L.milo_route(C.c_void_p(lin.data_ptr()), T, E, k, flags, C.c_void_p(ids.data_ptr()),
                         C.c_void_p(wts.data_ptr()), C.c_void_p(off.data_ptr()),
                         C.c_void_p(perm.data_ptr()), C.c_void_p(inv.data_ptr()),
                         C.c_void_p(st.data_ptr()), cur)
        if s:
            milo._check(s, "milo_route")
        milo.milo_moe_forward(layer, xin, route, out_dtype=out_dt, dev_status=st, y=y, ws=ws)

    # route (one kernel; from 512 tokens on a top-k kernel first), then the forward:
    # mma.sync path: prep x, gemm w1|w3 (compensator inside), prep h, gemm w2 (compensator and
    # combine inside); tcgen05 path: prep x, lorc w1|w3, gemm w1|w3, prep h, lorc w2, gemm w2,
    # combine, the compensator launches dropping out when no expert has one
    has_lorc = any(wk.experts[e][n].rank for e in range(wk.n_experts) for n in ("w1", "w3", "w2"))

    # --- correctness gate on the bench configuration itself
    step(x, logits)
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} on the bench workload")
    counts = np.diff(off.cpu().numpy())
    bytes_ = layer_bytes(wk, counts, args.lorc == "int3")
    forward = (7 if has_lorc else 5) if uses_tensor_path(bytes_) else 5
    launches_per_step = forward + (2 if T >= 512 else 1)

    # --- the timed step: one CUDA graph of the whole step (route + layer), its
    # launches and their programmatic dependencies captured once and replayed
    run_step = capture_step(torch, dev, lambda: step(x, logits)) if args.graph else (lambda: step(x, logits))

    # --- warm-up and clock soak (also brings the clocks to their loaded state)
    for _ in range(args.warmup):
        run_step()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    t_soak = time.perf_counter()
    while time.perf_counter() - t_soak < args.soak:
        for _ in range(20):
            run_step()
        torch.cuda.synchronize()

    # --- timed region 1: K steps bracketed by events on the launching stream.
    # No event between the kernels: they overlap through programmatic
    # dependent launch, which an event record in the stream would serialise.
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4 * args.steps)]
    for e in ev:            # torch creates the CUDA event on its first record
        e.record(stream)
    milo.milo_set_profile_events(None)
    barrier(dev)
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("milo/timed_steps")      # NVTX ranges name the regions for ncu --nvtx
    start.record(stream)
    for i in range(args.steps):
        run_step()
    stop.record(stream)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    barrier(dev)
    ms_total = start.elapsed_time(stop)
    # --- timed region 2: the same K steps with events around the two grouped
    # GEMM launches, for their average launch durations (roofline)
    torch.cuda.nvtx.range_push("milo/gemm_events")
    for i in range(args.steps):
        milo.milo_set_profile_events(ev[4 * i:4 * i + 4])
        step(x, logits)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    milo.milo_set_profile_events(None)
    barrier(dev)
    # --- timed region 3 (graph replays only): the same K steps with an event
    # after each, for the spread of the step time (a stream launch sequence
    # would lose its cross-step overlap to the events)
    spread = step_spread(torch, run_step, args.steps, stream, dev) if args.graph else None
    clocks = sampler.stop()
    glu_ms = statistics.mean(ev[4 * i].elapsed_time(ev[4 * i + 1]) for i in range(args.steps))
    w2_ms = statistics.mean(ev[4 * i + 2].elapsed_time(ev[4 * i + 3]) for i in range(args.steps))
    ms_total = max_over_ranks(ms_total, dev)
    ms_step = ms_total / args.steps
    value = world * T * args.steps / (ms_total / 1e3)
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} after the timed region")

    bytes_["graph"] = bool(args.graph)
    # --- end to end through the public API with host buffers
    if args.no_e2e:
        e2e_value, e2e_ms = None, None
    else:
        e2e_value, e2e_ms = run_e2e(args, torch, step, x, logits, y, out_dt, T, wk, dev, stream, world)
    return finish(args, wk, rank, world, T, ms_step, value, glu_ms, w2_ms, bytes_, x, logits, y,
                  e2e_value, launches_per_step, clocks, spread)


def nearest_rank(sorted_vals, q: float) -> float:
    """The q-quantile of sorted values by the nearest-rank rule."""
    i = min(len(sorted_vals) - 1, max(0, math.ceil(q * len(sorted_vals)) - 1))
    return sorted_vals[i]


def step_spread(torch, run_step, steps: int, stream, dev) -> dict:
    """Median, p10 and p90 of single step times (ms): `steps` more replays,
    an event recorded after each; every quantile is the max over ranks."""
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    for e in ev:
        e.record(stream)
    torch.cuda.synchronize()
    barrier(dev)
    torch.cuda.nvtx.range_push("milo/step_spread")
    ev[0].record(stream)
    for i in range(steps):
        run_step()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    barrier(dev)
    d = sorted(ev[i].elapsed_time(ev[i + 1]) for i in range(steps))
    return {"median": max_over_ranks(nearest_rank(d, 0.5), dev), "p10": max_over_ranks(nearest_rank(d, 0.1), dev),
            "p90": max_over_ranks(nearest_rank(d, 0.9), dev), "steps": steps}


def capture_step(torch, dev, fn):
    """One CUDA graph of fn's launches (stream capture; the library's
    programmatic launches become programmatic edges); returns its replay."""
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream(dev).wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g.replay


def run_e2e(args, torch, step, x, logits, y, out_dt, T, wk, dev, stream, world):
    x_h = torch.empty_like(x, device="cpu").pin_memory()
    x_h.copy_(x.cpu())
    l_h = torch.empty_like(logits, device="cpu").pin_memory()
    l_h.copy_(logits.cpu())
    y_h = torch.empty((T, wk.hidden), dtype=out_dt).pin_memory()
    x_d, l_d = torch.empty_like(x), torch.empty_like(logits)

    def e2e_step():
        x_d.copy_(x_h, non_blocking=True)
        l_d.copy_(l_h, non_blocking=True)
        step(x_d, l_d)
        y_h.copy_(y, non_blocking=True)

    if args.graph:   # the copies in and out are part of the captured step
        e2e_step = capture_step(torch, dev, e2e_step)

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    barrier(dev)
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("milo/e2e_steps")
    s2.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e2.record(stream)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    e2e_ms = max_over_ranks(s2.elapsed_time(e2), dev)
    e2e_value = world * T * args.steps / (e2e_ms / 1e3)
    return e2e_value, e2e_ms


def roofline(args, pk, bytes_, glu_ms, glu_gbs) -> dict:
    """Roofline of the dominant kernel, the w1|w3 grouped GEMM: HBM-bound on
    the mma.sync path (decode), tensor-bound on the tcgen05 path (prefill),
    where the fp16 dense peak equals the measured bf16 one (same rate)."""
    if uses_tensor_path(bytes_):
        tf = bytes_["glu_flops"] / (glu_ms / 1e3) / 1e12
        peak = pk["bf16_tflops"]
        return {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                "frac_of_sustained": tf / pk["bf16_tflops_sustained"],
                # the captures are of the default workloads (fp16 compensators)
                "traffic": profiled_traffic("tc_gemm_glu_prefill.md", tensor=True)
                if args.workload == "prefill" and args.tokens is None and args.lorc == "fp16" else None,
                "kernel": "tc_gemm_kernel<true> (w1|w3 grouped int3 GEMM on tcgen05 + compensator + SwiGLU)",
                "algorithmic_flops_per_launch": bytes_["glu_flops"], "ms_per_launch": glu_ms,
                "peak_source": "measured cuBLAS bf16 GEMM, burst (MEASURED_PEAKS.json bf16_tflops); "
                               "fp16 runs at the bf16 rate" if pk["source"] == "measured"
                else "fallback 1590 TFLOP/s"}
    return {"bound": "hbm", "achieved": glu_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": glu_gbs / pk["hbm_gbs"], "traffic": profiled_traffic("gemv_glu_mixtral_decode.md")
            if args.workload == "mixtral" and args.tokens is None and args.lorc == "fp16" else None,
            "kernel": "gemv_kernel<true> (w1|w3 grouped int3 GEMM + compensator + SwiGLU)",
            "algorithmic_bytes_per_launch": bytes_["glu_kernel"], "ms_per_launch": glu_ms,
            "peak_source": f"{pk['source']} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
            if pk["source"] == "measured" else "fallback 6650 GB/s"}


def finish(args, wk, rank, world, T, ms_step, value, glu_ms, w2_ms, bytes_, x, logits, y, e2e_value,
           launches_per_step, clocks, spread=None):
    pk = peaks()
    glu_gbs = bytes_["glu_kernel"] / (glu_ms / 1e3) / 1e9
    step_gbs = bytes_["step"] / (ms_step / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": describe(wk), "tokens_per_step": T, "x_dtype": wk.x_dtype,
                   "compensator": "int3 (U^T and V packed like the weights)" if args.lorc == "int3" else "fp16",
                   "y_dtype": "bf16",
                   "compute_dtype": "int3 codes x f16 activations (exact f16 code patterns), f32 accumulate",
                   "l2": f"inputs larger than L2: {bytes_['weights_only'] / 1e6:.0f} MB of packed weights "
                         f"streamed per step vs {L2_BYTES / 1e6:.0f} MB L2; no flush",
                   "parallelism": f"replica per GPU x{world}", "active_experts": bytes_["active_experts"],
                   "launch": "one CUDA graph per step (route + layer)" if bytes_.get("graph")
                   else "stream launches"},
        "roofline": roofline(args, pk, bytes_, glu_ms, glu_gbs),
        "layer_hbm": {"bytes_per_step": bytes_["step"], "achieved_gbs": step_gbs,
                      "frac": step_gbs / pk["hbm_gbs"]},
        "kernels": {"gemm_w1w3_ms": glu_ms, "gemm_w2_ms": w2_ms,
                    "gemm_w2_gbs": bytes_["w2_kernel"] / (w2_ms / 1e3) / 1e9,
                    "gemm_w1w3_gbs": glu_gbs,
                    "gemm_w1w3_tflops": bytes_["glu_flops"] / (glu_ms / 1e3) / 1e12,
                    "gemm_w2_tflops": bytes_["w2_flops"] / (w2_ms / 1e3) / 1e12},
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": x.numel() * x.element_size() + logits.numel() * logits.element_size(),
                "d2h_bytes_per_step": y.numel() * y.element_size()},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if spread is not None:
        line["step_ms"] = spread
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wk)
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------
# single-projection batch sweep (--workload sweep)
# ---------------------------------------------------------------------------

SWEEP_TOKENS = (1, 4, 16, 64, 256, 1024)
SWEEP_METRIC = ("grouped int3 + rank-32 compensator w1 projection (4096 -> 14336, 8 experts, Zipf routing): "
                "tokens/s per batch size, with HBM and tensor rooflines")


def sweep_cost(wk, counts) -> dict:
    """Algorithmic bytes and FLOPs of one grouped w1 projection call: each
    active expert's packed codes, fp16 scale and zero, and fp16 U and V, plus
    x in (bf16) and y out (fp32); FLOPs of the int3 contraction and of both
    compensator products."""
    H, I, T = wk.hidden, wk.inter, wk.T
    active = [e for e in range(wk.n_routed) if counts[e] > 0]
    qz = I * H * 3 // 8 + 2 * (H // 64) * I * 2
    nbytes = sum(qz + 2 * wk.experts[e]["w1"].rank * (I + H) for e in active) + T * H * 2 + T * I * 4
    flops = sum(2 * int(counts[e]) * (I * H + wk.experts[e]["w1"].rank * (I + H)) for e in active)
    return {"bytes": nbytes, "flops": flops, "active_experts": len(active)}


def run_sweep(args):
    """The w1 projection alone over 1 ... 1024 tokens, each routed to one
    Zipf-drawn expert: the crossover from the memory-bound mma.sync kernel to
    the tcgen05 kernel.  L2 is flushed (a 256 MB write) before every timed
    call, since the small batches touch fewer weights than L2 holds."""
    import torch

    import int3_gemm_rank_b200 as milo
    from int3_gemm_rank_b200 import build as milo_build

    rank, local, world = dist_env()
    if not os.path.exists(milo.LIB_PATH):
        milo_build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init("nccl")

    def f16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.float16).to(dev)

    base = wl.sweep(1)
    projs = []
    for e in range(base.n_routed):
        P = base.experts[e]["w1"]
        projs.append(milo.QWeight.quantize(f16(P.W), f16(P.U) if P.rank else None, f16(P.V) if P.rank else None))
    lin = milo.GroupedLinear(projs)
    # the unfused pipeline the paper compares against: a dequantisation pass
    # writing fp16 weights, then library fp16 GEMMs (cuBLAS through torch)
    W_hat = [torch.empty((base.inter, base.hidden), dtype=torch.float16, device=dev) for _ in projs]
    st = milo.new_status(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    pk = peaks()
    # prep and the grouped GEMM (compensator and combine inside) on the mma.sync path; prep,
    # compensator down-projection, grouped GEMM and combine on the tcgen05 path
    has_lorc = any(P.rank for P in (base.experts[e]["w1"] for e in range(base.n_routed)))
    points, launches = [], 0
    sampler = ClockSampler(local)
    sampler.start()
    for T in SWEEP_TOKENS:
        wk = wl.sweep(T) if T > 1 else base
        x = torch.from_numpy(np.ascontiguousarray(wk.x).view(np.int16)).view(torch.bfloat16).to(dev)
        ids = torch.from_numpy(np.ascontiguousarray(wk.ids, dtype=np.int32)).to(dev)
        r = milo.milo_route(None, 1, False, E=base.n_routed, ids=ids, dev_status=st)
        y = torch.empty((T, wk.inter), dtype=torch.float32, device=dev)
        ws = lin.workspace(T, 1, dev)

        def call():
            lin(x, r["offsets"], r["perm"], k=1, dev_status=st, y=y, ws=ws)

        for _ in range(args.warmup):
            call()
        # the timed call is one CUDA graph (its launches back to back on the
        # device, as in a decode loop); the flush before it is not timed
        graph_call = capture_step(torch, dev, call)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4 * args.steps)]
        for e in ev:            # torch creates the CUDA event on its first record
            e.record(stream)
        milo.milo_set_profile_events(None)
        barrier(dev)
        torch.cuda.synchronize()
        # pass 1: the whole call (all its kernels), no event inside it
        for i in range(args.steps):
            flush.zero_()
            ev[4 * i].record(stream)
            graph_call()
            ev[4 * i + 1].record(stream)
        torch.cuda.synchronize()
        # pass 2: events around the grouped GEMM launch alone
        for i in range(args.steps):
            flush.zero_()
            milo.milo_set_profile_events(ev[4 * i + 2:4 * i + 4])
            call()
        torch.cuda.synchronize()
        milo.milo_set_profile_events(None)
        # the unfused pipeline on the same rows: dequantise the active experts,
        # then per expert y = x W_hat^T + (x V^T) U^T in fp16 (cuBLAS)
        act = [e for e in range(base.n_routed) if (wk.ids[:, 0] == e).any()]
        rows = {e: torch.from_numpy(np.flatnonzero(wk.ids[:, 0] == e)).to(dev) for e in act}
        y_unf = torch.empty((T, wk.inter), dtype=torch.float32, device=dev)

        def unfused():
            for e in act:
                milo.milo_dequantize(projs[e].packed, wk.inter, wk.hidden, out=W_hat[e])
            xh = x.half()
            for e in act:
                xe = xh.index_select(0, rows[e])
                ye = xe @ W_hat[e].t()
                if projs[e].rank:
                    ye = ye + (xe @ projs[e].V.t()) @ projs[e].U.t()
                y_unf.index_copy_(0, rows[e], ye.float())

        # both grouped GEMM kernels on the same call, for the crossover
        by_path = {}
        for path in ("mma", "tc"):
            milo.milo_set_gemm_path(path)
            ws_p = torch.empty(lin.workspace_bytes(T, 1) + 256, dtype=torch.uint8, device=dev)

            def call_p():
                lin(x, r["offsets"], r["perm"], k=1, dev_status=st, y=y, ws=ws_p)

            call_p()
            gp = capture_step(torch, dev, call_p)
            pe = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps)]
            for i in range(args.steps):
                flush.zero_()
                pe[2 * i].record(stream)
                gp()
                pe[2 * i + 1].record(stream)
            torch.cuda.synchronize()
            by_path[path] = 1e3 * statistics.mean(pe[2 * i].elapsed_time(pe[2 * i + 1]) for i in range(args.steps))
            del gp, ws_p
        milo.milo_set_gemm_path("auto")
        unfused()
        graph_unf = capture_step(torch, dev, unfused)
        ue = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps)]
        for i in range(args.steps):
            flush.zero_()
            ue[2 * i].record(stream)
            graph_unf()
            ue[2 * i + 1].record(stream)
        torch.cuda.synchronize()
        unf_ms = statistics.mean(ue[2 * i].elapsed_time(ue[2 * i + 1]) for i in range(args.steps))
        unf_err = float(((y_unf - y).abs() / torch.maximum(y.abs(), y.pow(2).mean().sqrt())).max())
        call_ms = max_over_ranks(statistics.mean(ev[4 * i].elapsed_time(ev[4 * i + 1])
                                                 for i in range(args.steps)), dev)
        gemm_ms = statistics.mean(ev[4 * i + 2].elapsed_time(ev[4 * i + 3]) for i in range(args.steps))
        counts = np.bincount(wk.ids.ravel(), minlength=base.n_routed)
        cost = sweep_cost(wk, counts)
        forced = os.environ.get("MILO_GEMM", "")
        tensor = forced == "tc" if forced in ("mma", "tc") else T >= 64 * base.n_routed
        launches += 2 * args.steps * ((4 if has_lorc else 3) if tensor else 3)
        gbs = cost["bytes"] / (call_ms / 1e3) / 1e9
        tflops = cost["flops"] / (call_ms / 1e3) / 1e12
        points.append({"tokens": T, "kernel": "tc_gemm_kernel (tcgen05)" if tensor else "gemv_kernel (mma.sync)",
                       "active_experts": cost["active_experts"], "us_per_call": 1e3 * call_ms,
                       "gemm_us": 1e3 * gemm_ms, "tokens_per_s": world * T / (call_ms / 1e3),
                       "algorithmic_bytes": cost["bytes"], "algorithmic_flops": cost["flops"],
                       "hbm_gbs": gbs, "hbm_frac": gbs / pk["hbm_gbs"], "tflops": tflops,
                       "tensor_frac": tflops / pk["bf16_tflops"],
                       "us_per_call_mma": by_path["mma"], "us_per_call_tc": by_path["tc"],
                       "unfused_us_per_call": 1e3 * unf_ms, "speedup_vs_unfused": unf_ms / call_ms,
                       "unfused_vs_fused_max_rel_diff": unf_err})
    clocks = sampler.stop()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} on the sweep")
    top = points[-1]
    tensor_top = top["kernel"].startswith("tc_")
    line = {
        "metric": SWEEP_METRIC, "value": top["tokens_per_s"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": top["us_per_call"] / 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": f"w1 projection H{base.hidden} -> I{base.inter}, {base.n_routed} experts, rank "
                               f"{int(base.ranks[0])}, int3 g64, k = 1 with Zipf(1.1) expert ids, x bf16, y fp32; "
                               f"value and ms_per_step at {top['tokens']} tokens, every size under 'sweep'",
                   "l2": "flushed by a 256 MB write before every timed call",
                   "launch": "each timed call one CUDA graph replay; gemm_us from a second pass of stream "
                             "launches with events around the grouped GEMM",
                   "parallelism": f"replica per GPU x{world}"},
        "sweep": points,
        "unfused": "per point: the unfused pipeline on the same rows (milo_dequantize of the active experts to fp16, "
                   "then per expert x W_hat^T + (x V^T) U^T as fp16 cuBLAS GEMMs through torch), one CUDA graph "
                   "per call, L2 flushed before it; speedup = its time / the fused call's",
        "roofline": ({"bound": "tensor", "achieved": top["tflops"], "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                      "frac": top["tensor_frac"], "traffic": None}
                     if tensor_top else
                     {"bound": "hbm", "achieved": top["hbm_gbs"], "peak": pk["hbm_gbs"], "unit": "GB/s",
                      "frac": top["hbm_frac"], "traffic": None}),
        "e2e": None, "gpu_launches": launches, "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------
# single expert, decode (--workload single)
# ---------------------------------------------------------------------------

SINGLE_METRIC = ("single int3 expert with a rank-16 compensator, decode (1 token, 1024 -> 1024): "
                 "time per call and achieved HBM bandwidth over rotated weight copies")


def single_cost(P) -> dict:
    """Algorithmic bytes of one single-expert call (codes, fp16 scale and zero,
    fp16 U and V, x in fp16, y out fp32) and of its grouped GEMM launch (all
    but V, which the compensator's down-projection reads); FLOPs of the int3
    contraction and both compensator products."""
    n, k, r = P.n, P.k, P.rank
    blob = n * k * 3 // 8 + 2 * (k // 64) * n * 2
    act = k * 2 + n * 4
    return {"call": blob + 2 * r * (n + k) + act, "gemm": blob + 2 * r * n + act,
            "flops": 2 * (n * k + r * (n + k)), "copy": blob + 2 * r * (n + k)}


def run_single(args):
    """The single-expert decode call, milo_grouped_linear on one token (no
    routing: one expert).  Its 0.53 MB of weights fit in L2, so the step
    rotates over distinct copies of the packed weight and its compensator,
    at least 3 x L2 of them, and L2 is flushed (a 256 MB write) before each
    timed region; within a region a copy comes back only after 3 x L2 of
    other copies.  One step = one call; the K steps are one CUDA graph."""
    import torch

    import int3_gemm_rank_b200 as milo
    from int3_gemm_rank_b200 import build as milo_build

    rank, local, world = dist_env()
    if not os.path.exists(milo.LIB_PATH):
        milo_build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init("nccl")

    x_bits, P = wl.single()
    cost = single_cost(P)
    n_copies = -(-3 * L2_BYTES // cost["copy"])

    def f16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.float16).to(dev)

    q0 = milo.QWeight.quantize(f16(P.W), f16(P.U), f16(P.V))
    lins = [milo.GroupedLinear([milo.QWeight(q0.packed.clone(), P.n, P.k, q0.U.clone(), q0.V.clone())])
            for _ in range(n_copies)]
    x = f16(x_bits)
    st = milo.new_status(dev)
    r = milo.milo_route(None, 1, False, E=1, ids=torch.zeros((1, 1), dtype=torch.int32, device=dev),
                        dev_status=st)
    off, perm = r["offsets"], r["perm"]
    y = torch.empty((1, P.n), dtype=torch.float32, device=dev)
    ws = lins[0].workspace(1, 1, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    K = args.steps
    launches_per_call = 3          # prep, grouped GEMM (compensator inside), per-slot combine

    def calls(xin, base=0):
        for j in range(K):
            milo.milo_grouped_linear(lins[(base + j) % n_copies], xin, off, perm, 1, torch.float32, st, y, ws)

    # gate on the bench configuration: the calls run with a clean device status
    # (their parity with the oracle is tests/test_gpu_fullsize.py's single-expert case)
    calls(x)
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} on the single-expert workload")
    graph = capture_step(torch, dev, lambda: calls(x))
    for _ in range(args.warmup):
        graph()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    t_soak = time.perf_counter()
    while time.perf_counter() - t_soak < args.soak:
        graph()
        torch.cuda.synchronize()
    flush.zero_()
    barrier(dev)
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    graph()
    stop.record(stream)
    torch.cuda.synchronize()
    barrier(dev)
    ms_total = max_over_ranks(start.elapsed_time(stop), dev)
    # region 2: the calls launched one by one with events around the grouped GEMM
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * K)]
    for e in ev:
        e.record(stream)
    flush.zero_()
    torch.cuda.synchronize()
    for j in range(K):
        milo.milo_set_profile_events(ev[2 * j:2 * j + 2])
        milo.milo_grouped_linear(lins[j % n_copies], x, off, perm, 1, torch.float32, st, y, ws)
    torch.cuda.synchronize()
    milo.milo_set_profile_events(None)
    clocks = sampler.stop()
    gemm_ms = statistics.mean(ev[2 * j].elapsed_time(ev[2 * j + 1]) for j in range(K))
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} after the timed region")
    ms_call = ms_total / K
    pk = peaks()
    call_gbs = cost["call"] / (ms_call / 1e3) / 1e9
    gemm_gbs = cost["gemm"] / (gemm_ms / 1e3) / 1e9

    # end to end: x from pinned host memory and y back every call
    e2e = None
    if not args.no_e2e:
        x_h = x.cpu().pin_memory()
        y_h = torch.empty((1, P.n), dtype=torch.float32).pin_memory()
        x_d = torch.empty_like(x)

        def e2e_calls():
            for j in range(K):
                x_d.copy_(x_h, non_blocking=True)
                milo.milo_grouped_linear(lins[j % n_copies], x_d, off, perm, 1, torch.float32, st, y, ws)
                y_h.copy_(y, non_blocking=True)

        g2 = capture_step(torch, dev, e2e_calls)
        for _ in range(args.warmup):
            g2()
        flush.zero_()
        torch.cuda.synchronize()
        barrier(dev)
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        g2()
        e2.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(s2.elapsed_time(e2), dev)
        e2e = {"value": world * K / (e2e_ms / 1e3), "unit": "tokens/s", "us_per_call": 1e3 * e2e_ms / K,
               "h2d_bytes_per_step": x.numel() * 2, "d2h_bytes_per_step": y.numel() * 4}
    line = {
        "metric": SINGLE_METRIC, "value": world * K / (ms_total / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": ms_call, "us_per_call": 1e3 * ms_call,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": f"single expert decode: x fp16 [1 x {P.k}], W [{P.n} x {P.k}] int3 g64 "
                               f"(N(0, 0.02), 0.1 % outliers x20), rank {P.rank} fp16 U, V; y fp32",
                   "l2": f"{n_copies} rotated copies of the packed weight and compensator "
                         f"({n_copies * cost['copy'] / 1e6:.0f} MB, 3 x L2) and a 256 MB flush before each "
                         f"timed region",
                   "launch": f"one CUDA graph of the {K} calls", "parallelism": f"replica per GPU x{world}"},
        "roofline": {"bound": "hbm", "achieved": gemm_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": gemm_gbs / pk["hbm_gbs"], "traffic": None,
                     "kernel": "gemv_kernel<false> (grouped int3 GEMM + compensator, split-K)",
                     "algorithmic_bytes_per_launch": cost["gemm"], "ms_per_launch": gemm_ms,
                     "peak_source": f"{pk['source']} HBM copy bandwidth"},
        "call_hbm": {"bytes_per_call": cost["call"], "achieved_gbs": call_gbs, "frac": call_gbs / pk["hbm_gbs"],
                     "roofline_us": 1e6 * cost["call"] / (pk["hbm_gbs"] * 1e9)},
        "e2e": e2e, "gpu_launches": launches_per_call * K, "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = single_cpu_baseline(x_bits, P)
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def single_oracle_calls(x_bits, P, budget_s: float, max_calls: int = 1 << 30):
    """Oracle single-expert calls (the layer's linear, fp64) until budget_s."""
    import oracle
    ref = oracle.quantize_projection(P.W, P.U, P.V)
    X = wl.f16_bits_to_f32(x_bits).astype(np.float64)
    nthreads = cpu_threads()
    t0 = time.perf_counter()
    n = 0
    while n < max_calls and (n == 0 or time.perf_counter() - t0 < budget_s):
        oracle.linear(X, ref, nthreads=nthreads)
        n += 1
    return n, time.perf_counter() - t0, nthreads


def single_cpu_baseline(x_bits, P) -> dict:
    n, secs, nthreads = single_oracle_calls(x_bits, P, 10.0)
    return {"value": n / secs, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
            "sample": f"{n} oracle calls of the single-expert decode projection (1 token), {secs:.1f} s"}


def run_single_reference(args) -> int:
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    x_bits, P = wl.single()
    single_oracle_calls(x_bits, P, 0.0, max_calls=max(0, args.warmup))
    n, secs, nthreads = single_oracle_calls(x_bits, P, 1e9, max_calls=max(1, args.steps))
    value = n / secs
    line = {"impl": "reference", "metric": SINGLE_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": n, "warmup": args.warmup, "ms_per_step": 1e3 * secs / n, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"single expert decode: x fp16 [1 x {P.k}], W [{P.n} x {P.k}] int3 g64, "
                                   f"rank {P.rank} fp16 U, V; y fp32"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                             "sample": f"{n} oracle calls of the whole projection, one per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# offline quantiser (--workload quantize)
# ---------------------------------------------------------------------------

QUANT_METRIC = ("offline MiLo quantiser: weights quantised and compensated per second "
                "(HQQ int3, rank-r compensator by subspace iteration, refinement rounds)")
# fp32 operations of one HQQ iteration per weight outside the shrinkage (which
# is zero for all but outlier errors): t*inv, +z, rint, two clamps, -z, *s,
# t-w_r, |e|, err+, t-w_e, *inv, r-u, acc+, and the a^3 beta^2 pre-test's
# first product counted once -> 15
HQQ_OPS_PER_WEIGHT_ITER = 15
FP32_LANES = 148 * 4 * 32


def quant_matrices(rank_id: int, hidden: int = 4096, inter: int = 14336):
    """One Mixtral-shaped expert's w1, w3 [inter, hidden] and w2 [hidden, inter]."""
    return [wl.gen_weight(wl.rng_for("quantize", name, rank_id), n, k)
            for name, n, k in (("w1", inter, hidden), ("w3", inter, hidden), ("w2", hidden, inter))]


def _sgemm_launches(M: int, Nn: int, Kd: int) -> int:
    """Kernels one fp32 product of the quantiser launches: the tiled GEMM, plus
    the in-order sum of its reduction slices when a small output grid splits
    the reduction (64-wide tiles, 128 rows when M >= 128; split when the grid
    has fewer than 148 tiles and Kd >= 2048, at most 8 slices of a multiple of
    16)."""
    TM = 128 if M >= 128 else 64
    tiles = ((Nn + 63) // 64) * ((M + TM - 1) // TM)
    S = min(8, max(1, 296 // tiles)) if tiles < 148 and Kd >= 2048 else 1
    kslice = -(-((Kd + S - 1) // S) // 16) * 16
    return 2 if (Kd + kslice - 1) // kslice > 1 else 1


def quant_launches(shapes, r: int, rounds: int, sketch: int, power_iters: int) -> int:
    """Kernels milo_quantize_lorc launches for matrices of `shapes` [(N, K)]:
    per round the HQQ pack, the error and next target, the error sum and the
    copy of the best round; per compensator the products of the subspace
    iteration, a Gram matrix (two kernels) and a Cholesky factor for every
    basis pass, and the eigen-decomposition."""
    total = 0
    for N, K in shapes:
        if r == 0:
            total += 4
            continue
        l, q = sketch, power_iters
        n = 0

        def orth(M, passes):
            return passes * (3 + _sgemm_launches(M, l, l))

        n += _sgemm_launches(N, l, K) + orth(N, 1 if q > 0 else 2)
        for it in range(q):
            n += _sgemm_launches(K, l, N) + orth(K, 1) + _sgemm_launches(N, l, K) + orth(N, 1 if it + 1 < q else 2)
        n += _sgemm_launches(l, K, N) + 2 + 1 + _sgemm_launches(N, r, l) + _sgemm_launches(r, K, l)
        total += (rounds + 1) * (n + 4)
    return total


def quant_workload(r: int, rounds: int, sketch: int, power_iters: int, hqq_iters: int) -> str:
    return (f"quantise one Mixtral-shaped expert per GPU: w1, w3 [14336, 4096], w2 [4096, 14336]; "
            f"rank {r}, {rounds} refinement rounds, sketch {sketch}, {power_iters} power steps, "
            f"HQQ {hqq_iters} iterations")


def run_quantize_reference(args, rows: int = 256) -> int:
    """--impl reference --workload quantize: the oracle's quantiser as the
    reference arm (rank 0 only).  Each step quantises and compensates the next
    [rows, 4096] slice of the same w1 the GPU arm quantises whole."""
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    import oracle
    r, rounds = args.quant_rank, args.quant_rounds
    sketch = min(128, max(16, 2 * r)) if r > 0 else 0
    W1 = wl.gen_weight(wl.rng_for("quantize", "w1", 0), 14336, 4096)
    steps, warm = max(1, args.steps), max(0, args.warmup)
    times = []
    for s in range(warm + steps):
        lo = (s * rows) % W1.shape[0]
        W = np.ascontiguousarray(W1[lo:lo + rows])
        om = wl.rng_for("quantize", "omega_cpu", s).standard_normal((W.shape[1], sketch))
        t0 = time.perf_counter()
        oracle.quantize_lorc(W, r, rounds, om)
        if s >= warm:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = steps * rows * W1.shape[1] / total
    nthreads = cpu_threads()
    sample = (f"a [{rows}, {W1.shape[1]}] slice of w1 per step (HQQ in C over the host threads, "
              f"the subspace iteration in numpy BLAS)")
    line = {"impl": "reference", "metric": QUANT_METRIC, "value": value, "unit": "weights/s", "n_gpus": world,
            "steps": steps, "warmup": warm, "ms_per_step": 1e3 * total / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": quant_workload(r, rounds, sketch, 2, oracle.HQQ_ITERS), "sample": sample},
            "cpu_baseline": {"value": value, "unit": "weights/s", "cores": nthreads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "weights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def quant_cpu_baseline(r: int, rounds: int, budget_rows: int = 2048) -> dict:
    """The oracle's quantiser on a sampled [budget_rows, 4096] slice of w1."""
    import oracle
    W = np.ascontiguousarray(wl.gen_weight(wl.rng_for("quantize", "w1", 0), 14336, 4096)[:budget_rows])
    rng = wl.rng_for("quantize", "omega_cpu", 0)
    om = rng.standard_normal((W.shape[1], 2 * r))
    t0 = time.perf_counter()
    oracle.quantize_lorc(W, r, rounds, om)
    dt = time.perf_counter() - t0
    return {"value": W.size / dt, "unit": "weights/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"HQQ + rank-{r} compensator + {rounds} rounds on a [{W.shape[0]}, {W.shape[1]}] slice of "
                      f"w1 ({dt:.1f} s; HQQ in C over the host threads, the subspace iteration in numpy BLAS)"}


def run_quantize(args):
    import ctypes as C

    import torch

    import int3_gemm_rank_b200 as milo
    from int3_gemm_rank_b200 import build as milo_build

    rank, local, world = dist_env()
    if not os.path.exists(milo.LIB_PATH):
        milo_build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init("nccl")
    r, rounds = args.quant_rank, args.quant_rounds
    params = milo.lorc_params(r, rounds=rounds)
    L = milo.lib()
    jobs = []
    for i, Wn in enumerate(quant_matrices(rank)):
        N, K = Wn.shape
        W = torch.from_numpy(Wn.view(np.int16)).view(torch.float16).to(dev)
        om = torch.from_numpy(wl.rng_for("quantize", "omega", i).standard_normal((K, params.sketch))
                              .astype(np.float32)).to(dev)
        blob = torch.empty(milo.milo_packed_bytes(N, K), dtype=torch.uint8, device=dev)
        U = torch.empty((N, r), dtype=torch.float16, device=dev)
        V = torch.empty((r, K), dtype=torch.float16, device=dev)
        err = torch.empty(rounds + 1, dtype=torch.float32, device=dev)
        nb = milo.milo_quantize_lorc_workspace(N, K, params)
        ws = torch.empty(nb + 256, dtype=torch.uint8, device=dev)
        wp = ws.data_ptr() + (-ws.data_ptr()) % 256
        jobs.append((N, K, W, om, blob, U, V, err, wp, nb, ws))   # ws stays referenced: wp points into it
    st = milo.new_status(dev)
    sp = C.c_void_p(torch.cuda.current_stream(dev).cuda_stream)

    def step():
        for N, K, W, om, blob, U, V, err, wp, nb, _ws in jobs:
            s = L.milo_quantize_lorc(C.c_void_p(W.data_ptr()), N, K, C.byref(params), C.c_void_p(om.data_ptr()),
                                     C.c_void_p(blob.data_ptr()), C.c_void_p(U.data_ptr()),
                                     C.c_void_p(V.data_ptr()), C.c_void_p(err.data_ptr()), C.c_void_p(wp), nb,
                                     C.c_void_p(st.data_ptr()), sp)
            if s != 0:
                raise RuntimeError(f"milo_quantize_lorc: {L.milo_last_error().decode()}")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} on the quantiser workload")
    clock = ClockSampler(local)
    clock.start()
    barrier(dev)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)
    # the HQQ kernel alone (milo_hqq_pack launches the same kernel on W), on w1
    N1, K1, W1 = jobs[0][0], jobs[0][1], jobs[0][2]
    blob1 = torch.empty_like(jobs[0][4])
    hq = []
    for _ in range(max(3, min(args.steps, 20))):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        L.milo_hqq_pack(C.c_void_p(W1.data_ptr()), None, None, 0, N1, K1, params.hqq_iters,
                        C.c_float(params.hqq_beta), C.c_float(params.hqq_kappa), C.c_void_p(blob1.data_ptr()), None,
                        None, sp)
        b.record()
        hq.append((a, b))
    # the kurtosis reduction of the adaptive-rank policy, on w1 (HBM-bound)
    kws = torch.empty(4 * 592, dtype=torch.float64, device=dev)
    kout = torch.empty(1, dtype=torch.float64, device=dev)
    kt = []
    for _ in range(max(3, min(args.steps, 20))):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        L.milo_kurtosis(C.c_void_p(W1.data_ptr()), N1 * K1, C.c_void_p(kout.data_ptr()), C.c_void_p(kws.data_ptr()),
                        kws.numel() * 8, None, sp)
        b.record()
        kt.append((a, b))
    torch.cuda.synchronize()
    clocks = clock.stop()
    hqq_ms = statistics.median(a.elapsed_time(b) for a, b in hq[1:])
    kurt_ms = statistics.median(a.elapsed_time(b) for a, b in kt[1:])
    kurt_gbs = 2.0 * N1 * K1 / (kurt_ms / 1e3) / 1e9
    weights = sum(j[0] * j[1] for j in jobs)
    sm_mhz = clocks.get("sm_mhz") or 1965.0
    peak = FP32_LANES * sm_mhz * 1e6 / 1e12
    achieved = HQQ_OPS_PER_WEIGHT_ITER * N1 * K1 * params.hqq_iters / (hqq_ms / 1e3) / 1e12
    line = {
        "metric": QUANT_METRIC, "value": weights * world / (ms / 1e3), "unit": "weights/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": quant_workload(r, rounds, params.sketch, params.power_iters, params.hqq_iters),
                   "l2": "inputs larger than L2 (117 MB fp16 weight plus its 235 MB fp32 residual per matrix)",
                   "parallelism": f"replica per GPU x{world}"},
        "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "Top/s", "frac": achieved / peak,
                     "traffic": None, "kernel": "hqq_pack_kernel (HQQ zero-point fit + pack, w1 shape)",
                     "algorithmic_ops_per_launch": HQQ_OPS_PER_WEIGHT_ITER * N1 * K1 * params.hqq_iters,
                     "ms_per_launch": hqq_ms,
                     "peak_source": "derived: 148 SMs x 128 fp32 lanes x the sampled SM clock"},
        "kernels": {"hqq_pack_ms": hqq_ms, "kurtosis_ms": kurt_ms, "kurtosis_gbs": kurt_gbs,
                    "kurtosis_frac_hbm": kurt_gbs / peaks()["hbm_gbs"]},
        "gpu_launches": quant_launches([(j[0], j[1]) for j in jobs], r, rounds if r > 0 else 0, params.sketch,
                                       params.power_iters) * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = quant_cpu_baseline(r, rounds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("milo", "reference"), default="milo")
    ap.add_argument("--workload", choices=("mixtral", "deepseek", "prefill", "single", "quantize", "sweep"),
                    default="mixtral",
                    help="single: one 1024 x 1024 expert with a rank-16 compensator, 1 token; quantize: the "
                         "offline quantiser on one Mixtral-shaped expert; sweep: the w1 projection over "
                         "1 ... 1024 Zipf-routed tokens (each its own JSON line)")
    ap.add_argument("--quant-rank", type=int, default=32)
    ap.add_argument("--quant-rounds", type=int, default=3)
    ap.add_argument("--soak", type=float, default=1.0, help="seconds of untimed load before timing")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--lorc", choices=("fp16", "int3"), default="fp16",
                    help="compensator format: fp16 U, V (the configured workloads) or int3 blobs")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch the step's kernels one by one instead of replaying one CUDA graph")
    ap.add_argument("--experts", type=int, default=None, help="routed experts (profiler captures)")
    ap.add_argument("--tokens", type=int, default=None, help="tokens per step (profiler captures)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.workload == "quantize":
        if args.impl == "reference":
            return run_quantize_reference(args)
        return run_quantize(args)
    if args.workload == "single":
        if args.impl == "reference":
            return run_single_reference(args)
        return run_single(args)
    if args.workload == "sweep":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the reference arm covers the layer forward "
                              "and the quantiser; the sweep's parity is in the GPU tests"}))
            return 0
        return run_sweep(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_milo(args)


if __name__ == "__main__":
    sys.exit(main())
