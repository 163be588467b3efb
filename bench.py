"""Benchmark of the DSA decode step (lightning indexer + top-k + sparse latent
attention) on B200, one process per GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 4] [--no-cpu-baseline]

A step is one decode step of the whole batch (B sequences) of the chosen
workload (default: B = 8 sequences at 131072 tokens, the 128K-context case):
rotate/quantise the new queries and key, append the key, score every cached
key, select the top 2048, run the sparse latent attention.  Under torchrun each
rank runs its own batch (independent sequences, no collective on the data
path: weak scaling); the timed region is bracketed by a barrier and a device
synchronise, and the slowest rank's time counts.

Rank 0 prints ONE JSON line.  `--impl reference` times the CPU oracle instead
(the only reference implementation there is), on a bounded sample of the same
workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

import workloads

ROOT = os.path.dirname(os.path.abspath(__file__))
N_COPIES = 3            # rotating device copies of the decode state (each > L2)


# Source files of the dominant kernel (the indexer scorer); the committed ncu
# summary records their hash, so its DRAM traffic is reported only while the
# kernel is unchanged.
SCORER_SOURCES = ("top_kv_selection_b200/csrc/index_scores.cu", "top_kv_selection_b200/csrc/scorer.cuh",
                  "top_kv_selection_b200/csrc/quant.cuh", "top_kv_selection_b200/csrc/tc_ptx.cuh",
                  "top_kv_selection_b200/csrc/common.cuh")
SCORER_PROFILE = "profiles/index_scores_decode_B8_T131072.md"


def scorer_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in SCORER_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per scorer launch from the committed ncu summary, or None if
    the summary is missing or was taken on different kernel sources."""
    path = os.path.join(ROOT, SCORER_PROFILE)
    if not os.path.exists(path):
        return None
    fields = {}
    for line in open(path):
        if ":" in line and line.startswith("- "):
            k, v = line[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    if fields.get("source_sha256") != scorer_source_hash():
        return None
    try:
        return float(fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# --------------------------------------------------------------------------- #
# distributed plumbing
# --------------------------------------------------------------------------- #
def _dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(world, value: float) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64,
                     device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------- #
# clocks sampled during the timed region
# --------------------------------------------------------------------------- #
class ClockSampler:
    """Polls NVML (SM clock, max SM clock, clock-event reasons) in a background
    thread for as long as the context is open; open it around the timed region."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.dev = device_index
        self.samples = []
        self.max_mhz = None
        self._stop = False
        self._thread = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        p = torch.cuda.get_device_properties(self.dev)
        try:
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def _run(self, h):
        import pynvml
        while not self._stop:
            try:
                clk = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((clk, rs))
            except Exception:
                break
            time.sleep(0.001)

    def __enter__(self):
        import threading
        try:
            import pynvml
            h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, args=(h,), daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
        return self

    def __exit__(self, *exc):
        self._stop = True
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = set()
        for _, rs in self.samples:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(c for c, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(self.samples), "source": "nvml"}


# --------------------------------------------------------------------------- #
# device state of the decode step
# --------------------------------------------------------------------------- #
def build_state(dsa, wl, rank_seed_offset=0, n_copies=N_COPIES):
    """Device state for one decode step of wl (B sequences), n_copies rotating copies."""
    dev = "cuda"
    B, T = wl.B, wl.T
    dt = torch.bfloat16 if wl.attn_dtype == "bf16" else torch.float32
    k_cache = torch.empty(B, T, wl.D, dtype=torch.uint8, device=dev)
    k_scale = torch.empty(B, T, dtype=torch.float32, device=dev)
    kv = torch.empty(B, T, wl.dqk, dtype=dt, device=dev)
    q_idx = torch.empty(B, wl.H, wl.D, device=dev)
    w = torch.empty(B, wl.H, device=dev)
    k_new = torch.empty(B, wl.D, device=dev)
    q_mla = torch.empty(B, wl.Hq, wl.dqk, dtype=dt, device=dev)
    for b in range(B):
        s = workloads.decode_sequence(wl, b + rank_seed_offset)
        dsa.dsa_indexer_quant(s["keys"][:T - 1].to(dev), k_cache[b], k_scale[b])
        kv[b] = s["kv"].to(dev)
        q_idx[b] = s["q_idx"].to(dev)
        w[b] = s["w"].to(dev)
        k_new[b] = s["keys"][T - 1].to(dev)
        q_mla[b] = s["q_mla"].to(dev)
        del s
    K = wl.K
    dtc = dsa.DSA_BF16 if dt == torch.bfloat16 else dsa.DSA_F32
    need = dsa.dsa_decode_step_workspace_size(B, wl.H, wl.D, T, wl.topk, wl.Hq, wl.dc, wl.dr, dtc)
    copies = []
    for c in range(n_copies):
        copies.append(dict(
            k_cache=k_cache if c == 0 else k_cache.clone(),
            k_scale=k_scale if c == 0 else k_scale.clone(),
            kv=kv if c == 0 else kv.clone(),
            q_idx=q_idx.clone(), w=w.clone(), k_new=k_new.clone(), q_mla=q_mla.clone(),
            idx=torch.empty(B, K, dtype=torch.int32, device=dev),
            out=torch.empty(B, wl.Hq, wl.dc, dtype=dt, device=dev),
            lse=torch.empty(B, wl.Hq, dtype=torch.float32, device=dev),
            ws=torch.empty(need, dtype=torch.uint8, device=dev), T=T))
    return copies


def decode_step(dsa, wl, st, stream=None):
    dsa.dsa_decode_step(st["q_idx"], st["w"], st["k_new"], st["k_cache"], st["k_scale"],
                        st["kv"], st["q_mla"], st["T"], wl.topk, wl.softmax_scale_idx,
                        wl.sm_scale, st["idx"], st["out"], st["lse"], st["ws"], stream=stream)


def count_launches_per_step(wl, dsa, st) -> tuple[int, list[str]]:
    """Kernels one decode step launches, counted by the profiler on an untimed step."""
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        decode_step(dsa, wl, st)
        torch.cuda.synchronize()
    names = [e.name for e in prof.events() if e.device_type.name == "CUDA"
             and "memcpy" not in e.name.lower() and "memset" not in e.name.lower()]
    return len(names), sorted(set(names))


# --------------------------------------------------------------------------- #
# dominant kernel: the indexer scorer, timed alone on the same inputs
# --------------------------------------------------------------------------- #
def time_stages(dsa, wl, copies, iters):
    """Average device time of each stage of the decode step, each launched
    through its own entry point on the same inputs, with CUDA events on the
    launching stream and the state copies rotating as in the timed steps.
    Returns {stage: seconds per launch}; "decode_index_scores" is the dominant kernel."""
    dev = "cuda"
    B, T = wl.B, wl.T
    scores = torch.empty(B, 1, T, dtype=torch.float32, device=dev)
    scores2d = scores.view(B, T)
    idx = torch.empty(B, 1, wl.K, dtype=torch.int32, device=dev)
    dt = dsa.DSA_BF16 if wl.attn_dtype == "bf16" else dsa.DSA_F32
    ws = torch.empty(max(1, dsa.dsa_sparse_mla_attn_workspace_size(B, 1, wl.Hq, wl.dc, wl.dr,
                                                                    wl.K, dt)),
                     dtype=torch.uint8, device=dev)
    q_mla = copies[0]["q_mla"].reshape(B, 1, wl.Hq, wl.dqk).contiguous()
    out = torch.empty(B, 1, wl.Hq, wl.dc, dtype=copies[0]["out"].dtype, device=dev)
    lse = torch.empty(B, 1, wl.Hq, dtype=torch.float32, device=dev)

    def score(st):
        # the indexer half of the step, the same kernel the decode step launches
        dsa.dsa_decode_index_scores(st["q_idx"], st["w"], st["k_new"], st["k_cache"],
                                    st["k_scale"], T, wl.softmax_scale_idx, scores2d)

    def topk(st):
        dsa.dsa_topk_select(scores, T - 1, wl.topk, idx)

    def attn(st):
        dsa.dsa_sparse_mla_attn(q_mla, st["kv"], idx, T - 1, wl.sm_scale, out, lse, ws)

    stream = torch.cuda.current_stream()
    result = {}
    for name, fn in (("decode_index_scores", score), ("topk_select", topk),
                     ("sparse_mla_attn", attn)):
        for i in range(3):
            fn(copies[i % len(copies)])
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(iters):
            fn(copies[i % len(copies)])
        t1.record(stream)
        t1.synchronize()
        result[name] = t0.elapsed_time(t1) / iters * 1e-3
    return result


# --------------------------------------------------------------------------- #
# the CPU oracle as a baseline (bounded sample)
# --------------------------------------------------------------------------- #
def oracle_decode_sample(wl, n_seq: int, repeats: int = 1):
    """Time the oracle's per-step work (quantise q and the new key, score the
    T cached keys, select, attend) on n_seq sequences; the cache itself is
    quantised once, untimed, as a decode cache would already hold it."""
    import oracle
    per_seq = []
    for b in range(n_seq):
        s = workloads.decode_sequence(wl, b)
        keys = s["keys"].numpy()
        T = keys.shape[0]
        k_fp8, k_sc = oracle.indexer_quant(keys[:T - 1])
        k_fp8 = np.concatenate([k_fp8, np.zeros((1, wl.D), np.uint8)])[None]
        k_sc = np.concatenate([k_sc, np.zeros(1, np.float32)])[None]
        q_mla = s["q_mla"].float().numpy()[None, None]
        kv = s["kv"].float().numpy()[None]
        for _ in range(repeats):
            t0 = time.perf_counter()
            nk, ns = oracle.indexer_quant(keys[T - 1:T])
            k_fp8[0, T - 1], k_sc[0, T - 1] = nk[0], ns[0]
            qf, qs = oracle.indexer_quant(s["q_idx"].numpy())
            sc = oracle.index_scores(qf[None, None], qs[None, None], s["w"].numpy()[None, None],
                                     k_fp8, k_sc, T - 1, T, wl.softmax_scale_idx)
            idx = oracle.topk_select(sc, T - 1, wl.topk)
            oracle.sparse_mla(q_mla, kv, idx, T - 1, wl.sm_scale, wl.dc)
            per_seq.append(time.perf_counter() - t0)
    return per_seq


def bench_config(wl, world):
    """The workload description both arms print (identical dicts)."""
    return {"workload": wl.name, "B": wl.B, "T": wl.T, "H": wl.H, "D": wl.D, "topk": wl.topk,
            "Hq": wl.Hq, "dc": wl.dc, "dr": wl.dr,
            "l2": "inputs larger than L2 (a decode state is 1.4 GB)",
            "parallelism": f"dp{world} (independent batches per rank)"}


def run_reference(args, wl, world, rank):
    if rank != 0:
        return
    # One timed step of the reference arm is a bounded sample of the workload:
    # the oracle's decode pass for ONE sequence of the batch (sequences are
    # independent and alike).  ms_per_step is that timed work; the metric,
    # steps/s of the whole B-sequence step, is 1 / (B * t_seq).
    if args.warmup:
        oracle_decode_sample(wl, 1, repeats=max(args.warmup, 0))
    times = []
    for k in range(args.steps):
        times += oracle_decode_sample(wl, 1, repeats=1)
    t_seq = sum(times) / len(times)
    value = 1.0 / (wl.B * t_seq)
    line = {
        "metric": "dsa_decode_steps_per_s", "value": value, "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_seq * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": bench_config(wl, world),
        "timed_step": f"one of the {wl.B} sequences of a decode step per timed step "
                      f"(ms_per_step); value = 1 / ({wl.B} x that time)",
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": 1, "kind": "oracle",
                         "sample": f"sequence 0 of {wl.B}, one decode step per timed step "
                                   f"(T={wl.T}), extrapolated x{wl.B}; cache prebuilt"},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "indexer_gscores_per_s": wl.T / t_seq / 1e9,
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- #
# our arm
# --------------------------------------------------------------------------- #
def bind_local_cpus(device_index: int) -> list | None:
    """Restrict this process to the CPUs NVML reports as local to the GPU (its
    NUMA node), as a serving process is placed: pinned host buffers are then
    allocated, and the copies and launches issued, next to the GPU's PCIe root.
    Best effort: returns the CPU list, or None when NVML or the affinity call is
    unavailable.  Reads only; changes no GPU setting."""
    try:
        import pynvml
        pynvml.nvmlInit()
        p = torch.cuda.get_device_properties(device_index)
        try:
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
        n_words = (os.cpu_count() + 63) // 64
        words = pynvml.nvmlDeviceGetCpuAffinity(h, n_words)
        cpus = [64 * i + b for i, w in enumerate(words) for b in range(64) if (w >> b) & 1]
        cpus = [c for c in cpus if c < os.cpu_count()]
        if not cpus:
            return None
        os.sched_setaffinity(0, cpus)
        return cpus
    except Exception:
        return None


def run_ours(args, wl, world, rank, local):
    import __graft_entry__
    __graft_entry__._builder().build()
    import top_kv_selection_b200 as dsa

    local_cpus = bind_local_cpus(torch.cuda.current_device())

    # every rank draws its own independent sequences
    copies = build_state(dsa, wl, rank_seed_offset=rank * wl.B, n_copies=args.copies)
    torch.cuda.synchronize()
    per_step_launches, kernel_names = count_launches_per_step(wl, dsa, copies[0])

    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        decode_step(dsa, wl, copies[i % len(copies)])
    torch.cuda.synchronize()
    if dsa.dsa_get_device_error() != 0:
        raise RuntimeError("device error word set during warm-up")

    # the steps run as a decode server issues them: a CUDA graph of
    # graph_steps consecutive steps (the copies in rotation) replayed, the last
    # steps % graph_steps launched directly
    graph_steps = len(copies) * max(1, 12 // len(copies))
    graph = None
    if not args.eager and args.steps >= graph_steps:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(graph_steps):
                decode_step(dsa, wl, copies[i % len(copies)])
        graph.replay()                                  # untimed
        torch.cuda.synchronize()
    n_replays = args.steps // graph_steps if graph is not None else 0
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        start.record(stream)
        for _ in range(n_replays):
            graph.replay()
        for i in range(n_replays * graph_steps, args.steps):
            decode_step(dsa, wl, copies[i % len(copies)])
        end.record(stream)
        end.synchronize()
    torch.cuda.synchronize()
    _barrier(world)
    if dsa.dsa_get_device_error() != 0:
        raise RuntimeError("device error word set during the timed steps")
    elapsed = start.elapsed_time(end) * 1e-3
    elapsed = _max_over_ranks(world, elapsed)
    ms_per_step = elapsed / args.steps * 1e3
    value = world * args.steps / elapsed
    gscores = world * args.steps * wl.B * wl.T / elapsed / 1e9

    del graph
    # the same steps launched one by one (reported beside the graph-replayed figure)
    eager_ms = None
    if n_replays:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            decode_step(dsa, wl, copies[i % len(copies)])
        e1.record(stream)
        e1.synchronize()
        eager_ms = _max_over_ranks(world, e0.elapsed_time(e1) * 1e-3) / args.steps * 1e3

    # e2e: per-step inputs from pinned host memory, result back to the host
    e2e = run_e2e(dsa, wl, copies, args, world)

    # dominant kernel roofline (indexer scorer over the full cache)
    peak, peak_kind = _peaks()
    stages = time_stages(dsa, wl, copies, iters=max(10, min(args.steps, 500)))
    t_score = stages["decode_index_scores"]
    prefill = prologue = attn_fp8 = None
    prefill_chain = None
    if not args.no_prefill:
        prefill = time_prefill_scoring(dsa, measure_fp8_peak(sustained=False)["fp8_e4m3_tflops"])
        prologue = time_indexer_prologue(dsa, peak)
        try:
            prefill_chain = time_prefill_chain(dsa, peak)
        except Exception as exc:                   # reported, never fatal to the main line
            prefill_chain = {"error": f"{type(exc).__name__}: {exc}"[:200]}
    try:
        attn_fp8 = time_sparse_mla_fp8(dsa, peak, wl)
    except Exception as exc:                       # reported, never fatal to the main line
        attn_fp8 = {"error": f"{type(exc).__name__}: {exc}"[:200]}
    try:
        csa = time_csa_decode(dsa, peak, wl)
    except Exception as exc:                       # reported, never fatal to the main line
        csa = {"error": f"{type(exc).__name__}: {exc}"[:200]}
    # keys + scales of every cached token, plus the new tokens' fp32 queries,
    # weights and keys (the scores written are not algorithmic)
    score_bytes = wl.B * wl.T * (wl.D + 4) + wl.B * (wl.H * wl.D * 4 + wl.H * 4 + wl.D * 4)
    achieved = score_bytes / t_score / 1e9
    step_bytes = wl.B * (wl.T * (wl.D + 4) + wl.K * wl.dqk * 2 + wl.H * wl.D * 4
                         + wl.Hq * wl.dqk * 2 + wl.Hq * wl.dc * 2)

    line = {
        "metric": "dsa_decode_steps_per_s", "value": value, "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8_e4m3+bf16", "data": "synthetic",
        "config": bench_config(wl, world),
        "l2_detail": f"{len(copies)} rotating decode-state copies, each larger than L2",
        "launch": (f"CUDA graph of {graph_steps} steps replayed {n_replays}x"
                   + (f" + {args.steps - n_replays * graph_steps} direct" if
                      args.steps % graph_steps else "") if n_replays else "direct launches"),
        "eager_ms_per_step": eager_ms,
        # the scorer kernel's own rate (cached tokens scored per second), and the
        # same count over the whole step
        "indexer_gscores_per_s": wl.B * wl.T / t_score / 1e9,
        "indexer_gscores_roofline": peak * 1e9 / (wl.D + 4) / 1e9,
        "step_gscores_per_s": gscores,
        "step_roofline": {"bytes": step_bytes, "achieved_gbs": step_bytes / (ms_per_step * 1e-3)
                          / 1e9, "frac": step_bytes / (ms_per_step * 1e-3) / 1e9 / peak},
        "roofline": {"kernel": "decode_index_scores", "bound": "hbm", "achieved": achieved,
                     "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs", "unit": "GB/s",
                     "frac": achieved / peak, "traffic": profiled_traffic(),
                     "avg_launch_us": t_score * 1e6},
        "e2e": e2e,
        "host_cpus": (f"{len(local_cpus)} GPU-local CPUs (NVML affinity)" if local_cpus
                      else "not bound"),
        "gpu_launches": per_step_launches * args.steps,
        "kernels_per_step": per_step_launches, "kernels": kernel_names,
        "stage_us": {k: round(v * 1e6, 2) for k, v in stages.items()},
        "prefill_scoring": prefill,
        "indexer_prologue": prologue,
        "prefill_chain": prefill_chain,
        "sparse_mla_fp8": attn_fp8,
        "csa_indexer": csa,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        times = oracle_decode_sample(wl, wl.B)
        t_step = sum(times)
        line["cpu_baseline"] = {
            "value": 1.0 / t_step, "unit": "steps/s", "cores": 1, "kind": "oracle",
            "sample": f"all {wl.B} sequences of one decode step at T={wl.T} "
                      f"({t_step:.1f} s, single thread); caches prebuilt, untimed"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(dsa, wl, copies, args, world, graph_steps=12):
    """Same step through the public API with host buffers.  Every step's inputs
    are copied from pinned host memory and its selections and output read back
    into pinned host memory, inside the timed region; as a serving loop would,
    the copies run on their own streams (host-to-device, device-to-host) and
    overlap the neighbouring steps' kernels.  Events order each device state's
    reuse: the inputs of step i are written once step i - n (same state) has
    read them, and step i's kernels start once step i - n's results have been
    read back.  `graph_steps` steps (copies, calls and events) are captured in
    a CUDA graph and replayed, as a decode server replays its step graph; if
    the capture fails the same loop runs eagerly."""
    n = len(copies)
    st = copies[0]
    host_in = {k: st[k].cpu().pin_memory() for k in ("q_idx", "w", "k_new", "q_mla")}
    new_row = st["kv"][:, wl.T - 1].contiguous().cpu().pin_memory()
    host_idx = [torch.empty(st["idx"].shape, dtype=torch.int32).pin_memory() for _ in range(n)]
    host_out = [torch.empty(st["out"].shape, dtype=st["out"].dtype).pin_memory() for _ in range(n)]
    row_dev = [torch.empty_like(new_row, device="cuda") for _ in range(n)]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values()) + \
        new_row.numel() * new_row.element_size()
    d2h = host_idx[0].numel() * 4 + host_out[0].numel() * host_out[0].element_size()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def steps(count):
        compute = torch.cuda.current_stream()
        up.wait_stream(compute)
        down.wait_stream(compute)
        in_read, out_read = [None] * n, [None] * n
        for i in range(count):
            j = i % n
            s = copies[j]
            with torch.cuda.stream(up):
                if in_read[j] is not None:
                    up.wait_event(in_read[j])
                for k, t in host_in.items():
                    s[k].copy_(t, non_blocking=True)
                row_dev[j].copy_(new_row, non_blocking=True)
                s["kv"][:, wl.T - 1].copy_(row_dev[j])
                inputs = torch.cuda.Event()
                inputs.record(up)
            compute.wait_event(inputs)
            if out_read[j] is not None:
                compute.wait_event(out_read[j])
            decode_step(dsa, wl, s, stream=compute)
            done = torch.cuda.Event()
            done.record(compute)
            in_read[j] = done
            with torch.cuda.stream(down):
                down.wait_event(done)
                host_idx[j].copy_(s["idx"], non_blocking=True)
                host_out[j].copy_(s["out"], non_blocking=True)
                back = torch.cuda.Event()
                back.record(down)
            out_read[j] = back
        compute.wait_stream(up)
        compute.wait_stream(down)

    steps(max(args.warmup, n))
    torch.cuda.synchronize()
    graph = None
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            steps(graph_steps)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        if dsa.dsa_get_device_error() == 0:
            graph = g
    except Exception:                           # the eager loop below instead
        torch.cuda.synchronize()
    reps = max(1, -(-args.steps // graph_steps)) if graph is not None else 0
    n_steps = reps * graph_steps if graph is not None else args.steps
    stream = torch.cuda.current_stream()
    _barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    if graph is not None:
        for _ in range(reps):
            graph.replay()
    else:
        steps(n_steps)
    t1.record(stream)
    t1.synchronize()
    el = _max_over_ranks(world, t0.elapsed_time(t1) * 1e-3)
    return {"value": world * n_steps / el, "unit": "steps/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n_steps,
            "how": (f"CUDA graph of {graph_steps} steps replayed {reps} times" if graph is not None
                    else "eager loop (graph capture failed)") +
                   "; copies on their own streams, overlapping the neighbouring steps' kernels"}


def time_prefill_scoring(dsa, fp8_peak, iters=10):
    """Indexer scoring of the causal prefill (T = 8192 queries against their own
    8192 keys, 64 heads x 128, FP8): the FP8 tensor-bound workload.  Algorithmic
    work = the causal (query, key) pairs only: T(T+1)/2 x H x D x 2 flop.  The
    inputs are seeded random normals made on the device (performance only)."""
    wl = workloads.WORKLOADS[3]
    T, H, D = wl.T, wl.H, wl.D
    g = torch.Generator(device="cuda").manual_seed(wl.seed(0))
    q = torch.randn(1, T, H, D, device="cuda", generator=g)
    w = torch.randn(1, T, H, device="cuda", generator=g)
    keys = torch.randn(1, T, D, device="cuda", generator=g)
    q_fp8 = torch.empty(1, T, H, D, dtype=torch.uint8, device="cuda")
    q_scale = torch.empty(1, T, H, dtype=torch.float32, device="cuda")
    k_cache = torch.empty(1, T, D, dtype=torch.uint8, device="cuda")
    k_scale = torch.empty(1, T, dtype=torch.float32, device="cuda")
    dsa.dsa_indexer_quant(q, q_fp8, q_scale)
    dsa.dsa_indexer_quant(keys, k_cache, k_scale, n_rows=1, out_row_stride=T * D,
                          scale_row_stride=T)
    del q, keys
    scores = torch.empty(1, T, T, dtype=torch.float32, device="cuda")

    def one():
        dsa.dsa_index_scores(q_fp8, q_scale, w, k_cache, k_scale, 0, T, wl.softmax_scale_idx,
                             scores)

    for _ in range(3):
        one()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(iters):
        one()
    t1.record()
    t1.synchronize()
    t = t0.elapsed_time(t1) * 1e-3 / iters
    flop = T * (T + 1) // 2 * H * D * 2
    out = {"workload": wl.name, "queries": T, "keys": T, "gflop": flop / 1e9, "us": t * 1e6,
           "tflops": flop / t / 1e12, "fp8_peak_tflops": fp8_peak, "frac": flop / t / 1e12 / fp8_peak,
           "peak_kind": "measured in this run: torch._scaled_mm e4m3 8192^3, burst",
           "note": "causal pairs only; the -inf scores of masked positions are written too"}
    del scores
    return out


def time_indexer_prologue(dsa, peak_gbs, iters=20):
    """The fused indexer prologue (RoPE on 64 of 128 dims, not interleaved ->
    rotate_activation -> act_quant -> key cache append) over the queries and keys
    of the T = 8192 prefill, bf16 inputs as a projection produces them.  HBM-bound:
    algorithmic bytes = the bf16 inputs, the codes and scales written and the
    rotary table; 2 inputs + outputs > 126 MB of L2, so every launch streams."""
    wl = workloads.WORKLOADS[3]
    T, H, D, R = wl.T, wl.H, wl.D, 64
    g = torch.Generator(device="cuda").manual_seed(wl.seed(1))
    q = torch.randn(1, T, H, D, device="cuda", generator=g).to(torch.bfloat16)
    k = torch.randn(1, T, D, device="cuda", generator=g).to(torch.bfloat16)
    th = torch.rand(T, R // 2, device="cuda", generator=g) * 6.283185307179586
    cs = torch.stack([torch.cos(th), torch.sin(th)], dim=-1).contiguous()
    q_fp8 = torch.empty(1, T, H, D, dtype=torch.uint8, device="cuda")
    q_scale = torch.empty(1, T, H, dtype=torch.float32, device="cuda")
    k_cache = torch.empty(1, T, D, dtype=torch.uint8, device="cuda")
    k_scale = torch.empty(1, T, dtype=torch.float32, device="cuda")

    def one():
        dsa.dsa_indexer_prologue(q, k, cs, 0, q_fp8, q_scale, k_cache, k_scale)

    for _ in range(3):
        one()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(iters):
        one()
    t1.record()
    t1.synchronize()
    t = t0.elapsed_time(t1) * 1e-3 / iters
    nbytes = T * (H + 1) * (2 * D + D + 4) + T * (R // 2) * 8
    out = {"workload": "prefill_T8192_bf16_rope64", "vectors": T * (H + 1), "bytes": nbytes,
           "us": t * 1e6, "achieved_gbs": nbytes / t / 1e9, "peak_gbs": peak_gbs,
           "frac": nbytes / t / 1e9 / peak_gbs, "bound": "hbm"}
    del q, k, q_fp8, k_cache
    return out


def time_csa_decode(dsa, peak_gbs, wl, m=4, iters=20, copies=3):
    """The V4 CSA indexer at the decode workload's sizes: B sequences of T tokens
    compressed at rate m into T / m entries, 64 heads x 128, k = 2048 over the
    entries: dsa_index_scores_csa then dsa_topk_select_csa, timed together and
    the scorer alone.  Rotating entry caches (each B x T/m x 132 B) are seeded
    random normals made on the device (performance only).  Algorithmic bytes of
    the scorer: the entries' keys and scales plus the queries."""
    B, H, D, k = wl.B, wl.H, wl.D, wl.topk
    E = wl.T // m
    sp = wl.T - 1
    g = torch.Generator(device="cuda").manual_seed(wl.seed(5))
    states = []
    for _ in range(copies):
        keys = torch.randn(B, E, D, device="cuda", generator=g)
        kf = torch.empty(B, E, D, dtype=torch.uint8, device="cuda")
        ksc = torch.empty(B, E, dtype=torch.float32, device="cuda")
        dsa.dsa_indexer_quant(keys, kf, ksc, n_rows=B, out_row_stride=E * D, scale_row_stride=E)
        del keys
        q = torch.randn(B, 1, H, D, device="cuda", generator=g)
        qf = torch.empty(B, 1, H, D, dtype=torch.uint8, device="cuda")
        qs = torch.empty(B, 1, H, dtype=torch.float32, device="cuda")
        dsa.dsa_indexer_quant(q, qf, qs)
        w = torch.randn(B, 1, H, device="cuda", generator=g)
        states.append((qf, qs, w, kf, ksc))
    scores = torch.empty(B, 1, E, dtype=torch.float32, device="cuda")
    idx = torch.empty(B, 1, min(k, E), dtype=torch.int32, device="cuda")
    ws = torch.empty(max(1, dsa.dsa_topk_select_workspace_size(B, 1, E, k)), dtype=torch.uint8,
                     device="cuda")

    def score(i):
        qf, qs, w, kf, ksc = states[i % copies]
        dsa.dsa_index_scores_csa(qf, qs, w, kf, ksc, sp, E, m, wl.softmax_scale_idx, scores)

    def both(i):
        score(i)
        dsa.dsa_topk_select_csa(scores, sp, m, k, idx, ws)

    def timed(fn):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for i in range(iters):
            fn(i)
        t1.record()
        t1.synchronize()
        return t0.elapsed_time(t1) * 1e-3 / iters

    t_sc, t_both = timed(score), timed(both)
    nbytes = B * E * (D + 4) + B * H * (D + 8)
    return {"workload": f"{wl.name}_csa_m{m}", "entries": E, "compress": m, "k": k,
            "scores_us": t_sc * 1e6, "scores_plus_topk_us": t_both * 1e6, "scorer_bytes": nbytes,
            "achieved_gbs": nbytes / t_sc / 1e9, "peak_gbs": peak_gbs,
            "frac": nbytes / t_sc / 1e9 / peak_gbs, "bound": "hbm",
            "note": "entry keys are an input (the compressor is not on the pages); "
                    "top-k over (start_pos + 1) // m available entries"}


BF16_FALLBACK_TFLOPS = 1590.0


def _bf16_peak():
    """Dense bf16 tensor peak (TFLOP/s) for the prefill attention's roofline:
    the driver's measured cuBLAS figure when present, else the pool's earlier
    measurement."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        for key in ("bf16_tflops", "bf16_tflops_burst"):
            if key in p:
                return float(p[key]), "measured"
    return BF16_FALLBACK_TFLOPS, "fallback"


def time_prefill_chain(dsa, hbm_peak, iters=3):
    """The causal prefill of one T = 8192 sequence end to end on the device:
    the fused indexer prologue (RoPE, rotate_activation, act_quant, key cache
    write), the causal index scores (64 heads x 128, FP8), the per-row top-2048
    and the sparse MLA attention (128 heads over the selected latent rows,
    512 + 64 bf16).  Every stage is timed on its own with CUDA events, then the
    four back to back.  Inputs are seeded random normals made on the device
    (performance only; parity is the tests' job).

    Rooflines: the top-k reads the causal scores and writes the selections
    (HBM-bound); the attention's algorithmic work is the valid (query, selected
    row) pairs, sum_s min(s + 1, 2048), times 128 heads x (576 + 512) x 2 flop
    = 4.09 TFLOP, against the dense bf16 tensor peak."""
    wl = workloads.WORKLOADS[3]
    T, H, D, R = wl.T, wl.H, wl.D, 64
    Hq, dc, dr, k = wl.Hq, wl.dc, wl.dr, wl.topk
    dev = "cuda"
    g = torch.Generator(device=dev).manual_seed(wl.seed(3))
    q = torch.randn(1, T, H, D, device=dev, generator=g).to(torch.bfloat16)
    keys = torch.randn(1, T, D, device=dev, generator=g).to(torch.bfloat16)
    th = torch.rand(T, R // 2, device=dev, generator=g) * 6.283185307179586
    cs = torch.stack([torch.cos(th), torch.sin(th)], dim=-1).contiguous()
    w = torch.randn(1, T, H, device=dev, generator=g)
    q_fp8 = torch.empty(1, T, H, D, dtype=torch.uint8, device=dev)
    q_scale = torch.empty(1, T, H, dtype=torch.float32, device=dev)
    k_cache = torch.empty(1, T, D, dtype=torch.uint8, device=dev)
    k_scale = torch.empty(1, T, dtype=torch.float32, device=dev)
    scores = torch.empty(1, T, T, dtype=torch.float32, device=dev)
    idx = torch.empty(1, T, k, dtype=torch.int32, device=dev)
    topk_ws = torch.empty(max(1, dsa.dsa_topk_select_workspace_size(1, T, T, k)), dtype=torch.uint8,
                          device=dev)
    kv = torch.randn(1, T, dc + dr, device=dev, generator=g).to(torch.bfloat16)
    q_mla = torch.empty(1, T, Hq, dc + dr, dtype=torch.bfloat16, device=dev)
    for s0 in range(0, T, 1024):                       # 1.2 GB of queries, made in slices
        q_mla[:, s0:s0 + 1024] = torch.randn(1, min(1024, T - s0), Hq, dc + dr, device=dev,
                                             generator=g).to(torch.bfloat16)
    out = torch.empty(1, T, Hq, dc, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(1, T, Hq, dtype=torch.float32, device=dev)
    attn_ws = torch.empty(max(1, dsa.dsa_sparse_mla_attn_workspace_size(1, T, Hq, dc, dr, k,
                                                                        dsa.DSA_BF16)),
                          dtype=torch.uint8, device=dev)

    def prologue():
        dsa.dsa_indexer_prologue(q, keys, cs, 0, q_fp8, q_scale, k_cache, k_scale)

    def score():
        dsa.dsa_index_scores(q_fp8, q_scale, w, k_cache, k_scale, 0, T, wl.softmax_scale_idx, scores)

    def topk():
        dsa.dsa_topk_select(scores, 0, k, idx, topk_ws)

    def attn():
        dsa.dsa_sparse_mla_attn(q_mla, kv, idx, 0, wl.sm_scale, out, lse, attn_ws)

    def chain():
        prologue()
        score()
        topk()
        attn()

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(iters):
            fn()
        t1.record()
        t1.synchronize()
        return t0.elapsed_time(t1) * 1e-3 / iters

    t_pro, t_sc, t_tk, t_at, t_ch = (timed(f) for f in (prologue, score, topk, attn, chain))
    if dsa.dsa_get_device_error() != 0:
        raise RuntimeError("device error word set during the prefill chain")
    bf16_peak, bf16_kind = _bf16_peak()
    pairs = sum(min(s + 1, k) for s in range(T))
    attn_flop = pairs * Hq * (dc + dr + dc) * 2
    topk_bytes = T * (T + 1) // 2 * 4 + T * k * 4
    res = {
        "workload": wl.name, "T": T, "k": k,
        "prologue_us": t_pro * 1e6, "scores_us": t_sc * 1e6,
        "topk": {"rows": T, "positions": T, "k": k, "us": t_tk * 1e6, "bytes": topk_bytes,
                 "achieved_gbs": topk_bytes / t_tk / 1e9, "peak_gbs": hbm_peak,
                 "frac": topk_bytes / t_tk / 1e9 / hbm_peak, "bound": "hbm",
                 "note": "bytes = the causal scores read once + the selections written"},
        "sparse_mla": {"queries": T, "selected_pairs": pairs, "tflop": attn_flop / 1e12,
                       "us": t_at * 1e6, "tflops": attn_flop / t_at / 1e12,
                       "peak_tflops": bf16_peak, "peak_kind": f"{bf16_kind} bf16 dense",
                       "frac": attn_flop / t_at / 1e12 / bf16_peak, "bound": "tensor"},
        "chain_us": t_ch * 1e6,
        "chain_note": "prologue -> scores -> top-k -> attention back to back on one stream",
    }
    del q_mla, out, scores, attn_ws
    torch.cuda.empty_cache()
    return res


def time_sparse_mla_fp8(dsa, peak_gbs, wl, iters=32, sets=16):
    """Sparse attention over the FP8 latent cache (656 B rows) at the decode
    workload's sizes: B queries x 2048 selected rows of a B x T cache.  The
    selections rotate over `sets` independent random draws, so the rows gathered
    across the timed iterations (sets x B x 2048 x 656 B) exceed L2.  Algorithmic
    bytes per call: the FP8 rows gathered, the bf16 queries and outputs."""
    B, T, Hq, dc, dr, k = wl.B, wl.T, wl.Hq, wl.dc, wl.dr, wl.topk
    g = torch.Generator(device="cuda").manual_seed(wl.seed(2))
    rb = dsa.dsa_latent_row_bytes(dc, dr)
    cache = torch.empty(B, T, rb, dtype=torch.uint8, device="cuda")
    for b in range(B):                                   # quantise one sequence at a time
        kv = torch.randn(1, T, dc + dr, device="cuda", generator=g).to(torch.bfloat16)
        dsa.dsa_latent_quant(kv, cache[b:b + 1], dc)
        del kv
    q = torch.randn(B, 1, Hq, dc + dr, device="cuda", generator=g).to(torch.bfloat16)
    idxs = [torch.stack([torch.randperm(T, device="cuda", generator=g)[:k] for _ in range(B)])
            .to(torch.int32).reshape(B, 1, k).contiguous() for _ in range(sets)]
    out = torch.empty(B, 1, Hq, dc, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, 1, Hq, dtype=torch.float32, device="cuda")
    ws = torch.empty(dsa.dsa_sparse_mla_attn_fp8_workspace_size(B, 1, Hq, dc, dr, k),
                     dtype=torch.uint8, device="cuda")

    def one(i):
        dsa.dsa_sparse_mla_attn_fp8(q, cache, idxs[i % sets], T - 1, wl.sm_scale, dc, out, lse, ws)

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(iters):
        one(i)
    t1.record()
    t1.synchronize()
    t = t0.elapsed_time(t1) * 1e-3 / iters
    nbytes = B * k * rb + B * Hq * (dc + dr) * 2 + B * Hq * dc * 2
    res = {"workload": f"{wl.name}_fp8_latent", "rows": B * k, "row_bytes": rb, "bytes": nbytes,
           "us": t * 1e6, "achieved_gbs": nbytes / t / 1e9, "peak_gbs": peak_gbs,
           "frac": nbytes / t / 1e9 / peak_gbs, "bound": "hbm",
           "note": "656-byte rows decoded to bf16 while they are gathered, inside the attention kernel"}
    del cache, idxs, ws
    return res


def measure_fp8_peak(n=8192, iters=20, sustained=True):
    """Dense e4m3 GEMM throughput (torch._scaled_mm, N^3, best of `iters`) -- the
    FP8 tensor-core denominator for the prefill scorer's roofline."""
    a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn).t()
    one = torch.ones((), device="cuda")
    for _ in range(3):
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(iters):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        t1.record()
        t1.synchronize()
        best = min(best, t0.elapsed_time(t1) * 1e-3)
    if not sustained:
        return {"fp8_e4m3_tflops": 2 * n ** 3 / best / 1e12, "n": n}
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        k = 0
        while True:
            for _ in range(50):
                torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            k += 50
            t1.record()
            t1.synchronize()
            if t0.elapsed_time(t1) > 4000:
                break
    sustained = 2 * n ** 3 * k / (t0.elapsed_time(t1) * 1e-3) / 1e12
    return {"fp8_e4m3_tflops": 2 * n ** 3 / best / 1e12, "fp8_e4m3_tflops_sustained": sustained,
            "n": n, "how": "torch._scaled_mm e4m3 x e4m3 -> bf16, N^3, best of "
                           f"{iters} (burst) and back to back for 4 s (sustained)",
            "clocks": clk.summary()}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the prefill scoring measurement")
    ap.add_argument("--prologue-only", action="store_true",
                    help="time only the fused indexer prologue on the T=8192 prefill")
    ap.add_argument("--prefill-only", action="store_true",
                    help="only time the prefill scoring (T = 8192 causal) and exit")
    ap.add_argument("--prefill-chain-only", action="store_true",
                    help="only time the T = 8192 prefill chain (prologue, scores, top-k, "
                         "attention) and exit")
    ap.add_argument("--fp8-peak", action="store_true",
                    help="measure the dense FP8 GEMM peak and exit")
    ap.add_argument("--eager", action="store_true",
                    help="time the decode steps launched one by one instead of graph-replayed")
    ap.add_argument("--copies", type=int, default=N_COPIES,
                    help="rotating device copies of the decode state (each larger than L2)")
    args = ap.parse_args(argv)
    if args.fp8_peak:
        print(json.dumps(measure_fp8_peak()), flush=True)
        return
    if args.prologue_only:
        import __graft_entry__
        __graft_entry__._builder().build()
        import top_kv_selection_b200 as dsa
        print(json.dumps(time_indexer_prologue(dsa, _peaks()[0], iters=max(1, args.steps))),
              flush=True)
        return
    if args.prefill_only:
        import __graft_entry__
        __graft_entry__._builder().build()
        import top_kv_selection_b200 as dsa
        print(json.dumps(time_prefill_scoring(dsa, measure_fp8_peak(sustained=False)["fp8_e4m3_tflops"],
                                              iters=max(1, args.steps))), flush=True)
        return
    if args.prefill_chain_only:
        import __graft_entry__
        __graft_entry__._builder().build()
        import top_kv_selection_b200 as dsa
        print(json.dumps(time_prefill_chain(dsa, _peaks()[0], iters=max(1, min(args.steps, 10)))),
              flush=True)
        return
    wl = workloads.WORKLOADS[args.workload]
    if wl.mode != "decode":
        raise SystemExit("bench.py times decode workloads (1, 2 or 4)")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start the ranks under torch.distributed.run
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
               f"--nproc-per-node={args.gpus}", "--master-addr", "127.0.0.1",
               "--master-port", str(port), os.path.abspath(__file__),
               *(sys.argv[1:] if argv is None else argv)]
        os.execv(sys.executable, cmd)
    world, rank, local = _dist_init()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but the launcher started {world} ranks")
    try:
        if args.impl == "reference":
            run_reference(args, wl, world, rank)
        else:
            if not torch.cuda.is_available():
                raise SystemExit("no CUDA device: the product path has no CPU fallback")
            run_ours(args, wl, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
