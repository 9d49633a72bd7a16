#!/usr/bin/env python
"""DSA decode benchmark: queries/s at 1M-token context on B200 (one JSON line).

A step is one decode query through one DSA layer: compress the region the new token
completes, score every complete region with the 16-head indexer, select the own region
plus the top-511, and attend 64 query heads over the selected regions' K/V (4,096 tokens
per KV group).  Workload (default): one request, L = 1,048,576 tokens, k = 512, paged
K/V with a random page permutation, all inputs seeded synthetic N(0,1) bf16 / U(0,1).
Four independent layer caches (each 128 MiB of summaries + 3 GiB of K/V) are used round
robin, so consecutive steps never find their inputs in the 126 MB L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload decode_b1_1m|prefill_2k_256k]

--workload prefill_2k_256k[_local] times the chunked-prefill step instead (2,048 new query tokens
on a 262,144-token context: compress the 256 completed regions, FP8 indexer GEMM, top-512
per query and group, sparse GQA prefill attention) and prints its own line (tokens/s and
each stage's share; the indexer GEMM's roofline against the FP8 tensor peak); _local gives
the 8 queries of a region one indexer query, so neighbouring queries select the same regions.

--gpus N > 1 (under torchrun): every rank runs an independent replica (requests shard
across GPUs with no data-path collective, weak scaling); timing is the max over ranks.
--impl reference times the CPU oracle (the only other arm this method has) on the host.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DSA decode queries/s @1M ctx; indexer+attn HBM GB/s vs B200 peak"
UNIT = "queries/s"
L_CTX = 1 << 20
TOPK = 512
N_LAYERS = 4
KERNELS_PER_STEP = 4      # compress, scan (+ chunk maxima), cluster top-k, clustered attention
# DRAM bytes (read + write) of one scan launch on this workload, from one ncu capture of the
# current scan kernel (dram__bytes_read.sum + dram__bytes_write.sum); None once the kernel changes
SCAN_TRAFFIC_BYTES = 136_384_000 + 3_348_480
PREFILL_CTX, PREFILL_NEW = 262144, 2048
PREFILL_KERNELS = 6       # compress, quantize, GEMM, top-k, shared-selection attention, per-row attention
# DRAM bytes (read + write) of one gemm_scores_kernel launch on the prefill workload: None, the
# kernel changed (its roles now drain their last copies and MMAs before exiting) after the last
# capture that counted them (139,658,240 read + 1,020,275,000 written)
GEMM_TRAFFIC_BYTES = None


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--repeats", type=int, default=5, help="timed passes of --steps steps; the median is reported")
    ap.add_argument("--shard", choices=["replicas", "groups"], default="replicas",
                    help="replicas: independent requests per GPU; groups: KV-group shards of one request")
    ap.add_argument("--tp", type=int, default=0,
                    help="--shard groups: GPUs per request (1, 2 or 4; default min(world, 4)); on fewer GPUs "
                         "than tp the run times one shard of a tp-way split")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=N_LAYERS)
    ap.add_argument("--cpu-queries", type=int, default=32, help="oracle queries timed for cpu_baseline (30 s cap)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=["decode_b1_1m", "prefill_2k_256k", "prefill_2k_256k_local",
                                           "swa_decode_b8", "frontend_2k", "fp8_peak"], default="decode_b1_1m")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def scan_bytes(own: int) -> int:
    """Algorithmic bytes of one indexer scan: e4m3 summaries + fp32 scales of every
    eligible region, 4 groups."""
    return 4 * own * (256 + 4)


def step_bytes(own: int, k: int) -> int:
    """Algorithmic bytes of one decode step at position L-1: scan + selected K/V (4 groups
    x k regions x 8 tokens x 768 B) + index_q/gate + Q/O + the compressed region."""
    kv = 4 * min(k, own + 1) * 8 * 2 * 192 * 2
    return scan_bytes(own) + kv + 16 * 256 * 2 + 16 * 4 + 2 * 64 * 192 * 2 + 4 * 8 * 256 * 2 + 4 * 260


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML every 10 ms in a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, cuda_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            from cuda.bindings import runtime as rt
            pynvml.nvmlInit()
            self.nv = pynvml
            # NVML enumerates every GPU of the host: find ours by PCI bus id
            bus = rt.cudaDeviceGetPCIBusId(64, cuda_index)[1]
            bus = bus.split(b"\x00")[0].decode() if isinstance(bus, bytes) else str(bus)
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(0.01)

    def sample(self):
        if self.nv is None:
            return
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            self.raw_reasons = getattr(self, "raw_reasons", 0) | int(r)
            for bit, name in self.REASONS.items():
                if r & bit and name != "gpu_idle":
                    self.reasons.add(name)
        except Exception:
            pass

    def __enter__(self):
        self.sample()
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._t.join()
        self.sample()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ------------------------------------------------------------------ CPU oracle arm

def oracle_inputs(seed: int, device):
    """Host copies of one layer cache for the oracle (index_k, K/V, queries)."""
    import numpy as np
    import torch
    from sparse_long_context_dsa_b200 import workloads as W

    d = W.decode_batch([L_CTX], seed=seed, device=device, permute=True)

    def bits(t):
        return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)

    host = {k: bits(d[k]) for k in ("index_k", "index_q", "q", "k_cache", "v_cache")}
    host["gate"] = d["gate"].cpu().numpy()
    host["block_table"] = d["block_table"].cpu().numpy()
    host["q_pos"] = d["q_pos"].cpu().numpy()
    host["n_slots"] = d["n_slots"]
    del d
    return host


def oracle_time(host, n_queries: int, time_cap_s: float = float("inf")):
    """Times up to n oracle decode steps (compress the due region, score, select, attend),
    stopping early once time_cap_s has elapsed; returns (queries/s, threads, seconds, steps run)."""
    import numpy as np
    import oracle

    own = (L_CTX - 1) // 8
    src = [8 * r for r in range(own)]
    S, C = oracle.compress_regions(host["index_k"], src, list(range(own)), host["n_slots"])
    t0 = time.perf_counter()
    done = 0
    while done < n_queries and time.perf_counter() - t0 < time_cap_s:
        done += 1
        oracle.compress_regions(host["index_k"], [8 * own], [own], host["n_slots"], S, C)
        sc = oracle.indexer_scores(host["index_q"], host["gate"], [0], host["q_pos"], S, C, [0], ld=own)
        idx, cnt = oracle.topk_regions(np.nan_to_num(sc), host["q_pos"], TOPK)
        oracle.sparse_attention(host["q"], host["k_cache"], host["v_cache"], host["block_table"], [0],
                                host["q_pos"], idx, cnt)
    dt = time.perf_counter() - t0
    return done / dt if done else 0.0, oracle.get_threads(), dt, done


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import torch
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    host = oracle_inputs(1237, dev)
    if args.warmup > 0:
        oracle_time(host, 1)
    # each step is one decode query; the run stops after K of them or 90 s, whichever is first
    qps, cores, dt, done = oracle_time(host, args.steps, time_cap_s=90.0)
    line = {"impl": "reference", "metric": METRIC, "value": qps, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(done, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": "decode_b1_1m", "context": L_CTX, "topk": TOPK},
            "cpu_baseline": {"kind": "oracle", "value": qps, "unit": UNIT, "cores": cores,
                             "sample": f"{done} of {args.steps} decode queries at 1M context ({dt:.1f} s, "
                                       "the run bounded at 90 s), one layer cache"},
            "e2e": {"value": qps, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm

def build_layers(n_layers, seed0, device, g0=0, ng=4):
    """n_layers independent 1M-token layer caches; with ng < 4 only the summaries and K/V of
    groups g0 .. g0 + ng - 1 are kept (one GPU of a KV-group-sharded decode)."""
    import torch
    from sparse_long_context_dsa_b200 import pipeline
    from sparse_long_context_dsa_b200 import workloads as W

    layers = []
    for l in range(n_layers):
        d = W.decode_batch([L_CTX], seed=seed0 + 1000 * l, device=device, permute=True)
        n_slots = d["n_slots"]
        S = torch.zeros((4, n_slots, 256), dtype=torch.uint8, device=device)
        C = torch.zeros((4, n_slots), dtype=torch.float32, device=device)
        pipeline.compress_all(d["index_k"], [L_CTX - 1], [0], d["sum_base"], S, C)
        tail = d["index_k"][L_CTX - 8:].clone()            # the region this step completes
        del d["index_k"]
        if ng < 4:
            S, C = S[g0:g0 + ng].contiguous(), C[g0:g0 + ng].contiguous()
            d["k_cache"] = d["k_cache"][:, g0:g0 + ng].contiguous()
            d["v_cache"] = d["v_cache"][:, g0:g0 + ng].contiguous()
        torch.cuda.empty_cache()
        own = (L_CTX - 1) // 8
        step = pipeline.DecodeStep(S, C, d["sum_base"], d["block_table"], d["k_cache"], d["v_cache"], ld=own,
                                   k=TOPK, tail_tokens=8, g0=g0)
        step.load(d["index_q"], d["gate"], d["q"], d["q_pos"], tail)
        step.set_compress([0], [own])
        layers.append(dict(step=step, inputs=d))
    torch.cuda.synchronize()
    return layers


def capture(layers, n_steps, e2e=None, attn_only=False):
    """One CUDA graph of n_steps decode steps, layer i % len(layers) at step i.
    e2e: per-layer pinned host buffers: each step's inputs are copied in from them by a kernel
    and its output is written into them by the attention kernel.
    attn_only: only each step's attention (over the selection already in place)."""
    import torch

    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(n_steps):
                L = layers[i % len(layers)]
                st = L["step"]
                if attn_only:
                    st.run_attention()
                    continue
                if e2e is not None:
                    st.stage(e2e[i % len(layers)]["arena"])      # pinned host -> device, by a kernel
                # e2e: the attention writes the output straight into pinned host memory
                st.run(out=None if e2e is None else e2e[i % len(layers)]["out"])
    torch.cuda.current_stream().wait_stream(s)
    return g


def capture_scans(layers, n_steps):
    """One CUDA graph of the indexer scans of n_steps steps (layer i % len(layers) at i)."""
    import torch
    from sparse_long_context_dsa_b200 import dsa

    L_ = dsa.lib()
    p = dsa._p
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(n_steps):
                st = layers[i % len(layers)]["step"]
                dsa._check(L_.dsa_indexer_scores(p(st.index_q), p(st.gate), p(st.q_req), p(st.q_pos), st.B,
                                                 p(st.summaries), p(st.scales), st.summaries.shape[1],
                                                 p(st.sum_base), st.sum_base.numel(), p(st.scores), st.ld, st.flags,
                                                 p(st.ws_idx), st.ws_idx_n, dsa._stream()))
    torch.cuda.current_stream().wait_stream(s)
    return g


def run_groups(args):
    """Decode at 1M context with KV-group shards ([P2] §索引器打分: the 4 groups split cleanly):
    tp GPUs share each request, GPU i holding groups 4i/tp .. 4(i+1)/tp - 1 of its summaries and
    K/V; a step is that shard's compress / score / select / attend (one CUDA graph per layer)
    followed by an NCCL all-gather of the 16*ng output heads of every shard (world / tp
    replicas of tp shards).  On fewer GPUs than tp, a run times one shard's step alone (the
    per-GPU compute of a tp-way split, no gather)."""
    import datetime
    import torch
    import torch.distributed as dist
    from sparse_long_context_dsa_b200 import dsa, replicas

    rank, world, local = dist_env()
    tp = args.tp or min(world, 4)
    lone = world < tp                          # one shard of a tp-way split, timed alone
    if lone and world != 1:
        raise SystemExit("--tp larger than the number of GPUs runs on one GPU only")
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dsa.lib()
    replica, g0, ng = replicas.group_plan(0 if lone else rank, tp if lone else world, tp)
    grp = replicas.tp_group(world, tp) if (tp > 1 and not lone) else None
    layers = build_layers(args.layers, seed0=1237 + 7919 * replica, device=dev, g0=g0, ng=ng)
    for L in layers:
        L["step"].run()
    dsa.check_device()
    graphs = []
    for L in layers:                           # one graph per layer's step (compute only)
        graphs.append(capture([L], 1))
        graphs[-1].replay()
    torch.cuda.synchronize()
    gather = grp is not None

    def one_pass():
        for i in range(args.steps):
            j = i % len(layers)
            graphs[j].replay()
            if gather:
                replicas.gather_heads(layers[j]["step"].out, grp, tp)

    for i in range(max(args.warmup, 3)):
        graphs[i % len(graphs)].replay()
        if gather:
            replicas.gather_heads(layers[i % len(layers)]["step"].out, grp, tp)
    torch.cuda.synchronize()

    def timed():
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        replicas.barrier()
        torch.cuda.synchronize()
        a.record()
        one_pass()
        b.record()
        torch.cuda.synchronize()
        replicas.barrier()
        return replicas.max_over_ranks(a.elapsed_time(b), dev)

    sampler = ClockSampler(local)
    with sampler:
        passes = [timed() for _ in range(args.repeats)]
    ms = statistics.median(passes)
    dsa.check_device()
    n_rep = 1 if lone else world // tp
    qps = n_rep * args.steps / (ms / 1e3)
    own = (L_CTX - 1) // 8
    shard_bytes = step_bytes(own, TOPK) * ng // 4
    line = {
        "metric": METRIC, "value": qps, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "strong" if tp > 1 and n_rep == 1 else "weak", "vs_baseline": None,
        "dtype": "e4m3+bf16 (fp32 accumulate)", "data": "synthetic",
        "config": {"workload": "decode_b1_1m", "context": L_CTX, "topk": TOPK, "parallelism": f"groups tp{tp}",
                   "shard": {"g0": g0, "groups": ng, "replicas": n_rep},
                   "gather": "NCCL all-gather of the 16*ng output heads per step" if gather else
                   ("none: one shard of a %d-way split timed alone" % tp if lone else "none (tp = 1)"),
                   "layer_caches": args.layers, "l2": "inputs larger than L2 (layer caches round robin)",
                   "timing": f"median of {args.repeats} timed passes of {args.steps} steps"},
        "shard_hbm_gbs": shard_bytes * args.steps / (ms / 1e3) / 1e9,
        "passes_ms": passes, "gpu_launches": KERNELS_PER_STEP * args.steps, "clocks": sampler.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graphs
    if world > 1:
        dist.destroy_process_group()


def run_ours(args):
    import torch
    import torch.distributed as dist
    rank, world, local = dist_env()
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from sparse_long_context_dsa_b200 import dsa
    dsa.lib()

    layers = build_layers(args.layers, seed0=1237 + 7919 * rank, device=dev)
    own = (L_CTX - 1) // 8
    for L in layers:                 # one eager step per layer before any capture
        L["step"].run()
    dsa.check_device()

    from sparse_long_context_dsa_b200 import replicas
    barrier = replicas.barrier

    def max_over_ranks(x):
        return replicas.max_over_ranks(x, dev)

    # ---- warm-up graph and timed graph(s); each graph holds at most 250 steps
    chunk = min(args.steps, 250)
    n_full, rem = divmod(args.steps, chunk)
    g_warm = capture(layers, max(args.warmup, 3))
    g_main = capture(layers, chunk)
    g_tail = capture(layers, rem) if rem else None
    g_warm.replay()
    # every graph the timed region replays runs once untimed first (a graph's first replay
    # uploads it and pays one-time costs)
    g_main.replay()
    if g_tail is not None:
        g_tail.replay()
    g_warm.replay()
    dsa.check_device()
    torch.cuda.synchronize()

    def timed(graphs_once):
        """One timed pass of exactly K steps: barrier + synchronize on both sides, CUDA
        events on the replaying stream; the slowest rank's milliseconds."""
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        a.record()
        graphs_once()
        b.record()
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(a.elapsed_time(b))

    def main_pass():
        for _ in range(n_full):
            g_main.replay()
        if g_tail is not None:
            g_tail.replay()

    sampler = ClockSampler(local)
    with sampler:
        passes = [timed(main_pass) for _ in range(args.repeats)]
    ms = statistics.median(passes)
    # the scan's launch duration: the same scans (layer round robin) back to back in one graph,
    # CUDA events around it on its stream
    g_scan = capture_scans(layers, chunk)
    g_scan.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    scan_ms = []
    for _ in range(max(n_full, 3)):
        e0.record()
        g_scan.replay()
        e1.record()
        torch.cuda.synchronize()
        scan_ms.append(e0.elapsed_time(e1) / chunk)
    scan_avg_ms = max_over_ranks(statistics.median(scan_ms))
    # the attention alone (over the selections the steps left in place), back to back in one
    # graph: with the scan alone it splits the step's time (the selection takes the rest)
    g_sa = capture(layers, chunk, attn_only=True)
    g_sa.replay()
    torch.cuda.synchronize()
    sa_ms = []
    for _ in range(3):
        e0.record()
        g_sa.replay()
        e1.record()
        torch.cuda.synchronize()
        sa_ms.append(e0.elapsed_time(e1) / chunk)
    sa_avg_ms = max_over_ranks(statistics.median(sa_ms))
    del g_sa
    dsa.check_device()

    # ---- e2e: host (pinned) inputs in, result out, every step
    e2e_bufs = []
    for L in layers:
        st = L["step"]
        e2e_bufs.append(dict(arena=st.arena.cpu().pin_memory(),
                             out=torch.empty_like(st.out, device="cpu").pin_memory()))
    h2d = e2e_bufs[0]["arena"].numel()
    d2h = e2e_bufs[0]["out"].numel() * e2e_bufs[0]["out"].element_size()
    g_e2e = capture(layers, chunk, e2e=e2e_bufs)
    g_e2e_tail = capture(layers, rem, e2e=e2e_bufs) if rem else None
    g_e2e.replay()
    if g_e2e_tail is not None:
        g_e2e_tail.replay()
    torch.cuda.synchronize()

    def e2e_pass():
        for _ in range(n_full):
            g_e2e.replay()
        if g_e2e_tail is not None:
            g_e2e_tail.replay()

    e2e_ms = statistics.median([timed(e2e_pass) for _ in range(args.repeats)])
    dsa.check_device()
    # e2e results must equal the device-resident results (same inputs)
    assert torch.equal(e2e_bufs[0]["out"], layers[0]["step"].out.cpu())

    hbm, peak_kind = peaks()
    qps = replicas.job_throughput(args.steps, world, ms)
    scan_gbs = scan_bytes(own) / (scan_avg_ms / 1e3) / 1e9
    step_gbs = step_bytes(own, TOPK) * args.steps / (ms / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": qps, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3+bf16 (fp32 accumulate)", "data": "synthetic",
        "config": {"workload": "decode_b1_1m", "context": L_CTX, "topk": TOPK, "batch_per_gpu": 1,
                   "layer_caches": args.layers,
                   "l2": f"inputs larger than L2: {args.layers} layer caches of "
                         f"{scan_bytes(own) / 1e6:.0f} MB summaries + 3 GiB K/V used round robin",
                   "graph": "each step captured in a CUDA graph; kernels chained by programmatic dependent launch",
                   "timing": f"median of {args.repeats} timed passes of {args.steps} steps (every graph replayed "
                             "once untimed first)",
                   "scan_timing": "graph of the step's scans back to back, CUDA events around it"},
        "passes_ms": passes,
        "step_hbm_gbs": step_gbs,
        "roofline": {"kernel": "indexer scan (scan_kernel)", "bound": "hbm", "achieved": scan_gbs, "peak": hbm,
                     "unit": "GB/s", "frac": scan_gbs / hbm, "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": scan_bytes(own), "avg_launch_us": scan_avg_ms * 1e3,
                     "step_us": ms * 1e3 / args.steps, "attn_alone_us": sa_avg_ms * 1e3,
                     "traffic": SCAN_TRAFFIC_BYTES},
        "e2e": {"value": replicas.job_throughput(args.steps, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": KERNELS_PER_STEP * args.steps,
        "clocks": sampler.summary(),
    }
    # ---- CPU baseline: the oracle on this host, rank 0 at N = 1 only
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = oracle_inputs(1237, dev)
        v, cores, dt, done = oracle_time(host, args.cpu_queries, time_cap_s=30.0)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": f"{done} decode queries at 1M context "
                                          f"({dt:.1f} s), one layer cache"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    for L in layers:
        del L
    if world > 1:
        dist.destroy_process_group()


# ------------------------------------------------------------------ prefill workload

def prefill_flops():
    """Algorithmic FLOPs of the chunk: indexer 2*256*16 per (query, eligible region) and
    attention 4*192*64 per (query, attended token); both summed exactly over the chunk."""
    n_idx = n_att = 0
    for i in range(PREFILL_NEW):
        p = PREFILL_CTX + i
        own = p // 8
        n_idx += own
        n_att += 8 * min(TOPK - 1, own) + (p % 8 + 1)
    return 2 * 256 * 16 * n_idx, 4 * 192 * 16 * 4 * n_att


def run_prefill(args):
    import torch
    from sparse_long_context_dsa_b200 import dsa, pipeline
    from sparse_long_context_dsa_b200 import workloads as W

    rank, world, local = dist_env()
    if world > 1:
        raise SystemExit("--workload prefill_2k_256k runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dsa.lib()
    region_local = args.workload == "prefill_2k_256k_local"
    d = W.prefill_chunk(PREFILL_CTX, PREFILL_NEW, seed=1238, device=dev, permute=True, region_shared_q=region_local)
    n_slots = d["n_slots"]
    S = torch.zeros((4, n_slots, 256), dtype=torch.uint8, device=dev)
    C = torch.zeros((4, n_slots), dtype=torch.float32, device=dev)
    pipeline.compress_all(d["index_k"], [PREFILL_CTX], [0], d["sum_base"], S, C)
    total = PREFILL_CTX + PREFILL_NEW
    first, last = PREFILL_CTX // 8, total // 8
    src = torch.arange(first, last, dtype=torch.int64, device=dev) * 8
    dst = torch.arange(first, last, dtype=torch.int64, device=dev)
    ld = last
    scores = torch.zeros((PREFILL_NEW, 4, ld), dtype=torch.float32, device=dev)
    sel = torch.empty((PREFILL_NEW, 4, TOPK), dtype=torch.int32, device=dev)
    cnt = torch.empty((PREFILL_NEW, 4), dtype=torch.int32, device=dev)
    out = torch.empty((PREFILL_NEW, 64, 192), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    dev_in = dict(index_k=d["index_k"], src=src, index_q=d["index_q"], gate=d["gate"], q=d["q"], q_pos=d["q_pos"])

    def step(ev=None, inp=dev_in, o=out):
        rec = (lambda i: ev[i].record()) if ev else (lambda i: None)
        rec(0)
        dsa.compress_regions(inp["index_k"], inp["src"], dst, S, C)
        rec(1)
        dsa.indexer_scores(inp["index_q"], inp["gate"], d["q_req"], inp["q_pos"], S, C, d["sum_base"], scores,
                           dsa.Q_FP8)
        rec(2)
        dsa.topk_regions(scores, inp["q_pos"], TOPK, sel, cnt)
        rec(3)
        dsa.sparse_attn_prefill(inp["q"], d["k_cache"], d["v_cache"], d["block_table"], d["q_req"], inp["q_pos"],
                                sel, cnt, out=o)
        rec(4)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    dsa.check_device()
    stage = [0.0] * 4
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    with sampler:
        for i in range(args.steps):
            flush.zero_()                      # L2 flushed between steps (outside the timed stages)
            step(evs[i])
        torch.cuda.synchronize()
    for ev in evs:
        for j in range(4):
            stage[j] += ev[j].elapsed_time(ev[j + 1])
    dsa.check_device()
    ms = sum(stage)
    f_idx, f_att = prefill_flops()
    fp8_peak, kind = tensor_peak(fp8=True)
    t_gemm = stage[1] / args.steps * 1e-3
    # e2e: every chunk's host inputs (pinned) in and its output out, through the same calls.
    # Chunks are pipelined as a layer's prefill is: the next chunk's inputs (which do not depend
    # on this chunk's output) are copied in on one stream while this chunk computes, into the
    # other of two input sets, and each chunk's output is copied out on a third stream.
    names = ["index_q", "gate", "q", "q_pos"]
    host = {n: d[n].cpu().pin_memory() for n in names}
    host["index_k"] = d["index_k"][PREFILL_CTX:].cpu().pin_memory()     # the chunk's new rows
    sets = [dict({n: torch.empty_like(t, device=dev) for n, t in host.items()}, src=src - PREFILL_CTX)
            for _ in range(2)]
    outs = [torch.empty_like(out) for _ in range(2)]
    host_out = torch.empty_like(out, device="cpu").pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = host_out.numel() * host_out.element_size()
    comp, up, down = torch.cuda.current_stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(n):
        ready = [torch.cuda.Event() for _ in range(2)]      # set b holds its chunk's inputs
        done = [torch.cuda.Event() for _ in range(2)]       # the chunk in set b has been computed
        out_free = [torch.cuda.Event() for _ in range(2)]   # outs[b] has been copied out

        def upload(i):
            b = i % 2
            if i >= 2:
                up.wait_event(done[b])                      # chunk i - 2 no longer reads set b
            with torch.cuda.stream(up):
                for k, t in host.items():
                    sets[b][k].copy_(t, non_blocking=True)
            ready[b].record(up)

        up.wait_stream(comp)
        down.wait_stream(comp)
        upload(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                upload(i + 1)
            comp.wait_event(ready[b])
            if i >= 2:
                comp.wait_event(out_free[b])
            step(inp=sets[b], o=outs[b])
            done[b].record(comp)
            down.wait_event(done[b])
            with torch.cuda.stream(down):
                host_out.copy_(outs[b], non_blocking=True)
            out_free[b].record(down)
        comp.wait_stream(up)
        comp.wait_stream(down)

    e2e_run(2)                                               # untimed: first use of the streams
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(comp)
    e2e_run(args.steps)
    t1.record(comp)
    torch.cuda.synchronize()
    dsa.check_device()
    assert torch.equal(host_out, out.cpu())                  # the same result as the device-resident path
    e2e_ms = t0.elapsed_time(t1)
    line = {
        "metric": "DSA chunked-prefill query tokens/s (2,048 new on 262,144 ctx)", "value":
            PREFILL_NEW * args.steps / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 indexer, bf16 attention (fp32 accumulate)",
        "data": "synthetic",
        "config": {"workload": args.workload, "context": PREFILL_CTX, "new_tokens": PREFILL_NEW, "topk": TOPK,
                   "queries": "the 8 queries of a region share index_q and gates" if region_local
                   else "independent N(0,1)",
                   "l2": "flushed (256 MiB write) before every step, outside the timed stages"},
        "stages_ms": {"compress": stage[0] / args.steps, "indexer_gemm": stage[1] / args.steps,
                      "topk": stage[2] / args.steps, "attention": stage[3] / args.steps},
        "roofline": {"kernel": "indexer GEMM (quantize + gemm_scores_kernel)", "bound": "tensor",
                     "achieved": f_idx / t_gemm / 1e12, "peak": fp8_peak, "unit": "TFLOP/s",
                     "frac": f_idx / t_gemm / 1e12 / fp8_peak, "peak_kind": kind, "flops_per_launch": f_idx,
                     "traffic": GEMM_TRAFFIC_BYTES},
        "attention": {"flops": f_att, "tflops": f_att / (stage[3] / args.steps * 1e-3) / 1e12,
                      "peak_bf16": tensor_peak(fp8=False)[0]},
        "e2e": {"value": PREFILL_NEW * args.steps / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": PREFILL_KERNELS * args.steps,
        "clocks": sampler.summary(),
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = prefill_oracle_time(d, n_queries=128, time_cap_s=30.0)
    print(json.dumps(line), flush=True)


def prefill_oracle_time(d, n_queries: int, time_cap_s: float):
    """The oracle on the host over a bounded sample of the same chunk: the chunk's 256 new
    regions compressed, then per query (the chunk's first ones, up to n_queries or the time
    cap) the scores over every region, the top-512 and the attention.  The summaries of the
    cached context come from the oracle itself (untimed)."""
    import numpy as np
    import torch
    import oracle

    def bits(t):
        return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)

    index_k = bits(d["index_k"])
    kc, vc = bits(d["k_cache"]), bits(d["v_cache"])
    index_q, q = bits(d["index_q"]), bits(d["q"])
    gate, qp = d["gate"].cpu().numpy(), d["q_pos"].cpu().numpy()
    bt = d["block_table"].cpu().numpy()
    first, last = PREFILL_CTX // 8, (PREFILL_CTX + PREFILL_NEW) // 8
    S, C = oracle.compress_regions(index_k, [8 * r for r in range(first)], list(range(first)), last)
    t0 = time.perf_counter()
    oracle.compress_regions(index_k, [8 * r for r in range(first, last)], list(range(first, last)), last, S, C)
    done = 0
    while done < n_queries and time.perf_counter() - t0 < time_cap_s:
        i = done
        sc = oracle.indexer_scores(index_q[i:i + 1], gate[i:i + 1], [0], qp[i:i + 1], S, C, [0], ld=last)
        idx, cnt = oracle.topk_regions(np.nan_to_num(sc), qp[i:i + 1], TOPK)
        oracle.sparse_attention(q[i:i + 1], kc, vc, bt, [0], qp[i:i + 1], idx, cnt)
        done += 1
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": "tokens/s", "cores": oracle.get_threads(), "kind": "oracle",
            "sample": f"the chunk's 256 new regions compressed and {done} of its queries scored, selected and "
                      f"attended ({dt:.1f} s)"}


SWA_BATCH, SWA_LAYERS, SWA_WINDOW, SWA_RING = 8, 69, 512, 8


def swa_bytes_per_query() -> int:
    """Algorithmic bytes of one window-layer decode query: the window's K and V (512 tokens
    x 4 groups x 192 x 2 B each), Q and O (64 x 192 x 2 B each), the new token's K and V read
    and written into the ring (4 x 192 x 2 B each, twice)."""
    kv = SWA_WINDOW * 4 * 192 * 2 * 2
    qo = 2 * 64 * 192 * 2
    new = 2 * 2 * 4 * 192 * 2
    return kv + qo + new


def run_swa(args):
    """Decode of the window layers ([P1] §滑窗注意力: 69 of 92 layers attend the last 512
    tokens from a ring buffer): a step is one layer for a batch of 8 requests at ~1M
    positions, the new tokens appended to each request's ring and attended over their last
    512 tokens; steps rotate through 69 layers' rings (868 MB, larger than L2)."""
    import numpy as np
    import torch
    from sparse_long_context_dsa_b200 import dsa, pipeline

    import torch.distributed as dist
    from sparse_long_context_dsa_b200 import replicas

    rank, world, local = dist_env()
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dsa.lib()
    g = torch.Generator(device=dev)
    g.manual_seed(1240 + rank)
    max_pages = (L_CTX + 64) // 64 + 1
    bt = pipeline.ring_block_table(SWA_BATCH, max_pages, SWA_RING, dev)
    layers = []
    for _ in range(SWA_LAYERS):
        kr = torch.randn((SWA_BATCH * SWA_RING, 4, 64, 192), generator=g, device=dev).to(torch.bfloat16)
        vr = torch.randn(kr.shape, generator=g, device=dev).to(torch.bfloat16)
        st = pipeline.WindowDecodeStep(kr, vr, bt, SWA_WINDOW)
        st.load(torch.randn((SWA_BATCH, 64, 192), generator=g, device=dev).to(torch.bfloat16),
                torch.randn((SWA_BATCH, 4, 192), generator=g, device=dev).to(torch.bfloat16),
                torch.randn((SWA_BATCH, 4, 192), generator=g, device=dev).to(torch.bfloat16),
                torch.full((SWA_BATCH,), L_CTX - 1, dtype=torch.int32, device=dev))
        layers.append(st)
    for i in range(max(args.warmup, 3)):
        layers[i % SWA_LAYERS].run()
    torch.cuda.synchronize()
    dsa.check_device()

    def graph(n):
        gr = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(gr, stream=s):
                for i in range(n):
                    layers[i % SWA_LAYERS].run()
        torch.cuda.current_stream().wait_stream(s)
        return gr

    n = args.steps
    gr = graph(n)
    gr.replay()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    replicas.barrier()
    with sampler:
        torch.cuda.synchronize()
        t0.record()
        gr.replay()
        t1.record()
        torch.cuda.synchronize()
    dsa.check_device()
    ms = replicas.max_over_ranks(t0.elapsed_time(t1), dev)
    step_us = ms * 1e3 / n
    bytes_step = SWA_BATCH * swa_bytes_per_query()
    launches = int(dsa.lib().dsa_window_decode_launches(SWA_BATCH, SWA_WINDOW))   # 1: append folded into the clustered kernel
    peak, kind = peaks()
    achieved = bytes_step / (step_us * 1e-6) / 1e9
    # e2e: per step the step's input arena read from pinned host memory by the library's copy
    # kernel and the output written by the attention kernel straight into pinned host memory,
    # both inside the graph (as a caller's decode loop would capture it)
    host = [st.arena.cpu().pin_memory() for st in layers[:4]]
    out_host = torch.empty((SWA_BATCH, 64, 192), dtype=torch.bfloat16).pin_memory()
    n_e2e = n
    ge = torch.cuda.CUDAGraph()
    s_e = torch.cuda.Stream()
    s_e.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s_e):
        with torch.cuda.graph(ge, stream=s_e):
            for i in range(n_e2e):
                st = layers[i % SWA_LAYERS]
                st.stage(host[i % 4])
                st.run(out_host)
    torch.cuda.current_stream().wait_stream(s_e)
    ge.replay()                                          # the graph's first replay pays one-time costs
    torch.cuda.synchronize()
    t0.record()
    ge.replay()
    t1.record()
    torch.cuda.synchronize()
    dsa.check_device()
    e2e_ms = replicas.max_over_ranks(t0.elapsed_time(t1), dev)
    h2d = host[0].numel()
    d2h = out_host.numel() * out_host.element_size()
    line = {
        "metric": "window-layer decode queries/s (8 requests at 1M context, 512-token ring)",
        "value": world * SWA_BATCH * n / (ms / 1e3), "unit": "queries/s", "n_gpus": world, "steps": n,
        "warmup": max(args.warmup, 3), "ms_per_step": ms / n, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 (fp32 softmax and accumulate)", "data": "synthetic",
        "config": {"workload": "swa_decode_b8", "batch": SWA_BATCH, "position": L_CTX - 1, "window": SWA_WINDOW,
                   "ring_pages": SWA_RING, "layers": SWA_LAYERS,
                   "l2": "69 layers' rings rotate (868 MB > L2)"},
        "roofline": {"kernel": ("window step (sparse_attn_cluster_kernel with the append folded in)" if launches == 1
                                else "window step (kv_append_kernel + sparse_attn_kernel [+ combine_kernel])"),
                     "bound": "hbm",
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": kind, "bytes_per_step": bytes_step, "traffic": None},
        "e2e": {"value": world * SWA_BATCH * n_e2e / (e2e_ms / 1e3), "unit": "queries/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches * n,
        "clocks": sampler.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline:
        import oracle
        st = layers[0]
        kc, vc, btc = (st.k_ring.cpu().contiguous().view(torch.int16).numpy().view(np.uint16),
                       st.v_ring.cpu().contiguous().view(torch.int16).numpy().view(np.uint16), bt.cpu().numpy())
        qb = st.q.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        qp = st.q_pos.cpu().numpy()
        reps = 40
        c0 = time.perf_counter()
        for _ in range(reps):
            oracle.window_attention(qb, kc, vc, btc, np.arange(SWA_BATCH), qp, SWA_WINDOW)
        dt = time.perf_counter() - c0
        line["cpu_baseline"] = {"value": reps * SWA_BATCH / dt, "unit": "queries/s", "cores": oracle.get_threads(),
                                "kind": "oracle", "sample": f"{reps} x 8 window queries on one layer's rings"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del gr
    if world > 1:
        dist.destroy_process_group()


FE_TOKENS, FE_HID = 2048, 6144


def run_frontend(args):
    """The indexer front end for a 2,048-token prefill chunk ([P2] §索引器打分: index_q /
    index_k / index_z projected from the hidden state, normalised, partially rotated): one
    dsa_indexer_frontend call per step, hidden size 6,144 (a reading: the pages give none),
    synthetic weights; L2 flushed before every step (the weights, 63 MB, would stay in it)."""
    import numpy as np
    import torch
    from sparse_long_context_dsa_b200 import dsa

    rank, world, local = dist_env()
    if world > 1:
        raise SystemExit("--workload frontend_2k runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dsa.lib()
    g = torch.Generator(device=dev)
    g.manual_seed(1241)
    T, hid = FE_TOKENS, FE_HID
    hidden = torch.randn((T, hid), generator=g, device=dev).to(torch.bfloat16)
    w = (torch.randn((dsa.FRONTEND_ROWS, hid), generator=g, device=dev) / hid ** 0.5).to(torch.bfloat16)
    gq = (1.0 + 0.1 * torch.randn(256, generator=g, device=dev)).to(torch.bfloat16)
    gk = (1.0 + 0.1 * torch.randn(256, generator=g, device=dev)).to(torch.bfloat16)
    pos = (262144 + torch.arange(T, device=dev)).to(torch.int32)
    iq = torch.empty((T, 16, 256), dtype=torch.bfloat16, device=dev)
    ik = torch.empty((T, 4, 256), dtype=torch.bfloat16, device=dev)
    z = torch.empty((T, 16), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(max(args.warmup, 3)):
        dsa.indexer_frontend(hidden, w, gq, gk, pos, iq, ik, z)
    torch.cuda.synchronize()
    dsa.check_device()
    n = min(args.steps, 50)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    sampler = ClockSampler(local)
    with sampler:
        for a, b in evs:
            flush.zero_()
            a.record()
            dsa.indexer_frontend(hidden, w, gq, gk, pos, iq, ik, z)
            b.record()
        torch.cuda.synchronize()
    dsa.check_device()
    ms = sum(a.elapsed_time(b) for a, b in evs) / n
    flops = 2.0 * T * hid * dsa.FRONTEND_ROWS
    peak, kind = tensor_peak(fp8=False)
    achieved = flops / (ms * 1e-3) / 1e12
    # e2e: hidden states from pinned host memory, the three outputs back
    h_host = hidden.cpu().pin_memory()
    oq, ok_, oz = (torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (iq, ik, z))
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = min(n, 10)
    torch.cuda.synchronize()
    t0.record()
    for _ in range(n_e2e):
        hidden.copy_(h_host, non_blocking=True)
        dsa.indexer_frontend(hidden, w, gq, gk, pos, iq, ik, z)
        oq.copy_(iq, non_blocking=True)
        ok_.copy_(ik, non_blocking=True)
        oz.copy_(z, non_blocking=True)
    t1.record()
    torch.cuda.synchronize()
    e2e_ms = t0.elapsed_time(t1) / n_e2e
    line = {
        "metric": "indexer front-end tokens/s (hidden 6,144 -> index_q, index_k, gates)", "value": T / (ms * 1e-3),
        "unit": "tokens/s", "n_gpus": 1, "steps": n, "warmup": max(args.warmup, 3), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 (fp32 accumulate)",
        "data": "synthetic",
        "config": {"workload": "frontend_2k", "tokens": T, "hidden": hid, "rows": dsa.FRONTEND_ROWS,
                   "l2": "flushed (256 MiB write) before every step"},
        "roofline": {"kernel": "frontend_kernel (tcgen05 bf16 GEMM + RMSNorm/RoPE/sigmoid epilogue)",
                     "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "peak_kind": kind, "flops_per_launch": flops, "traffic": None},
        "e2e": {"value": T / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h_host.numel() * 2,
                "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in (oq, ok_, oz))},
        "gpu_launches": n,
        "clocks": sampler.summary(),
    }
    if not args.no_cpu_baseline:
        import oracle
        rows = np.arange(8)
        hb = hidden[rows].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        wb = w.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        gqb = gq.cpu().view(torch.int16).numpy().view(np.uint16)
        gkb = gk.cpu().view(torch.int16).numpy().view(np.uint16)
        c0 = time.perf_counter()
        oracle.indexer_frontend(hb, wb, gqb, gkb, pos.cpu().numpy()[rows])
        dt = time.perf_counter() - c0
        line["cpu_baseline"] = {"value": len(rows) / dt, "unit": "tokens/s", "cores": oracle.get_threads(),
                                "kind": "oracle", "sample": f"{len(rows)} tokens of the chunk"}
    print(json.dumps(line), flush=True)


def run_fp8_peak(args):
    """The dense e4m3 tensor peak of this GPU, measured the way the bf16 figure is: a cuBLAS
    e4m3 x e4m3 GEMM (torch._scaled_mm, 8192^3, bf16 output, 2 * 8192^3 FLOP) as a burst
    (the best of 10 single launches, CUDA events) and sustained (back to back for 4 s)."""
    import torch

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    n = 8192
    g = torch.Generator(device=dev)
    g.manual_seed(1242)
    a = torch.randn((n, n), generator=g, device=dev).to(torch.float8_e4m3fn)
    b = torch.randn((n, n), generator=g, device=dev).to(torch.float8_e4m3fn).t()   # column-major
    one = torch.ones((), dtype=torch.float32, device=dev)
    out = torch.empty((n, n), dtype=torch.bfloat16, device=dev)

    def mm():
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16, out=out)

    for _ in range(5):
        mm()
    torch.cuda.synchronize()
    flop = 2.0 * n ** 3
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    burst = []
    for _ in range(10):
        e0.record()
        mm()
        e1.record()
        torch.cuda.synchronize()
        burst.append(flop / (e0.elapsed_time(e1) * 1e-3) / 1e12)
    sampler = ClockSampler(0)
    with sampler:
        reps, t0 = 0, time.perf_counter()
        e0.record()
        while time.perf_counter() - t0 < 4.0:
            for _ in range(20):
                mm()
            reps += 20
            torch.cuda.synchronize()
        e1.record()
        torch.cuda.synchronize()
    sustained = flop * reps / (e0.elapsed_time(e1) * 1e-3) / 1e12
    line = {"metric": "dense e4m3 GEMM TFLOP/s (torch._scaled_mm 8192^3, bf16 out)", "value": max(burst),
            "unit": "TFLOP/s", "n_gpus": 1, "burst_tflops": max(burst), "sustained_tflops": sustained,
            "sustained_launches": reps, "higher_is_better": True, "dtype": "e4m3", "data": "synthetic",
            "config": {"workload": "fp8_peak", "m": n, "n": n, "k": n}, "clocks": sampler.summary()}
    print(json.dumps(line), flush=True)


# Dense e4m3 GEMM peak of this machine's B200s, burst (cuBLAS e4m3 8192^3 through
# torch._scaled_mm: `python bench.py --workload fp8_peak`; sustained under the power cap: 2,643)
FP8_PEAK_TFLOPS = 3093.0


def tensor_peak(fp8: bool):
    """Dense tensor peak in TFLOP/s: e4m3 the measured burst GEMM figure above; bf16 the
    measured cuBLAS burst figure of MEASURED_PEAKS.json, else the fallback."""
    if fp8:
        return FP8_PEAK_TFLOPS, "measured e4m3 (cuBLAS 8192^3 burst, bench.py --workload fp8_peak)"
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v, kind = float(json.load(f)["bf16_tflops"]), "measured bf16"
    except Exception:
        v, kind = 1590.0, "fallback bf16"
    return v, kind


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload.startswith("prefill_2k_256k"):
        run_prefill(args)
    elif args.workload == "swa_decode_b8":
        run_swa(args)
    elif args.workload == "frontend_2k":
        run_frontend(args)
    elif args.workload == "fp8_peak":
        run_fp8_peak(args)
    elif args.shard == "groups":
        run_groups(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
