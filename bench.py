#!/usr/bin/env python
"""Benchmark of the single-GPU MoE token-routing step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config decode_30b_a3b]

One step = the whole hot path over one batch: mask -> create_indices ->
MXFP4 dispatch -> [NVFP4 activation quantisation] -> grouped NVFP4 GEMV ->
combine, replayed as one CUDA graph.  Inputs are resident in HBM when the
timed region starts; L2 is flushed (a 512 MiB memset, outside the timed
events) before every timed step.  Metric: routed token-expert pairs per
second, whole job.  With N > 1 (torchrun) every rank runs an independent
replica of the workload (weak scaling; the path has no exchange step).

Also reported: the grouped GEMV's achieved HBM bandwidth against the
measured copy bandwidth (roofline), the pipeline's algorithmic-byte
fraction, an end-to-end figure through the public API with host buffers,
SM clocks sampled during the timed region, and the CPU oracle timed on a
bounded sample of the same workload (rank 0, N = 1).

``--impl reference`` times the CPU oracle itself as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

FLUSH_BYTES = 512 << 20
THROTTLE_BITS = {  # clocks_event_reasons.active bitmask (NVML)
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="decode_30b_a3b", choices=sorted(wl.CONFIGS))
    ap.add_argument("--cpu-sample-tokens", type=int, default=48)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


METRIC = "routed token-expert pairs/s end-to-end at 1 B200"


def workload_config(cfg, mode: str, routed_pairs: int, active_experts: int) -> dict:
    """The config keys both arms report for a workload."""
    return {"workload": cfg.name, "N": cfg.N, "real_token_count": cfg.real, "K": cfg.K,
            "E": cfg.E, "top_k": cfg.top_k, "N_out": cfg.N_out, "mode": mode,
            "routed_pairs": routed_pairs, "active_experts": active_experts,
            "parallelism": "replicas"}


def max_over_ranks(value: float, world: int, device="cpu") -> float:
    """The largest value over the ranks (a replica job's time is its slowest
    replica's); with one rank, the value itself."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: int, world: int, ms: float) -> float:
    """Whole-job throughput: every rank processes units_per_rank in ms."""
    return world * units_per_rank / (ms * 1e-3)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "MEASURED_PEAKS.json hbm_gbs (of measured)"
    return 6650.0, "profiling-recipe fallback 6.65 TB/s (of fallback)"


def profiled_traffic(workload: str):
    """DRAM bytes per GEMV launch from the committed ncu summary of this
    workload, or None when there is none or the kernel sources differ from the
    ones that were profiled (the summary records their sha256)."""
    import hashlib
    import re
    path = os.path.join(ROOT, "profiles", f"grouped_gemv_nvfp4_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_t = re.search(r"traffic_bytes_per_launch = (\d+)", text)
    m_h = re.search(r"source_sha256\(([^)]*)\) = ([0-9a-f]{64})", text)
    if not (m_t and m_h):
        return None
    h = hashlib.sha256()
    for name in m_h.group(1).split("+"):
        with open(os.path.join(ROOT, "permute_fp4_dispatch_b200", "csrc", name.strip()), "rb") as f:
            h.update(f.read())
    return int(m_t.group(1)) if h.hexdigest() == m_h.group(2) else None


# ------------------------------------------------------------------ byte model
def algorithmic_bytes(cfg, mode: str, A: int, R: int, routed_tokens: int) -> dict:
    """Algorithmic HBM bytes per step, per kernel (each input read once, each output
    written once).  A = active experts, R = routed pairs."""
    N, K, E, k, No = cfg.N, cfg.K, cfg.E, cfg.top_k, cfg.N_out
    S = N * k
    stride = -(-(K // 2 + K // 32) // 16) * 16
    masked_rows = N - min(max(cfg.real, 0), N)
    b = {}
    b["mask"] = masked_rows * k * 8
    b["create_indices"] = S * 8 + S * 4 * 2 + (E + 1) * 4 * 2 + E * 4 + 8
    b["dispatch_mxfp4"] = routed_tokens * K * 2 + R * stride + E * 4
    if mode == "w4a4":
        b["quant_act_nvfp4"] = N * K * 2 + N * (K // 2 + K // 16)
        act = routed_tokens * (K // 2 + K // 16)
    else:
        act = routed_tokens * K * 2
    b["grouped_gemv"] = A * No * (K // 2 + K // 16) + act + R * No * 2 + A * 4
    b["combine"] = R * No * 2 + N * k * (4 + 8) + N * No * 2
    return b


# ------------------------------------------------------------------ clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100", "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        if self.path and os.path.exists(self.path):
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        for r in rows:
            try:
                mask = int(r[4], 16)
            except ValueError:
                continue
            for bit, name in THROTTLE_BITS.items():
                if mask & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------------ CPU oracle sample
def oracle_sample_step(cfg, mode, x, ids, rw, tokens, wq, sfw, gw, experts):
    """The oracle chain on a bounded sample: mask and create_indices over the whole
    routing map; MXFP4 dispatch, GEMV and combine for the sampled tokens' pairs."""
    import oracle
    ids_m = oracle.mask_padding(ids, cfg.real)
    idx = oracle.create_indices(ids_m, cfg.E)
    sub = {e: i for i, e in enumerate(experts)}
    rows = x[tokens]
    oracle.mxfp4_encode_rows(np.repeat(rows, cfg.top_k, axis=0))
    local = np.array([[sub.get(int(e), -1) for e in ids_m[t]] for t in tokens], np.int64)
    if mode == "w4a4":
        xq, sfa = oracle.nvfp4_quantize_bf16(rows, 1.0)
        y = oracle.grouped_gemv("w4a4", local, wq, sfw, gw, xq=xq, sfa=sfa)
    else:
        y = oracle.grouped_gemv("w4a16", local, wq, sfw, gw, act_bf16=rows)
    yb = wl.f32_to_bf16_bits(np.nan_to_num(y).astype(np.float32))
    oracle.combine(yb, rw[tokens], ids_m[tokens], cfg.E, cfg.epilogue)
    return idx


def oracle_setup(cfg, mode, n_tokens):
    import oracle
    x, ids, rw = wl.activations_bf16(cfg), wl.routing(cfg), wl.router_weights(cfg)
    ids_m = oracle.mask_padding(ids, cfg.real)
    real = min(max(cfg.real, 0), cfg.N)
    tokens = np.arange(min(n_tokens, real))
    experts = sorted({int(e) for t in tokens for e in ids_m[t] if 0 <= e < cfg.E})
    wq, sfw, gw = oracle.quantize_weights_nvfp4(wl.expert_weights_f32_many(cfg, experts))
    return x, ids, rw, tokens, wq, sfw, gw, experts


def routed_pairs_and_active(cfg):
    """Routed pairs and active experts of the whole workload, from the oracle."""
    import oracle
    idx = oracle.create_indices(oracle.mask_padding(wl.routing(cfg), cfg.real), cfg.E)
    return int(idx["expert_start_indices"][-1]), int(idx["expert_usage_stats"][1])


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(cfg, mode, n_tokens, repeats=1) -> dict:
    setup = oracle_setup(cfg, mode, n_tokens)
    tokens = setup[3]
    t0 = time.perf_counter()
    for _ in range(repeats):
        oracle_sample_step(cfg, mode, *setup[:3], tokens, *setup[4:])
    dt = (time.perf_counter() - t0) / repeats
    pairs = len(tokens) * cfg.top_k
    return {"value": pairs / dt, "unit": "routed pairs/s", "cores": 1, "kind": "oracle",
            "sample": (f"{len(tokens)} tokens ({pairs} routed pairs) of {cfg.name}: mask + "
                       f"create_indices over all {cfg.N} rows, MXFP4 dispatch, "
                       f"{mode.upper()} GEMV and combine for the sampled pairs; "
                       f"{dt:.2f} s per sample, single-threaded C, host has {cpu_cores()} cores")}


# ------------------------------------------------------------------ reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return
    cfg = wl.config(args.config)
    mode = cfg.modes[0]
    # size the per-step sample so that warm-up + timed steps take about 2.5 minutes
    probe = oracle_setup(cfg, mode, 1)
    t0 = time.perf_counter()
    oracle_sample_step(cfg, mode, *probe[:3], probe[3], *probe[4:])
    t_token = time.perf_counter() - t0
    budget = min(15.0, 150.0 / max(1, args.steps + args.warmup))
    n_tokens = int(max(1, min(args.cpu_sample_tokens, budget / max(t_token, 1e-6))))
    setup = oracle_setup(cfg, mode, n_tokens)
    tokens = setup[3]
    full_idx = routed_pairs_and_active(cfg)
    for _ in range(args.warmup):
        oracle_sample_step(cfg, mode, *setup[:3], tokens, *setup[4:])
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_sample_step(cfg, mode, *setup[:3], tokens, *setup[4:])
        times.append(time.perf_counter() - t0)
    pairs = len(tokens) * cfg.top_k
    dt = float(np.mean(times))
    value = pairs / dt
    line = {
        "impl": "reference", "metric": METRIC,
        "value": value, "unit": "routed pairs/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(cfg, mode, full_idx[0], full_idx[1]),
                       sample_tokens=int(len(tokens))),
        "e2e": {"value": value, "unit": "routed pairs/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "cpu_baseline": {"value": value, "unit": "routed pairs/s", "cores": 1, "kind": "oracle",
                         "sample": f"{len(tokens)} tokens ({pairs} pairs) per step, "
                                   f"single-threaded C oracle"},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from permute_fp4_dispatch_b200.build import build
    from permute_fp4_dispatch_b200.pipeline import RoutingPipeline

    build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = wl.config(args.config)
    mode = cfg.modes[0]
    x, ids, rw = wl.activations_bf16(cfg), wl.routing(cfg), wl.router_weights(cfg)

    pipe = RoutingPipeline(cfg.N, cfg.K, cfg.E, cfg.top_k, cfg.N_out, mode=mode,
                           epilogue=cfg.epilogue, device=dev)
    # pinned host copies of the step's inputs (for the end-to-end measurement)
    # a step's inputs live in one pinned host buffer laid out like the device
    # input arena, so they travel in one copy
    h_in, h_views = pipe.host_inputs()
    h_x, h_ids, h_rw, h_real = (h_views[k] for k in ("x", "routing_map", "router_weights",
                                                       "real_token_count"))
    h_x.copy_(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16))
    h_ids.copy_(torch.from_numpy(ids))
    h_rw.copy_(torch.from_numpy(rw))
    h_real.fill_(cfg.real)
    h_out = torch.empty((cfg.N, cfg.N_out), dtype=torch.bfloat16).pin_memory()
    pipe.x.copy_(h_x)
    pipe.routing_map.copy_(h_ids)
    pipe.router_weights.copy_(h_rw)
    pipe.real_token_count.copy_(h_real)
    for e0 in range(0, cfg.E, 16):
        es = list(range(e0, min(cfg.E, e0 + 16)))
        pipe.quantize_weights(torch.from_numpy(wl.expert_weights_f32_many(cfg, es)).to(dev),
                              expert_base=e0)
        torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)
    side = torch.cuda.Stream(device=dev)   # MXFP4 dispatch, concurrent with the GEMV
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True, external=True)  # noqa: E731
    g_ev = (ev(), ev())
    with torch.cuda.stream(stream):
        pipe.routing_map.copy_(h_ids)
        pipe.run(stream, side_stream=side)                 # warm-up outside capture
    stream.synchronize()
    stats = pipe.expert_usage_stats.cpu().numpy().view(np.uint32)
    A = int(stats[1])
    R = int(pipe.expert_start_indices[-1].item())
    routed_tokens = int((pipe.restore_token_order.view(cfg.N, cfg.top_k) != -1)
                        .any(dim=1).sum().item())

    # masking is idempotent for a fixed real_token_count, so replays need no map restore
    # The step graph as a user runs it, and the same step with two timing events
    # around the GEMV (recorded from a side stream, so the programmatic launches
    # stay intact).  Event-record nodes add about 3 us of graph overhead to a
    # step, so the headline steps replay the first graph and the GEMV's launch
    # time comes from K further timed steps of the second.
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            pipe.run(stream, side_stream=side)
    graph_t = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph_t, stream=stream):
            pipe.run(stream, gemv_events=g_ev, side_stream=side)

    def timed_steps(n, g, gemv_times=False):
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        gs = []
        for i in range(n):
            with torch.cuda.stream(stream):
                flush.zero_()
                starts[i].record(stream)
                g.replay()
                ends[i].record(stream)
            ends[i].synchronize()
            if gemv_times:
                # gemv events are re-recorded by every replay: read them before the next one
                gs.append(g_ev[0].elapsed_time(g_ev[1]))
        torch.cuda.synchronize()
        return [starts[i].elapsed_time(ends[i]) for i in range(n)], gs

    def barrier():
        if world > 1:
            dist.barrier()

    timed_steps(args.warmup, graph)
    timed_steps(args.warmup, graph_t, True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t_step, _ = timed_steps(args.steps, graph)
        _, t_gemv = timed_steps(args.steps, graph_t, True)
        torch.cuda.synchronize()
    barrier()
    clocks = clk.summary()
    ms_step = max_over_ranks(float(np.mean(t_step)), world, dev)
    ms_gemv = float(np.mean(t_gemv))

    # end to end through the public API, host buffers: one CUDA graph per step
    # holding the H2D copy of the step's inputs from pinned memory (routing
    # inputs first; the activations on a forked stream, overlapping mask and
    # create_indices) and the pipeline, whose combine stores the step's result
    # straight into pinned host memory (a device-accessible pointer under
    # unified addressing), so the result crosses PCIe without a separate copy
    e2e_ms = []
    h2d = h_in.numel()   # routing map, router weights, real_token_count, x (+ alignment gaps)
    d2h = h_out.numel() * 2
    xcopy = torch.cuda.Stream(device=dev)
    rb = pipe.routing_bytes
    e2e_graph = torch.cuda.CUDAGraph()

    def e2e_step_ops():
        cur = torch.cuda.current_stream()
        pipe.inputs[:rb].copy_(h_in[:rb], non_blocking=True)
        fork_x = torch.cuda.Event()
        fork_x.record(cur)
        xcopy.wait_event(fork_x)
        with torch.cuda.stream(xcopy):
            pipe.inputs[rb:].copy_(h_in[rb:], non_blocking=True)
        x_ready = torch.cuda.Event()
        x_ready.record(xcopy)
        pipe.run(cur, side_stream=side, x_ready=x_ready)

    dev_out = pipe.output
    pipe.output = h_out                                   # the combine's output buffer
    with torch.cuda.stream(stream):
        e2e_step_ops()                                    # warm-up outside capture
        with torch.cuda.graph(e2e_graph, stream=stream):
            e2e_step_ops()
    pipe.output = dev_out
    stream.synchronize()
    for i in range(args.warmup + args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            flush.zero_()
            e0.record(stream)
            e2e_graph.replay()
            e1.record(stream)
        e1.synchronize()
        if i >= args.warmup:
            e2e_ms.append(e0.elapsed_time(e1))
    torch.cuda.synchronize()
    # the result that reached the host is the device step's result
    with torch.cuda.stream(stream):
        graph.replay()
    stream.synchronize()
    assert torch.equal(h_out.view(torch.int16), pipe.output.cpu().view(torch.int16))
    e2e_step = max_over_ranks(float(np.mean(e2e_ms)), world, dev)

    peak, peak_src = measured_peaks()
    bytes_ = algorithmic_bytes(cfg, mode, A, R, routed_tokens)
    gemv_gbs = bytes_["grouped_gemv"] / (ms_gemv * 1e-3) / 1e9
    total_bytes = sum(bytes_.values())
    line = {
        "metric": METRIC,
        "value": job_rate(R, world, ms_step),
        "unit": "routed pairs/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp4xbf16->f32" if mode == "w4a16" else "fp4xfp4->f32",
        "data": "synthetic (seeded; weights N(0,0.02) quantised to NVFP4 on device)",
        "config": dict(workload_config(cfg, mode, R, A),
                       l2="flushed before every step (512 MiB memset outside the timed events)",
                       graph=("one CUDA graph per step: mask + create_indices, GEMV, "
                              "combine, chained by programmatic dependent launch, the "
                              "dispatch on a stream forked after mask + create_indices, "
                              "beside the GEMV; the GEMV's launch time from K more steps of "
                              "the same graph with timing events around it")),
        "roofline": {"kernel": "grouped_gemv_nvfp4", "bound": "hbm", "achieved": gemv_gbs,
                     "peak": peak, "unit": "GB/s", "frac": gemv_gbs / peak,
                     "traffic": profiled_traffic(cfg.name),
                     "algorithmic_bytes": bytes_["grouped_gemv"], "us_per_launch": ms_gemv * 1e3,
                     "peak_source": peak_src},
        "pipeline_roofline": {"algorithmic_bytes": total_bytes,
                              "achieved_gbs": total_bytes / (ms_step * 1e-3) / 1e9,
                              "frac": total_bytes / (ms_step * 1e-3) / 1e9 / peak,
                              "bytes_by_kernel": bytes_},
        "e2e": {"value": job_rate(R, world, e2e_step), "unit": "routed pairs/s",
                "ms_per_step": e2e_step, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": pipe.launches_per_run() * args.steps,
        "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, mode, args.cpu_sample_tokens)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph, graph_t, e2e_graph


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
