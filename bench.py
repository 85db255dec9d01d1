#!/usr/bin/env python
"""Benchmark of the single-GPU MoE token-routing step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config decode_30b_a3b]

One step = the whole hot path over one batch: mask -> create_indices ->
MXFP4 dispatch -> [NVFP4 activation quantisation] -> grouped NVFP4 GEMV ->
combine, replayed as one CUDA graph.  Inputs are resident in HBM when the
timed region starts; L2 is flushed before every timed step (a 512 MiB memset
outside the timed events; ``--flush write+read`` adds a 512 MiB read so the
step does not write back the flush's own dirty lines).  Metric: routed
token-expert pairs per second, whole job.  With N > 1 (torchrun) every rank runs an independent
replica of the workload (weak scaling; the path has no exchange step).

Also reported: the grouped GEMV's achieved HBM bandwidth against the
measured copy bandwidth (roofline), every kernel's time and HBM fraction,
the pipeline's algorithmic-byte fraction, an end-to-end figure through the
public API with host buffers, SM clocks sampled during the timed region, the
CPU oracle timed on a bounded sample of the same workload (rank 0, N = 1),
and under "workloads" the same figures for the other synthetic workloads
(tiny, decode large-expert, prefill index stress, gpt-oss-shaped W4A4).

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
    ap.add_argument("--no-workloads", action="store_true",
                    help="time the headline workload only")
    ap.add_argument("--flush", choices=["write", "write+read"], default="write",
                    help="how L2 is flushed between timed steps")
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


def measured_peaks() -> dict:
    """HBM copy bandwidth and dense bf16 tensor throughput measured on this
    pool's B200s (MEASURED_PEAKS.json), else the recipe's fallback figures."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "source": "MEASURED_PEAKS.json hbm_gbs / bf16_tflops (of measured)"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
            "source": "profiling-recipe fallback 6.65 TB/s, 1.59 PFLOP/s (of fallback)"}


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
    # the fused dispatch + quantisation reads every row once and writes both encodings
    b["dispatch_quant"] = (N * K * 2 + R * stride + E * 4 + N * (K // 2 + K // 16)
                           if mode == "w4a4" else 0)
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
# which entries of the byte model each launch of a step accounts for
KERNEL_BYTES = {"mask+create_indices": ("mask", "create_indices"),
                "dispatch+quant_act": ("dispatch_quant",)}
OTHER_WORKLOADS = ("tiny", "decode_large_expert", "prefill_index_stress", "gpt_oss_120b_w4a4")
WORKLOAD_STEPS_CAP = 20    # timed steps per workload beyond the headline one


def dense_flops(cfg, R: int) -> int:
    """2 * R * N_out * K: the GEMV's multiply-adds over the routed pairs."""
    return 2 * R * cfg.N_out * cfg.K


def count_kernel_nodes(graph):
    """Kernel nodes of a captured CUDA graph (captured with keep_graph=True):
    the launches one replay makes.  None when the graph cannot be inspected."""
    try:
        from cuda.bindings import runtime as rt
        g = rt.cudaGraph_t(init_value=graph.raw_cuda_graph())
        err, _, n = rt.cudaGraphGetNodes(g, 0)
        err, nodes, n = rt.cudaGraphGetNodes(g, n)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        kernel = rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
        return sum(1 for nd in nodes[:n] if rt.cudaGraphNodeGetType(nd)[1] == kernel)
    except Exception:
        return None


def describe_step_graph(pipe) -> str:
    if pipe.order == "gemv_groups":
        return ("one CUDA graph per step: mask, the GEMV on the routing map (it groups the "
                "pairs in-kernel) and the combine, chained by programmatic dependent launch; "
                "create_indices and the MXFP4 dispatch on a stream forked after the mask")
    return ("one CUDA graph per step: mask + create_indices, GEMV, combine, chained by "
            "programmatic dependent launch; the MXFP4 dispatch on a stream forked after "
            "mask + create_indices, beside the GEMV")


class L2Flush:
    """Between timed steps: write a buffer larger than L2, which evicts every
    line of the step's inputs and outputs; mode "write+read" then reads
    another one, so that the next step starts with clean lines of unrelated
    data instead of the flush buffer's dirty ones.  Runs outside the timed
    events."""

    def __init__(self, dev, mode: str):
        import torch
        self.mode = mode
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev) \
            if mode == "write+read" else None

    def __call__(self):
        self.w.zero_()
        if self.r is not None:
            self.r.sum()

    def describe(self) -> str:
        if self.r is None:
            return "flushed before every step: 512 MiB memset, outside the timed events"
        return ("flushed before every step: 512 MiB memset then a 512 MiB read, outside the "
                "timed events (no step input or output left in L2, no dirty flush lines)")


def make_pipeline(cfg, mode, dev, weights: str):
    """Pipeline with the workload's inputs resident on the device and its
    expert library quantised by the library's own kernel.  ``weights``:
    "numpy" draws them by the seeded recipe (the CPU oracle's inputs), "torch"
    draws N(0, 0.02) with torch's CUDA generator (same distribution, seconds
    instead of minutes for multi-GB libraries)."""
    import torch
    from permute_fp4_dispatch_b200.pipeline import RoutingPipeline
    pipe = RoutingPipeline(cfg.N, cfg.K, cfg.E, cfg.top_k, cfg.N_out, mode=mode,
                           epilogue=cfg.epilogue, device=dev)
    h_in, views = pipe.host_inputs()
    x, ids, rw = wl.activations_bf16(cfg), wl.routing(cfg), wl.router_weights(cfg)
    views["x"].copy_(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16))
    views["routing_map"].copy_(torch.from_numpy(ids))
    views["router_weights"].copy_(torch.from_numpy(rw))
    views["real_token_count"].fill_(cfg.real)
    pipe.inputs.copy_(h_in)
    chunk = 16
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000 + cfg.seed)
    for e0 in range(0, cfg.E, chunk):
        e1 = min(cfg.E, e0 + chunk)
        if weights == "numpy":
            w = torch.from_numpy(wl.expert_weights_f32_many(cfg, range(e0, e1))).to(dev)
        else:
            w = torch.randn((e1 - e0, cfg.N_out, cfg.K), generator=gen, device=dev) * 0.02
        pipe.quantize_weights(w, expert_base=e0)
        del w
    torch.cuda.synchronize()
    return pipe, h_in


def measure_workload(cfg, mode, dev, steps, warmup, flush, peaks, weights, headline=False,
                     world=1):
    """Device-timed steps of the captured pipeline, per-kernel times, the
    whole-step and per-kernel HBM fractions, and the end-to-end step through
    the public API with host buffers.  Returns (record, extras)."""
    import torch
    pipe, h_in = make_pipeline(cfg, mode, dev, weights)
    h_out = torch.empty((cfg.N, cfg.N_out), dtype=torch.bfloat16).pin_memory()
    stream = torch.cuda.Stream(device=dev)
    side = torch.cuda.Stream(device=dev)   # MXFP4 dispatch, concurrent with the GEMV
    with torch.cuda.stream(stream):
        pipe.run(stream, side_stream=side)               # warm-up outside capture
    stream.synchronize()
    stats = pipe.expert_usage_stats.cpu().numpy().view(np.uint32)
    A = int(stats[1])
    R = int(pipe.expert_start_indices[-1].item())
    routed_tokens = int((pipe.restore_token_order.view(cfg.N, cfg.top_k) != -1)
                        .any(dim=1).sum().item())
    hbm_peak, bf16_peak = peaks["hbm_gbs"], peaks["bf16_tflops"]

    # masking is idempotent for a fixed real_token_count, so replays need no map restore
    graph = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            pipe.run(stream, side_stream=side)
    graph.instantiate()
    launches = count_kernel_nodes(graph)
    if launches is None:
        launches = pipe.launches_per_run()

    def replay_times(n, g, after=None):
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        extra = []
        for i in range(n):
            with torch.cuda.stream(stream):
                flush()
                starts[i].record(stream)
                g.replay()
                ends[i].record(stream)
            ends[i].synchronize()
            if after is not None:
                extra.append(after())
        torch.cuda.synchronize()
        return [starts[i].elapsed_time(ends[i]) for i in range(n)], extra

    replay_times(warmup, graph)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    t_step, _ = replay_times(steps, graph)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    ms_step = max_over_ranks(float(np.mean(t_step)), world, dev)

    # per-kernel times: a CUDA graph of the same steps on one stream with a
    # timing event recorded between consecutive kernels (each kernel then
    # waits for the previous one to finish: no programmatic overlap), L2
    # flushed before every replay
    steps_k = pipe.kernel_steps()
    names = [n for n, _ in steps_k]
    kev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(names) + 1)]
    kgraph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        for _, fn in steps_k:                            # warm-up outside capture
            fn(stream)
        with torch.cuda.graph(kgraph, stream=stream):
            kev[0].record(stream)
            for i, (_, fn) in enumerate(steps_k):
                fn(stream)
                kev[i + 1].record(stream)
    _, rows = replay_times(warmup + steps, kgraph,
                           after=lambda: [kev[i].elapsed_time(kev[i + 1]) for i in range(len(names))])
    per = {n: [row[i] for row in rows[warmup:]] for i, n in enumerate(names)}
    model = algorithmic_bytes(cfg, mode, A, R, routed_tokens)
    bytes_ = {n: sum(model[k] for k in KERNEL_BYTES.get(n, (n,))) for n in names}
    kernels = {}
    for n in names:
        us = float(np.mean(per[n])) * 1e3
        b = bytes_[n]
        rec = {"us": us, "algorithmic_bytes": b, "gbs": b / (us * 1e-6) / 1e9,
               "hbm_frac": b / (us * 1e-6) / 1e9 / hbm_peak}
        if n == "grouped_gemv":
            fl = dense_flops(cfg, R)
            rec["tflops"] = fl / (us * 1e-6) / 1e12
            rec["tensor_frac_of_bf16_peak"] = rec["tflops"] / bf16_peak
        kernels[n] = rec
    total_bytes = sum(bytes_.values())

    # end to end through the public API, host buffers: one CUDA graph per step
    # holding the H2D copy of the step's inputs from pinned memory (routing
    # inputs first; the activations on a forked stream, overlapping mask and
    # create_indices) and the pipeline, whose combine stores the step's result
    # straight into pinned host memory (a device-accessible pointer under
    # unified addressing), so the result crosses PCIe without a separate copy
    xcopy = torch.cuda.Stream(device=dev)
    rb = pipe.routing_bytes

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

    e2e_graph = torch.cuda.CUDAGraph()
    dev_out = pipe.output
    pipe.output = h_out                                   # the combine's output buffer
    with torch.cuda.stream(stream):
        e2e_step_ops()                                    # warm-up outside capture
        with torch.cuda.graph(e2e_graph, stream=stream):
            e2e_step_ops()
    pipe.output = dev_out
    stream.synchronize()
    t_e2e, _ = replay_times(warmup + steps, e2e_graph)
    e2e_ms = max_over_ranks(float(np.mean(t_e2e[warmup:])), world, dev)
    # the result that reached the host is the device step's result
    with torch.cuda.stream(stream):
        graph.replay()
    stream.synchronize()
    assert torch.equal(h_out.view(torch.int16), pipe.output.cpu().view(torch.int16))

    record = {
        "mode": mode, "routed_pairs": R, "active_experts": A, "steps": steps,
        "us_per_step": ms_step * 1e3, "pairs_per_s": job_rate(R, world, ms_step),
        "kernels_us_source": ("CUDA events between consecutive kernels inside one captured "
                              "graph of the same steps (serialised, no programmatic overlap)"),
        "kernels": kernels,
        "pipeline_hbm": {"algorithmic_bytes": total_bytes,
                         "achieved_gbs": total_bytes / (ms_step * 1e-3) / 1e9,
                         "frac": total_bytes / (ms_step * 1e-3) / 1e9 / hbm_peak},
        "e2e": {"us_per_step": e2e_ms * 1e3, "pairs_per_s": job_rate(R, world, e2e_ms),
                "h2d_bytes_per_step": h_in.numel(), "d2h_bytes_per_step": h_out.numel() * 2},
        "weights": ("seeded numpy recipe" if weights == "numpy"
                    else "N(0,0.02) from torch's CUDA generator"),
        "gpu_launches_per_step": launches,
        "step_graph": describe_step_graph(pipe),
    }
    extras = {"pipe": pipe, "graph": graph, "kgraph": kgraph, "stream": stream, "side": side,
              "bytes": bytes_,
              "replay_times": replay_times, "e2e_graph": e2e_graph, "A": A, "R": R,
              "routed_tokens": routed_tokens}
    return record, extras


def run_ours(args, rank, world, local_rank):
    import torch

    from permute_fp4_dispatch_b200.build import build

    build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = wl.config(args.config)
    mode = cfg.modes[0]
    peaks = measured_peaks()
    flush = L2Flush(dev, args.flush)

    with ClockSampler(local_rank) as clk:
        head, ex = measure_workload(cfg, mode, dev, args.steps, args.warmup, flush, peaks,
                                    weights="numpy", headline=True, world=world)
        # the GEMV's own launch time: K further steps of the same graph with two
        # timing events around the GEMV, recorded from a side stream so the
        # programmatic launches stay intact (event-record nodes add graph time,
        # so the headline steps replay the graph without them)
        pipe, stream, side = ex["pipe"], ex["stream"], ex["side"]
        ev = lambda: torch.cuda.Event(enable_timing=True, external=True)  # noqa: E731
        g_ev = (ev(), ev())
        graph_t = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(graph_t, stream=stream):
                pipe.run(stream, gemv_events=g_ev, side_stream=side)
        ex["replay_times"](args.warmup, graph_t)
        _, t_gemv = ex["replay_times"](args.steps, graph_t,
                                       after=lambda: g_ev[0].elapsed_time(g_ev[1]))
        workloads = {}
        if world == 1 and not args.no_workloads:
            for name in OTHER_WORKLOADS:
                if name == cfg.name:
                    continue
                wc = wl.config(name)
                recs = {}
                for m in wc.modes:
                    rec, wex = measure_workload(
                        wc, m, dev, min(args.steps, WORKLOAD_STEPS_CAP), min(args.warmup, 3),
                        flush, peaks, weights="numpy" if name == "tiny" else "torch")
                    recs[m] = rec
                    del wex
                    torch.cuda.empty_cache()
                workloads[name] = recs if len(recs) > 1 else next(iter(recs.values()))
    clocks = clk.summary()

    ms_step = head["us_per_step"] * 1e-3
    ms_gemv = float(np.mean(t_gemv))
    R, A = ex["R"], ex["A"]
    bytes_ = ex["bytes"]
    hbm = peaks["hbm_gbs"]
    gemv_gbs = bytes_["grouped_gemv"] / (ms_gemv * 1e-3) / 1e9
    total_bytes = sum(bytes_.values())
    line = {
        "metric": METRIC,
        "value": head["pairs_per_s"],
        "unit": "routed pairs/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp4xbf16->f32" if mode == "w4a16" else "fp4xfp4->f32",
        "data": "synthetic (seeded; weights N(0,0.02) quantised to NVFP4 on device)",
        "config": dict(workload_config(cfg, mode, R, A),
                       l2=flush.describe(),
                       graph=head["step_graph"] + ("; the GEMV's launch time from K more "
                                                    "steps of the same graph with timing "
                                                    "events around it")),
        "roofline": {"kernel": "grouped_gemv_nvfp4", "bound": "hbm", "achieved": gemv_gbs,
                     "peak": hbm, "unit": "GB/s", "frac": gemv_gbs / hbm,
                     "traffic": profiled_traffic(cfg.name),
                     "algorithmic_bytes": bytes_["grouped_gemv"], "us_per_launch": ms_gemv * 1e3,
                     "peak_source": peaks["source"]},
        "pipeline_roofline": {"algorithmic_bytes": total_bytes,
                              "achieved_gbs": total_bytes / (ms_step * 1e-3) / 1e9,
                              "frac": total_bytes / (ms_step * 1e-3) / 1e9 / hbm,
                              "bytes_by_kernel": bytes_},
        "kernels": head["kernels"],
        "e2e": {"value": head["e2e"]["pairs_per_s"], "unit": "routed pairs/s",
                "ms_per_step": head["e2e"]["us_per_step"] * 1e-3,
                "h2d_bytes_per_step": head["e2e"]["h2d_bytes_per_step"],
                "d2h_bytes_per_step": head["e2e"]["d2h_bytes_per_step"]},
        "gpu_launches": head["gpu_launches_per_step"] * args.steps,
        "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
    }
    if workloads:
        line["workloads"] = workloads
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, mode, args.cpu_sample_tokens)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph_t, ex


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
