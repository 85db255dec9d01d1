"""Shared helpers for the GPU parity tests (torch <-> numpy marshalling, tolerances)."""
import numpy as np
import torch

import oracle
import workloads as wl


def dev(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint32:
        a = a.view(np.int32)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def host_u32(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


def host_bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def host_bf16_f64(t: torch.Tensor) -> np.ndarray:
    return wl.bf16_bits_to_f32(host_bf16_bits(t)).astype(np.float64)


def float_tol(ref: np.ndarray) -> np.ndarray:
    """Per-element bound for fp outputs: 5e-3 relative above a 1e-3 floor."""
    return np.maximum(1e-3, 5e-3 * np.abs(ref))


def assert_float_parity(gpu: np.ndarray, ref: np.ndarray, extra: np.ndarray | float = 0.0,
                        what: str = ""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(gpu - ref)
    bound = float_tol(ref) + extra
    bad = ~(err <= bound)
    if bad.any():
        i = np.flatnonzero(bad.ravel())[:5]
        raise AssertionError(
            f"{what}: {bad.sum()} / {bad.size} elements out of tolerance; first gpu="
            f"{gpu.ravel()[i]}, ref={ref.ravel()[i]}, bound={np.broadcast_to(bound, ref.shape).ravel()[i]}")


def check_indices(gpu: dict, ref: dict, S: int):
    for k in ("token_expert_order", "restore_token_order", "expert_start_indices",
              "expert_usage_stats", "scales_offset"):
        np.testing.assert_array_equal(gpu[k], ref[k], err_msg=k)
    np.testing.assert_array_equal(gpu["expert_ids"], ref["expert_ids"], err_msg="expert_ids")


def pipeline_indices(pipe) -> dict:
    return dict(
        token_expert_order=host_u32(pipe.token_expert_order),
        expert_start_indices=host_u32(pipe.expert_start_indices),
        restore_token_order=host_u32(pipe.restore_token_order),
        expert_ids=pipe.expert_ids.cpu().numpy(),
        expert_usage_stats=host_u32(pipe.expert_usage_stats),
        scales_offset=host_u32(pipe.scales_offset),
    )


def load_inputs(pipe, cfg, x_bits, ids, rw):
    pipe.x.copy_(dev(x_bits))
    pipe.routing_map.copy_(dev(ids))
    pipe.router_weights.copy_(dev(rw))
    pipe.real_token_count.fill_(cfg.real)


def quantize_all_weights(pipe, cfg, chunk: int = 16):
    """GPU-quantise the seeded fp32 weights of every expert, a few at a time."""
    for e0 in range(0, cfg.E, chunk):
        es = list(range(e0, min(cfg.E, e0 + chunk)))
        w = torch.from_numpy(wl.expert_weights_f32_many(cfg, es)).cuda()
        pipe.quantize_weights(w, expert_base=e0)
        torch.cuda.synchronize()


def oracle_weights(cfg, experts):
    return oracle.quantize_weights_nvfp4(wl.expert_weights_f32_many(cfg, experts))


def oracle_gemv_rows_threaded(mode, ids, wq, sfw, gw, act_bf16=None, xq=None, sfa=None,
                              g_a: float = 1.0, rows_per_task: int = 4, threads: int | None = None):
    """oracle.grouped_gemv over every row of ``ids`` [M, top_k], computed in
    independent row chunks on a thread pool (the oracle's C code runs with the
    GIL released).  Same function, same arithmetic per element; only the rows
    are spread over the host cores."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    M = ids.shape[0]
    out = np.full((M, ids.shape[1], wq.shape[1]), np.nan)
    n = threads or max(1, min(32, len(os.sched_getaffinity(0))))

    def run(m0):
        m1 = min(M, m0 + rows_per_task)
        kw = {}
        if act_bf16 is not None:
            kw["act_bf16"] = act_bf16[m0:m1]
        if xq is not None:
            kw["xq"], kw["sfa"] = xq[m0:m1], sfa[m0:m1]
        out[m0:m1] = oracle.grouped_gemv(mode, ids[m0:m1], wq, sfw, gw, g_a=g_a, **kw)

    with ThreadPoolExecutor(n) as ex:
        list(ex.map(run, range(0, M, rows_per_task)))
    return out


def decode_passes(ids: np.ndarray, E: int, tokens_per_pass: int) -> int:
    """(expert, pass) pairs of a routing map when every expert's pairs are
    taken tokens_per_pass at a time."""
    valid = ids[(ids >= 0) & (ids < E)]
    counts = np.bincount(valid, minlength=E)
    return int(((counts + tokens_per_pass - 1) // tokens_per_pass).sum())
