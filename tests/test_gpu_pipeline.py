"""End-to-end GPU parity on the five workloads at their full sizes, in the
launch configuration the benchmark times (RoutingPipeline.run).

Indices and recv_counts are compared in full; MXFP4 rows, NVFP4 activation
codes, GEMV outputs and combined rows on samples the oracle computes one by
one.  The combine check uses the oracle's own chain (fp64 GEMV outputs, no
intermediate rounding), so its bound adds the bf16 rounding of the GPU's
expert outputs: sum_j |w_j| * |y_j| * 2^-8.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from permute_fp4_dispatch_b200.build import build
from permute_fp4_dispatch_b200.pipeline import RoutingPipeline
import permute_fp4_dispatch_b200 as moe
from tests.gpu_helpers import (assert_float_parity, check_indices, host_bf16_f64, host_u32,
                               load_inputs, oracle_weights, pipeline_indices,
                               quantize_all_weights)

pytestmark = pytest.mark.gpu

CONFIGS = ["tiny", "decode_30b_a3b", "decode_large_expert", "prefill_index_stress",
           "gpt_oss_120b_w4a4"]


@pytest.fixture(scope="module", autouse=True)
def cuda_library():
    build()
    moe.library()
    yield
    assert moe.moe_get_device_error(clear=True) == 0


def make_pipeline(cfg, mode):
    return RoutingPipeline(cfg.N, cfg.K, cfg.E, cfg.top_k, cfg.N_out, mode=mode,
                           epilogue=cfg.epilogue)


@pytest.mark.parametrize("name", CONFIGS)
def test_pipeline_full_size(name):
    cfg = wl.config(name)
    rng = np.random.default_rng(11)
    x = wl.activations_bf16(cfg)
    ids = wl.routing(cfg)
    rw = wl.router_weights(cfg)
    ids_m = oracle.mask_padding(ids, cfg.real)
    ref_idx = oracle.create_indices(ids_m, cfg.E)
    R = int(ref_idx["expert_start_indices"][-1])
    for mode in cfg.modes:
        pipe = make_pipeline(cfg, mode)
        load_inputs(pipe, cfg, x, ids, rw)
        quantize_all_weights(pipe, cfg)
        pipe.run()
        torch.cuda.synchronize()

        # step 1 + 2: the masked map and the grouping, in full
        np.testing.assert_array_equal(pipe.routing_map.cpu().numpy(), ids_m)
        check_indices(pipeline_indices(pipe), ref_idx, cfg.slots)
        # step 3: sampled rows of the MXFP4 buffer, all counts
        rows = rng.choice(R, size=min(R, 256), replace=False)
        tok = ref_idx["token_expert_order"][rows] // cfg.top_k
        np.testing.assert_array_equal(pipe.recv_buf[torch.from_numpy(rows).cuda()].cpu().numpy(),
                                      oracle.mxfp4_encode_rows(x[tok]))
        valid = ids_m[(ids_m >= 0) & (ids_m < cfg.E)]
        np.testing.assert_array_equal(host_u32(pipe.recv_counts),
                                      np.bincount(valid, minlength=cfg.E))
        # step 4a (W4A4): activation codes in full
        if mode == "w4a4":
            xq, sfa = oracle.nvfp4_quantize_bf16(x, 1.0)
            np.testing.assert_array_equal(pipe.sfa.cpu().numpy(), sfa)
            np.testing.assert_array_equal(pipe.xq.cpu().numpy(), xq)
        # sampled tokens: their experts' weights through the oracle
        real_rows = np.arange(min(cfg.real, cfg.N))
        toks = rng.choice(real_rows, size=min(3, real_rows.size), replace=False)
        experts = sorted({int(e) for t in toks for e in ids_m[t] if 0 <= e < cfg.E})
        wq, sfw, gw = oracle_weights(cfg, experts)
        sub = {e: i for i, e in enumerate(experts)}
        np.testing.assert_array_equal(pipe.wq[experts].cpu().numpy(), wq)
        np.testing.assert_array_equal(pipe.sfw[experts].cpu().numpy(), sfw)
        cols = np.sort(rng.choice(cfg.N_out, size=min(cfg.N_out, 48), replace=False))
        y_gpu = host_bf16_f64(pipe.expert_out)
        out_gpu = host_bf16_f64(pipe.output)
        for t in toks:
            local = np.array([[sub.get(int(e), -1) for e in ids_m[t]]], np.int64)
            yref = np.zeros((cfg.top_k, cols.size))
            for j in range(cfg.top_k):
                samples = [(0, j, int(n)) for n in cols]
                if mode == "w4a16":
                    yref[j] = oracle.gemv_elements("w4a16", local, wq, sfw, gw, samples,
                                                   act_bf16=x[t:t + 1])
                else:
                    yref[j] = oracle.gemv_elements("w4a4", local, wq, sfw, gw, samples,
                                                   xq=xq[t:t + 1], sfa=sfa[t:t + 1])
                assert_float_parity(y_gpu[t, j, cols], yref[j], what=f"{name} gemv t={t} j={j}")
            w = rw[t].astype(np.float64)
            comb = (w[:, None] * yref).sum(0)
            if cfg.epilogue == "scale":
                comb *= pipe.alpha
            extra = (np.abs(w)[:, None] * np.abs(yref)).sum(0) * 2.0 ** -8
            assert_float_parity(out_gpu[t, cols], comb, extra=extra, what=f"{name} combine t={t}")
        # padding rows combine to epi(0) = 0
        assert np.all(out_gpu[cfg.real:] == 0.0)


def test_graph_replay_follows_real_token_count():
    """The captured pipeline reads real_token_count at replay time."""
    cfg = wl.config("tiny")
    x, ids, rw = wl.activations_bf16(cfg), wl.routing(cfg), wl.router_weights(cfg)
    pipe = make_pipeline(cfg, "w4a16")
    load_inputs(pipe, cfg, x, ids, rw)
    quantize_all_weights(pipe, cfg)
    pipe.run()                                   # warm-up outside capture
    torch.cuda.synchronize()
    ids_t = pipe.routing_map.clone()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            pipe.run(stream=s)
    for real in (13, 5, 16, 0):
        pipe.routing_map.copy_(torch.from_numpy(ids).cuda())
        pipe.real_token_count.fill_(real)
        g.replay()
        torch.cuda.synchronize()
        ref = oracle.create_indices(oracle.mask_padding(ids, real), cfg.E)
        check_indices(pipeline_indices(pipe), ref, cfg.slots)
        out = host_bf16_f64(pipe.output)
        assert np.all(out[real:] == 0.0)
    del ids_t


def test_pipeline_repeatable_bitwise():
    cfg = wl.config("decode_30b_a3b")
    x, ids, rw = wl.activations_bf16(cfg), wl.routing(cfg), wl.router_weights(cfg)
    pipe = make_pipeline(cfg, "w4a16")
    load_inputs(pipe, cfg, x, ids, rw)
    quantize_all_weights(pipe, cfg)
    outs = []
    for _ in range(3):
        pipe.routing_map.copy_(torch.from_numpy(ids).cuda())
        pipe.run()
        outs.append((pipe.output.clone(), pipe.recv_buf.clone(), pipe.expert_out.clone()))
    torch.cuda.synchronize()
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))


@pytest.mark.parametrize("order,fork", [("routing_first", "gemv"), ("routing_first", "routing"),
                                        ("gemv_groups", None)])
@pytest.mark.parametrize("mode", ["w4a16", "w4a4"])
def test_forked_dispatch_graph_matches_sequential(mode, order, fork):
    """The side-stream work (dispatch; create_indices too in the gemv_groups
    order) inside a captured graph gives the same bytes as the one-stream
    order, for every step's output, in both step orders."""
    cfg = wl.config("decode_30b_a3b")
    x, ids, rw = wl.activations_bf16(cfg), wl.routing(cfg), wl.router_weights(cfg)
    pipe = make_pipeline(cfg, mode)
    pipe.order = order
    if fork:
        pipe.dispatch_fork = fork
    load_inputs(pipe, cfg, x, ids, rw)
    quantize_all_weights(pipe, cfg)
    pipe.run()
    torch.cuda.synchronize()
    ref = [t.clone() for t in (pipe.output, pipe.recv_buf, pipe.recv_counts, pipe.expert_out,
                               pipe.token_expert_order, pipe.restore_token_order)]
    for t in (pipe.output, pipe.recv_buf, pipe.expert_out):
        t.view(torch.uint8).fill_(0x5A)
    main, side = torch.cuda.Stream(), torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(main):
        pipe.run(stream=main, side_stream=side)      # warm-up outside capture
        with torch.cuda.graph(g, stream=main):
            pipe.run(stream=main, side_stream=side)
    for _ in range(2):
        for t in (pipe.output, pipe.recv_buf, pipe.expert_out):
            t.view(torch.uint8).fill_(0x5A)
        pipe.routing_map.copy_(torch.from_numpy(ids).cuda())
        g.replay()
        torch.cuda.synchronize()
        got = (pipe.output, pipe.recv_buf, pipe.recv_counts, pipe.expert_out,
               pipe.token_expert_order, pipe.restore_token_order)
        for a, b in zip(ref, got):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
