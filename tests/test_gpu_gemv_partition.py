"""GPU parity of the grouped GEMV where its work partition is stressed:

* more (expert, pass) pairs than persistent CTAs (the round-aligned
  partition branch), in W4A16 and W4A4, through the decode variant and the
  host's own choice;
* a skewed routing where one expert needs many passes;
* every routed pair and every column of the decode 30B-A3B-like workload at
  full size, through the pipeline the benchmark times.

Element by element against the oracle's fp64 value within
max(1e-3, 5e-3 * |ref|) (FlashRT "grouped-moe-gemv" card, Available
functions: grouped_w4a16_gemv_bf16 / grouped_w4a4_gemv_bf16)."""
import numpy as np
import pytest
import torch

import oracle
import permute_fp4_dispatch_b200 as moe
import workloads as wl
from permute_fp4_dispatch_b200.build import build
from permute_fp4_dispatch_b200.pipeline import RoutingPipeline
from tests.gpu_helpers import (assert_float_parity, decode_passes, host_bf16_bits, host_bf16_f64,
                               load_inputs, oracle_gemv_rows_threaded, oracle_weights,
                               quantize_all_weights)

pytestmark = pytest.mark.gpu

SENTINEL = 0x4B1D


@pytest.fixture(scope="module", autouse=True)
def cuda_library():
    build()
    moe.library()
    yield
    assert moe.moe_get_device_error(clear=True) == 0


def run_case(cfg, mode, variant, monkeypatch, g_a=1.0):
    if variant != "auto":
        monkeypatch.setenv("MOE_GEMV_VARIANT", variant)
    x, ids, rw = wl.activations_bf16(cfg), wl.routing(cfg), wl.router_weights(cfg)
    pipe = RoutingPipeline(cfg.N, cfg.K, cfg.E, cfg.top_k, cfg.N_out, mode=mode,
                           act_global=g_a, dispatch=False)
    load_inputs(pipe, cfg, x, ids, rw)
    quantize_all_weights(pipe, cfg)
    pipe.expert_out.view(torch.int16).fill_(SENTINEL)
    pipe.mask()
    pipe.create_indices()
    if mode == "w4a4":
        pipe.quantize_activations()
    pipe.gemv()
    torch.cuda.synchronize()
    ids_m = oracle.mask_padding(ids, cfg.real)
    wq, sfw, gw = oracle_weights(cfg, range(cfg.E))
    if mode == "w4a16":
        ref = oracle_gemv_rows_threaded("w4a16", ids_m, wq, sfw, gw, act_bf16=x)
    else:
        xq, sfa = oracle.nvfp4_quantize_bf16(x, g_a)
        np.testing.assert_array_equal(pipe.xq.cpu().numpy(), xq)
        ref = oracle_gemv_rows_threaded("w4a4", ids_m, wq, sfw, gw, xq=xq, sfa=sfa, g_a=g_a)
    routed = ~np.isnan(ref[..., 0])
    assert np.all(host_bf16_bits(pipe.expert_out)[~routed] == SENTINEL)
    assert_float_parity(host_bf16_f64(pipe.expert_out)[routed], ref[routed],
                        what=f"{cfg.name} {mode} {variant}")
    return ids_m


# 256 experts at K = 2048 with about ten tokens each: more (expert, pass)
# pairs than the GPU has SMs, so every CTA takes a round-aligned range that
# spans passes of different experts.
MANY = wl.small_config("many_passes", N=320, real=320, K=2048, E=256, top_k=8, N_out=64, seed=21)
# one expert takes a large share of the pairs: many passes of one expert
SKEW = wl.small_config("skewed", N=400, real=391, K=1024, E=64, top_k=4, N_out=48,
                       routing="zipf", zipf_s=1.6, seed=22)


@pytest.mark.parametrize("variant", ["mma", "bs", "auto"])
@pytest.mark.parametrize("mode", ["w4a16", "w4a4"])
def test_gemv_more_passes_than_ctas(mode, variant, monkeypatch):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    ids = oracle.mask_padding(wl.routing(MANY), MANY.real)
    assert decode_passes(ids, MANY.E, 16) > sms      # the case this test exists for
    g_a = 1.0 if mode == "w4a16" else float(np.float32(0.75))
    run_case(MANY, mode, variant, monkeypatch, g_a)


@pytest.mark.parametrize("variant", ["mma", "tc", "bs", "auto"])
@pytest.mark.parametrize("mode", ["w4a16", "w4a4"])
def test_gemv_skewed_expert_many_passes(mode, variant, monkeypatch):
    ids = oracle.mask_padding(wl.routing(SKEW), SKEW.real)
    counts = np.bincount(ids[ids >= 0], minlength=SKEW.E)
    assert counts.max() >= 8 * 16                    # one expert spans 8+ passes of 16
    run_case(SKEW, mode, variant, monkeypatch)


def test_gemv_decode_full_size_every_element():
    """decode_30b_a3b through RoutingPipeline.run (the benchmark's launch
    configuration): every routed pair, every column."""
    cfg = wl.config("decode_30b_a3b")
    x, ids, rw = wl.activations_bf16(cfg), wl.routing(cfg), wl.router_weights(cfg)
    pipe = RoutingPipeline(cfg.N, cfg.K, cfg.E, cfg.top_k, cfg.N_out, mode="w4a16",
                           epilogue=cfg.epilogue)
    load_inputs(pipe, cfg, x, ids, rw)
    quantize_all_weights(pipe, cfg)
    main, side = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(main):
        pipe.run(stream=main, side_stream=side)
    torch.cuda.synchronize()
    ids_m = oracle.mask_padding(ids, cfg.real)
    wq, sfw, gw = oracle_weights(cfg, range(cfg.E))
    np.testing.assert_array_equal(pipe.wq.cpu().numpy(), wq)
    ref = oracle_gemv_rows_threaded("w4a16", ids_m, wq, sfw, gw, act_bf16=x)
    routed = ~np.isnan(ref[..., 0])
    assert routed.sum() == cfg.N * cfg.top_k
    assert_float_parity(host_bf16_f64(pipe.expert_out)[routed], ref[routed],
                        what="decode_30b_a3b all pairs")
    # the combined rows too, against the oracle's combine of the GPU's expert outputs
    y_bits = host_bf16_bits(pipe.expert_out)
    comb = oracle.combine(y_bits, rw, ids_m, cfg.E, cfg.epilogue)
    assert_float_parity(host_bf16_f64(pipe.output), comb, what="decode_30b_a3b combine")
