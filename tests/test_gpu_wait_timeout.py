"""Bounded pipeline waits of the grouped GEMV.

Every mbarrier wait in the GEMV kernels has a time limit; when it runs out
the kernel sets MOE_DEVERR_WAIT_TIMEOUT, stops issuing work, waits (again
with a limit) for the copies it already started, releases its tensor memory
and returns.  These tests make a wait run out on purpose -- through the
library's test hook MOE_TEST_WAIT_LIMIT_NS, read at every GEMV launch, set to
0, under which a wait passes only if its stage has already landed, so the
first wait for a copy still in flight expires -- and check that the error bit is raised, that the call returns, and that
the next call with the normal limit matches the oracle again.  Nothing here
faults or hangs the GPU: the data always arrives, only the wait gives up
early.
"""
import numpy as np
import pytest
import torch

import oracle
import permute_fp4_dispatch_b200 as moe
import workloads as wl
from permute_fp4_dispatch_b200.build import build
from permute_fp4_dispatch_b200.pipeline import RoutingPipeline
from tests.gpu_helpers import (assert_float_parity, host_bf16_f64, load_inputs, oracle_weights,
                               quantize_all_weights)

pytestmark = pytest.mark.gpu

CFG = wl.small_config("timeout", N=48, real=45, K=2048, E=6, top_k=2, N_out=96, seed=31)


@pytest.fixture(scope="module", autouse=True)
def cuda_library():
    build()
    moe.library()
    moe.moe_get_device_error(clear=True)
    yield
    assert moe.moe_get_device_error(clear=True) == 0


@pytest.mark.parametrize("variant,mode", [("mma", "w4a16"), ("tc", "w4a16"), ("bs", "w4a4")])
def test_expired_wait_is_reported_and_the_next_call_is_exact(variant, mode, monkeypatch):
    monkeypatch.setenv("MOE_GEMV_VARIANT", variant)
    x, ids, rw = wl.activations_bf16(CFG), wl.routing(CFG), wl.router_weights(CFG)
    pipe = RoutingPipeline(CFG.N, CFG.K, CFG.E, CFG.top_k, CFG.N_out, mode=mode, dispatch=False)
    load_inputs(pipe, CFG, x, ids, rw)
    quantize_all_weights(pipe, CFG)
    pipe.mask()
    pipe.create_indices()
    if mode == "w4a4":
        pipe.quantize_activations()
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(clear=True) == 0

    # a zero limit: the first wait that does not find its stage already there gives up
    monkeypatch.setenv("MOE_TEST_WAIT_LIMIT_NS", "0")
    flags = 0
    for _ in range(3):
        pipe.gemv()
        torch.cuda.synchronize()                 # the kernel returned
        flags = moe.moe_get_device_error(clear=True)
        if flags:
            break
    assert flags == moe.MOE_DEVERR_WAIT_TIMEOUT

    # the context is intact and the normal limit gives the exact result again
    monkeypatch.delenv("MOE_TEST_WAIT_LIMIT_NS")
    pipe.expert_out.zero_()
    pipe.gemv()
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(clear=True) == 0
    ids_m = oracle.mask_padding(ids, CFG.real)
    wq, sfw, gw = oracle_weights(CFG, range(CFG.E))
    if mode == "w4a16":
        ref = oracle.grouped_gemv("w4a16", ids_m, wq, sfw, gw, act_bf16=x)
    else:
        xq, sfa = oracle.nvfp4_quantize_bf16(x, 1.0)
        ref = oracle.grouped_gemv("w4a4", ids_m, wq, sfw, gw, xq=xq, sfa=sfa)
    routed = ~np.isnan(ref[..., 0])
    assert_float_parity(host_bf16_f64(pipe.expert_out)[routed], ref[routed], what=variant)
