"""GPU parity, step by step: every kernel against the CPU oracle on the same
seeded inputs, through the C ABI (Python binding).  Bit-exact for indices,
counts, FP4 codes and E8M0 / E4M3 scales; fp outputs within
max(1e-3, 5e-3 * |ref|) of the oracle's unrounded fp64 value."""
import numpy as np
import pytest
import torch

import oracle
import permute_fp4_dispatch_b200 as moe
import workloads as wl
from permute_fp4_dispatch_b200.build import build
from permute_fp4_dispatch_b200.pipeline import RoutingPipeline
from tests.gpu_helpers import (assert_float_parity, check_indices, dev, host_bf16_bits,
                               host_bf16_f64, host_u32, load_inputs, oracle_weights,
                               pipeline_indices, quantize_all_weights)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_library():
    build()
    moe.library()
    yield
    assert moe.moe_get_device_error(clear=True) == 0


# ------------------------------------------------------------------ step 1
@pytest.mark.parametrize("N,k,real,tp", [(16, 2, 13, 0), (640, 8, 512, 0), (4096, 4, 3000, 0),
                                         (16, 2, 0, 0), (16, 2, -3, 0), (16, 2, 99, 0),
                                         (10, 3, 25, 2), (10, 3, 15, 1), (1, 1, 0, 0)])
def test_mask_parity(N, k, real, tp):
    rng = np.random.default_rng(N + real)
    m = rng.integers(-2, 50, (N, k)).astype(np.int64)
    t = dev(m)
    cnt = torch.tensor([real], dtype=torch.int32, device="cuda")
    moe.moe_mask_padding(t, N, k, cnt, tp)
    np.testing.assert_array_equal(t.cpu().numpy(), oracle.mask_padding(m, real, tp))


# ------------------------------------------------------------------ step 2
def gpu_create_indices(ids: np.ndarray, E: int) -> dict:
    S = ids.size
    order = torch.empty(max(S, 1), dtype=torch.int32, device="cuda")
    restore = torch.empty(max(S, 1), dtype=torch.int32, device="cuda")
    start = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    eids = torch.empty(E, dtype=torch.int32, device="cuda")
    stats = torch.empty(2, dtype=torch.int32, device="cuda")
    soff = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    ws_bytes = moe.moe_create_indices_workspace_bytes(S, E)
    ws = torch.full((ws_bytes,), 0x5A, dtype=torch.uint8, device="cuda")
    t = dev(ids.reshape(-1).astype(np.int64)) if S else torch.empty(1, dtype=torch.int64,
                                                                     device="cuda")
    moe.moe_create_indices(t, S, E, order, start, restore, eids, stats, soff, ws, ws_bytes)
    out = dict(token_expert_order=host_u32(order)[:S], expert_start_indices=host_u32(start),
               restore_token_order=host_u32(restore)[:S], expert_ids=eids.cpu().numpy(),
               expert_usage_stats=host_u32(stats), scales_offset=host_u32(soff))
    return out


@pytest.mark.parametrize("S,E,lo", [(0, 4, 0), (1, 1, 0), (32, 8, -1), (1000, 5, -2),
                                    (1024, 128, 0), (5120, 256, -1), (16384, 128, -1),
                                    (16385, 64, 0), (40000, 64, -1), (98304, 64, 0),
                                    (50000, 1024, -3), (200000, 7, -1)])
def test_create_indices_parity(S, E, lo):
    rng = np.random.default_rng(S * 7 + E)
    ids = rng.integers(lo, E + 2, S).astype(np.int64)
    check_indices(gpu_create_indices(ids, E), oracle.create_indices(ids, E), S)


def test_create_indices_deterministic_and_skewed():
    rng = np.random.default_rng(3)
    # heavy skew: one expert takes most slots (tiled path)
    ids = np.where(rng.random(60000) < 0.9, 5, rng.integers(0, 64, 60000)).astype(np.int64)
    ref = oracle.create_indices(ids, 64)
    for _ in range(5):
        check_indices(gpu_create_indices(ids, 64), ref, ids.size)


# ------------------------------------------------------------------ steps 1 + 2 fused
def gpu_mask_and_create_indices(m: np.ndarray, E: int, real: int, tp: int):
    N, k = m.shape
    S = N * k
    t = dev(m.astype(np.int64)) if S else torch.empty(1, dtype=torch.int64, device="cuda")
    cnt = torch.tensor([real], dtype=torch.int32, device="cuda")
    order = torch.full((max(S, 1),), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    restore = torch.full((max(S, 1),), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    start = torch.full((E + 1,), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    eids = torch.full((E,), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    stats = torch.full((2,), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    soff = torch.full((E + 1,), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    ws_bytes = moe.moe_create_indices_workspace_bytes(S, E)
    ws = torch.full((max(ws_bytes, 256),), 0x5A, dtype=torch.uint8, device="cuda")
    moe.moe_mask_and_create_indices(t, N, k, cnt, tp, E, order, start, restore, eids, stats,
                                    soff, ws, ws_bytes)
    out = dict(token_expert_order=host_u32(order)[:S], expert_start_indices=host_u32(start),
               restore_token_order=host_u32(restore)[:S], expert_ids=eids.cpu().numpy(),
               expert_usage_stats=host_u32(stats), scales_offset=host_u32(soff))
    return t.cpu().numpy()[:S].reshape(N, k) if S else m, out


@pytest.mark.parametrize("N,k,E,real,tp", [
    (128, 8, 128, 128, 0),      # decode-sized, nothing masked
    (128, 8, 128, 77, 0),       # ragged real count
    (13, 2, 8, 9, 1),           # tp_rank offset: rows 0.. of rank 1 start at 13
    (64, 16, 1024, 50, 0),      # E = 1024 (one expert per thread)
    (1024, 1, 3, 1000, 0),      # top_k = 1, S = 1024 exactly
    (37, 3, 12, -5, 0),         # real <= 0: everything masked
    (37, 3, 12, 4000, 0),       # real > N: nothing masked
    (1, 1, 1, 1, 0),            # minimal
    (129, 8, 64, 100, 0),       # S = 1032 > 1024: the two-call path
])
def test_mask_and_create_indices_equals_two_steps(N, k, E, real, tp):
    rng = np.random.default_rng(N * 31 + k + E)
    m = rng.integers(-2, E + 2, (N, k)).astype(np.int64)   # includes -1 and out-of-range ids
    masked_ref = oracle.mask_padding(m, real, tp)
    ref = oracle.create_indices(masked_ref.reshape(-1), E)
    masked_gpu, got = gpu_mask_and_create_indices(m, E, real, tp)
    np.testing.assert_array_equal(masked_gpu, masked_ref)
    check_indices(got, ref, N * k)
    # and byte for byte what the separate entry points give
    sep = gpu_create_indices(masked_ref, E)
    for key in sep:
        np.testing.assert_array_equal(got[key], sep[key], err_msg=key)


# ------------------------------------------------------------------ codecs (exhaustive)
def all_finite_bf16(shuffle_seed=None) -> np.ndarray:
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]          # drop Inf / NaN
    if shuffle_seed is not None:
        bits = np.random.default_rng(shuffle_seed).permutation(bits)
    n = -(-bits.size // 256) * 256
    out = np.zeros(n, np.uint16)
    out[: bits.size] = bits
    return out.reshape(-1, 256)


def gpu_mxfp4_rows(x_bits: np.ndarray) -> np.ndarray:
    N, K = x_bits.shape
    ids = np.zeros((N, 1), np.int64)                    # every token to expert 0, in order
    idx = gpu_tensors_indices(ids, 1)
    stride = moe.moe_mxfp4_row_stride(K)
    recv = torch.full((N, stride), 0xA5, dtype=torch.uint8, device="cuda")
    counts = torch.empty(1, dtype=torch.int32, device="cuda")
    moe.moe_dispatch_mxfp4(dev(x_bits), N, K, 1, 1, idx["restore"], idx["start"], idx["eids"],
                           idx["stats"], recv, N, counts)
    return recv.cpu().numpy()


def gpu_tensors_indices(ids: np.ndarray, E: int) -> dict:
    S = ids.size
    r = dict(order=torch.empty(S, dtype=torch.int32, device="cuda"),
             restore=torch.empty(S, dtype=torch.int32, device="cuda"),
             start=torch.empty(E + 1, dtype=torch.int32, device="cuda"),
             eids=torch.empty(E, dtype=torch.int32, device="cuda"),
             stats=torch.empty(2, dtype=torch.int32, device="cuda"))
    ws_bytes = moe.moe_create_indices_workspace_bytes(S, E)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    moe.moe_create_indices(dev(ids.reshape(-1)), S, E, r["order"], r["start"], r["restore"],
                           r["eids"], r["stats"], None, ws, ws_bytes)
    return r


@pytest.mark.parametrize("seed", [None, 1, 2])
def test_mxfp4_exhaustive_bf16(seed):
    x = all_finite_bf16(seed)
    np.testing.assert_array_equal(gpu_mxfp4_rows(x), oracle.mxfp4_encode_rows(x))


@pytest.mark.parametrize("K", [32, 96, 2048, 7168 + 32])
def test_mxfp4_rows_random_scales(K):
    rng = np.random.default_rng(K)
    x = (rng.standard_normal((37, K)) * np.exp(rng.uniform(-30, 30, (37, 1)))).astype(np.float32)
    x[0, :64] = 0.0
    x[1, :32] = -0.0
    xb = wl.f32_to_bf16_bits(x)
    np.testing.assert_array_equal(gpu_mxfp4_rows(xb), oracle.mxfp4_encode_rows(xb))


def gpu_nvfp4_act(x_bits: np.ndarray, g: float):
    M, K = x_bits.shape
    xq = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    sfa = torch.empty((M, K // 16), dtype=torch.uint8, device="cuda")
    moe.moe_quantize_activations_nvfp4(dev(x_bits), M, K, g, xq, sfa)
    return xq.cpu().numpy(), sfa.cpu().numpy()


@pytest.mark.parametrize("seed,g", [(None, 1.0), (1, 1.0), (2, 0.37), (None, 3.5e-3)])
def test_nvfp4_activation_exhaustive_bf16(seed, g):
    x = all_finite_bf16(seed)
    g = float(np.float32(g))
    q, s = gpu_nvfp4_act(x, g)
    rq, rs = oracle.nvfp4_quantize_bf16(x, g)
    np.testing.assert_array_equal(s, rs)
    np.testing.assert_array_equal(q, rq)


@pytest.mark.parametrize("M,K", [(5, 16), (33, 2880), (3, 4096 + 16)])
def test_nvfp4_activation_shapes(M, K):
    rng = np.random.default_rng(M * K)
    xb = wl.f32_to_bf16_bits((rng.standard_normal((M, K)) * 3).astype(np.float32))
    q, s = gpu_nvfp4_act(xb, 1.0)
    rq, rs = oracle.nvfp4_quantize_bf16(xb, 1.0)
    np.testing.assert_array_equal(s, rs)
    np.testing.assert_array_equal(q, rq)


@pytest.mark.parametrize("E,N,K", [(3, 32, 128), (2, 40, 2880), (4, 16, 4096)])
def test_quantize_weights_parity(E, N, K):
    rng = np.random.default_rng(E * N + K)
    w = (rng.standard_normal((E, N, K)) * 0.02).astype(np.float32)
    w[-1] = 0.0 if E > 2 else w[-1]
    wq = torch.empty((E, N, K // 2), dtype=torch.uint8, device="cuda")
    sfw = torch.empty((E, N, K // 16), dtype=torch.uint8, device="cuda")
    gw = torch.empty(E, dtype=torch.float32, device="cuda")
    moe.moe_quantize_weights_nvfp4(dev(w), E, N, K, wq, sfw, gw)
    rq, rs, rg = oracle.quantize_weights_nvfp4(w)
    np.testing.assert_array_equal(gw.cpu().numpy(), rg)
    np.testing.assert_array_equal(sfw.cpu().numpy(), rs)
    np.testing.assert_array_equal(wq.cpu().numpy(), rq)


# ------------------------------------------------------------------ step 3
@pytest.mark.parametrize("cfg", [wl.config("tiny"), wl.small_config(K=96, N=9, real=7, E=5, top_k=2),
                                 wl.config("decode_30b_a3b"),
                                 wl.small_config(N=300, real=290, K=7168, E=16, top_k=8)])
def test_dispatch_parity(cfg):
    x = wl.activations_bf16(cfg)
    ids = wl.routing(cfg)
    pipe = RoutingPipeline(cfg.N, cfg.K, cfg.E, cfg.top_k, 64, mode="w4a16")
    load_inputs(pipe, cfg, x, ids, wl.router_weights(cfg))
    pipe.recv_buf.fill_(0xA5)
    pipe.mask()
    pipe.create_indices()
    pipe.dispatch_mxfp4()
    ids_m = oracle.mask_padding(ids, cfg.real)
    ref_idx = oracle.create_indices(ids_m, cfg.E)
    check_indices(pipeline_indices(pipe), ref_idx, cfg.slots)
    ref_recv, ref_counts = oracle.dispatch_mxfp4(x, cfg.top_k, cfg.E, ref_idx, fill=0xA5)
    np.testing.assert_array_equal(pipe.recv_buf.cpu().numpy(), ref_recv)
    np.testing.assert_array_equal(host_u32(pipe.recv_counts), ref_counts)


def test_dispatch_capacity_overflow_is_reported():
    cfg = wl.config("tiny")
    x = wl.activations_bf16(cfg)
    pipe = RoutingPipeline(cfg.N, cfg.K, cfg.E, cfg.top_k, 64, recv_capacity=10)
    load_inputs(pipe, cfg, x, wl.routing(cfg), wl.router_weights(cfg))
    pipe.mask()
    pipe.create_indices()
    pipe.dispatch_mxfp4()
    assert moe.moe_get_device_error(clear=True) & moe.MOE_DEVERR_RECV_OVERFLOW
    ref_idx = oracle.create_indices(oracle.mask_padding(wl.routing(cfg), cfg.real), cfg.E)
    ref_recv, _ = oracle.dispatch_mxfp4(x, cfg.top_k, cfg.E, ref_idx)
    np.testing.assert_array_equal(pipe.recv_buf.cpu().numpy(), ref_recv[:10])


@pytest.mark.parametrize("cfg", [
    wl.config("tiny"),
    wl.small_config("dq_large_k", N=300, real=290, K=7168, E=16, top_k=8),
    wl.small_config("dq_ragged", N=64, real=50, K=2880, E=12, top_k=4, outlier_frac=0.01,
                    outlier_mult=20.0),
    wl.small_config("dq_k32", N=33, real=33, K=96, E=5, top_k=2),
])
def test_dispatch_quantize_fused_equals_separate(cfg):
    """Steps 3 and 4a from one read of x give byte for byte what the two
    separate calls give (MXFP4 rows and counts, NVFP4 codes and scales)."""
    x = wl.activations_bf16(cfg)
    pipe = RoutingPipeline(cfg.N, cfg.K, cfg.E, cfg.top_k, 64, mode="w4a4", act_global=0.375)
    load_inputs(pipe, cfg, x, wl.routing(cfg), wl.router_weights(cfg))
    pipe.mask()
    pipe.create_indices()
    pipe.recv_buf.fill_(0xA5)
    pipe.dispatch_mxfp4()
    pipe.quantize_activations()
    torch.cuda.synchronize()
    sep = [t.clone() for t in (pipe.recv_buf, pipe.recv_counts, pipe.xq, pipe.sfa)]
    for t in (pipe.recv_buf, pipe.xq, pipe.sfa):
        t.fill_(0xA5)
    pipe.recv_counts.fill_(-1)
    pipe.dispatch_quantize()
    torch.cuda.synchronize()
    for a, b, name in zip(sep, (pipe.recv_buf, pipe.recv_counts, pipe.xq, pipe.sfa),
                          ("recv_buf", "recv_counts", "xq", "sfa")):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), name
    # and the oracle's codes for every row
    xq, sfa = oracle.nvfp4_quantize_bf16(x, 0.375)
    np.testing.assert_array_equal(pipe.xq.cpu().numpy(), xq)
    np.testing.assert_array_equal(pipe.sfa.cpu().numpy(), sfa)


# ------------------------------------------------------------------ step 4b
SENTINEL = 0x4B1D      # bf16 bits of an unlikely finite value (~1.03e7)

GEMV_CASES = [
    ("tiny-w4a16", wl.config("tiny"), "w4a16"),
    ("tiny-w4a4", wl.config("tiny"), "w4a4"),
    # ragged row block (200 % 16 = 8), K % 256 != 0 (4-byte scale copies), 2 chunks
    ("ragged-w4a16", wl.small_config(), "w4a16"),
    ("ragged-w4a4", wl.small_config(), "w4a4"),
    # many tokens per expert: several 32-token passes and full 128-row rounds
    ("passes-w4a16", wl.small_config("passes", N=300, real=290, K=512, E=4, top_k=2,
                                     N_out=264), "w4a16"),
    ("passes-w4a4", wl.small_config("passes", N=300, real=290, K=512, E=4, top_k=2,
                                    N_out=264), "w4a4"),
    # 128-token passes of the tensor-memory variant with a ragged last chunk
    # (544 = 2 x 256 + 32) and gathered scale rows
    ("passes-ragged-k", wl.small_config("passes_rk", N=300, real=290, K=544, E=4, top_k=2,
                                        N_out=136), "w4a16"),
    # minimal K, N
    ("minimal", wl.small_config("minimal", N=3, real=3, K=64, E=2, top_k=1, N_out=8), "w4a16"),
    # K % 256 == 0 with a partial last stage of 1024 columns (2304 = 2 x 1024 + 256),
    # ragged row block, 8-token passes and two-group passes of the decode variant
    ("lines-w4a16", wl.small_config("lines", N=40, real=37, K=2304, E=5, top_k=2, N_out=200),
     "w4a16"),
    ("lines-w4a4", wl.small_config("lines", N=40, real=37, K=2304, E=5, top_k=2, N_out=200),
     "w4a4"),
    # decode-like: K = 2048 (two full stages), about 16 tokens per expert
    ("decode-like", wl.small_config("dlike", N=64, real=64, K=2048, E=16, top_k=4, N_out=136),
     "w4a16"),
    # K = 32 * odd (K % 64 == 32): 2-byte aligned scale rows, a partial last chunk
    ("k32odd-w4a16", wl.small_config("k32odd", N=30, real=28, K=224, E=5, top_k=2, N_out=72),
     "w4a16"),
    ("k32odd-w4a4", wl.small_config("k32odd", N=30, real=28, K=224, E=5, top_k=2, N_out=72),
     "w4a4"),
    # activations spanning many binades (per-chunk power-of-two scaling)
    ("wide-range", wl.small_config("wide", N=24, real=24, K=1024, E=6, top_k=2, N_out=128,
                                   outlier_frac=0.05, outlier_mult=3000.0), "w4a16"),
]


def run_gemv_case(cfg, mode, act_global=1.0):
    x = wl.activations_bf16(cfg)
    ids = wl.routing(cfg)
    pipe = RoutingPipeline(cfg.N, cfg.K, cfg.E, cfg.top_k, cfg.N_out, mode=mode,
                           act_global=act_global, dispatch=False)
    load_inputs(pipe, cfg, x, ids, wl.router_weights(cfg))
    quantize_all_weights(pipe, cfg)
    pipe.expert_out.view(torch.int16).fill_(SENTINEL)
    pipe.mask()
    pipe.create_indices()
    if mode == "w4a4":
        pipe.quantize_activations()
    pipe.gemv()
    torch.cuda.synchronize()
    return pipe, x, oracle.mask_padding(ids, cfg.real)


@pytest.fixture(params=["auto", "mma", "tc", "bs"])
def gemv_variant(request, monkeypatch):
    """Run a GEMV case through the host's choice and through each kernel variant
    (a variant that does not apply to the case -- the block-scaled one for
    W4A16, the decode one for K % 256 != 0 -- leaves the host's choice)."""
    if request.param != "auto":
        monkeypatch.setenv("MOE_GEMV_VARIANT", request.param)
    yield request.param


@pytest.mark.parametrize("name,cfg,mode", GEMV_CASES, ids=[c[0] for c in GEMV_CASES])
def test_gemv_parity(name, cfg, mode, gemv_variant):
    g_a = 1.0 if mode == "w4a16" else float(np.float32(0.5))
    pipe, x, ids = run_gemv_case(cfg, mode, g_a)
    wq, sfw, gw = oracle_weights(cfg, range(cfg.E))
    np.testing.assert_array_equal(pipe.wq.cpu().numpy(), wq)
    np.testing.assert_array_equal(pipe.sfw.cpu().numpy(), sfw)
    np.testing.assert_array_equal(pipe.w_global.cpu().numpy(), gw)
    if mode == "w4a16":
        ref = oracle.grouped_gemv("w4a16", ids, wq, sfw, gw, act_bf16=x)
    else:
        xq, sfa = oracle.nvfp4_quantize_bf16(x, g_a)
        np.testing.assert_array_equal(pipe.xq.cpu().numpy(), xq)
        np.testing.assert_array_equal(pipe.sfa.cpu().numpy(), sfa)
        ref = oracle.grouped_gemv("w4a4", ids, wq, sfw, gw, xq=xq, sfa=sfa, g_a=g_a)
    out_bits = host_bf16_bits(pipe.expert_out)
    routed = ~np.isnan(ref[..., 0])
    # unrouted slots are never written
    assert np.all(out_bits[~routed] == SENTINEL)
    assert_float_parity(host_bf16_f64(pipe.expert_out)[routed], ref[routed], what=name)


def test_gemv_token_major_equals_flattened_pairs(gemv_variant):
    cfg = wl.small_config("flat", N=50, real=44, K=320, E=7, top_k=4, N_out=136)
    pipe, x, ids = run_gemv_case(cfg, "w4a16")
    # same pairs as a [R, 1] map: one activation row per (token, slot)
    R_ids = ids.reshape(-1, 1)
    xr = np.repeat(x, cfg.top_k, axis=0)
    flat = RoutingPipeline(cfg.N * cfg.top_k, cfg.K, cfg.E, 1, cfg.N_out, dispatch=False)
    flat.x.copy_(dev(xr))
    flat.routing_map.copy_(dev(R_ids))
    flat.real_token_count.fill_(cfg.N * cfg.top_k)
    flat.wq.copy_(pipe.wq)
    flat.sfw.copy_(pipe.sfw)
    flat.w_global.copy_(pipe.w_global)
    flat.expert_out.view(torch.int16).fill_(SENTINEL)
    flat.create_indices()
    flat.gemv()
    np.testing.assert_array_equal(host_bf16_bits(flat.expert_out).reshape(-1),
                                  host_bf16_bits(pipe.expert_out).reshape(-1))


def bare_gemv(pipe, cfg, out, ws, stream=None):
    """The card's call shape: the routing map and a workspace, no grouping."""
    act = pipe.x if pipe.gemv_mode == moe.MOE_W4A16 else pipe.xq
    moe.moe_grouped_gemv_nvfp4(pipe.gemv_mode, act, pipe.sfa, pipe.act_global, pipe.routing_map,
                               cfg.N, cfg.top_k, pipe.wq, pipe.sfw, pipe.w_global, cfg.E,
                               cfg.N_out, cfg.K, out=out, workspace=ws, ws_bytes=ws.numel(),
                               stream=stream)


@pytest.mark.parametrize("mode", ["w4a16", "w4a4"])
def test_gemv_from_the_routing_map_alone(mode, gemv_variant):
    """indices [M, top_k] plus caller workspace and no step-2 grouping gives
    the same bits as the call that is handed the grouping."""
    cfg = wl.small_config("bare", N=50, real=44, K=512, E=7, top_k=4, N_out=136)
    pipe, x, ids = run_gemv_case(cfg, mode)
    ws = torch.full((moe.moe_grouped_gemv_workspace_bytes(cfg.N, cfg.top_k, cfg.E, cfg.K),), 0x5A,
                    dtype=torch.uint8, device="cuda")
    out = torch.empty_like(pipe.expert_out)
    out.view(torch.int16).fill_(SENTINEL)
    bare_gemv(pipe, cfg, out, ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bf16_bits(out), host_bf16_bits(pipe.expert_out))


IN_KERNEL_CASES = [
    ("tiny", wl.config("tiny"), None),
    ("decode_30b_a3b", wl.config("decode_30b_a3b"), None),
    # more passes than CTAs: a CTA's range spans several passes (token lists)
    ("many_passes", wl.small_config("many_passes", N=320, real=300, K=2048, E=256, top_k=8,
                                    N_out=64, seed=21), None),
    # one expert with many passes, through the decode variant
    ("skewed", wl.small_config("skewed", N=400, real=391, K=1024, E=64, top_k=4, N_out=48,
                               routing="zipf", zipf_s=1.6, seed=22), "mma"),
    # three stages per block, 8-token passes, ragged row block
    ("lines", wl.small_config("lines", N=40, real=37, K=2304, E=5, top_k=2, N_out=200), "mma"),
]


@pytest.mark.parametrize("name,cfg,variant", IN_KERNEL_CASES, ids=[c[0] for c in IN_KERNEL_CASES])
def test_gemv_groups_the_map_in_kernel(name, cfg, variant, monkeypatch):
    """Decode-sized W4A16 on the routing map alone: every CTA groups the map
    itself (stable, as moe_create_indices defines it), and the result equals,
    bit for bit, the same kernel handed the step-2 grouping -- with masked
    rows, -1 and out-of-range ids in the map."""
    if variant:
        monkeypatch.setenv("MOE_GEMV_VARIANT", variant)
    variant_id, in_kernel = moe.moe_grouped_gemv_plan(moe.MOE_W4A16, cfg.N, cfg.top_k, cfg.E,
                                                      cfg.N_out, cfg.K)
    assert variant_id == moe.MOE_GEMV_DECODE and in_kernel
    pipe, x, ids = run_gemv_case(cfg, "w4a16")
    m = pipe.routing_map.cpu().numpy()
    rng = np.random.default_rng(9)
    hit = rng.random(m.shape) < 0.03                  # ids that route nowhere
    m[hit] = np.where(rng.random(hit.sum()) < 0.5, -1, cfg.E + 5)
    pipe.routing_map.copy_(dev(m))
    pipe.create_indices()
    pipe.expert_out.view(torch.int16).fill_(SENTINEL)
    pipe.gemv()                                       # on the grouping
    torch.cuda.synchronize()
    ref = host_bf16_bits(pipe.expert_out)
    pipe.expert_out.view(torch.int16).fill_(SENTINEL)
    pipe.gemv_on_map()                                # on the map alone
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bf16_bits(pipe.expert_out), ref)
    wq, sfw, gw = oracle_weights(cfg, range(cfg.E))
    yref = oracle.grouped_gemv("w4a16", m, wq, sfw, gw, act_bf16=x)
    routed = ~np.isnan(yref[..., 0])
    assert np.all(ref[~routed] == SENTINEL)
    assert_float_parity(host_bf16_f64(pipe.expert_out)[routed], yref[routed], what=name)


def test_gemv_from_the_routing_map_follows_graph_replays():
    """The map is read on the device: a captured call follows new expert ids
    written between replays."""
    cfg = wl.small_config("bare_graph", N=40, real=40, K=256, E=6, top_k=2, N_out=64)
    pipe, x, _ = run_gemv_case(cfg, "w4a16")
    ws = torch.empty(moe.moe_grouped_gemv_workspace_bytes(cfg.N, cfg.top_k, cfg.E, cfg.K),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty_like(pipe.expert_out)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        bare_gemv(pipe, cfg, out, ws, s)              # warm-up outside capture
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            bare_gemv(pipe, cfg, out, ws, s)
    wq, sfw, gw = oracle_weights(cfg, range(cfg.E))
    rng = np.random.default_rng(5)
    for _ in range(3):
        ids = np.stack([rng.choice(cfg.E, cfg.top_k, replace=False) for _ in range(cfg.N)])
        ids[rng.random(ids.shape) < 0.1] = -1        # some slots route nowhere
        pipe.routing_map.copy_(dev(ids.astype(np.int64)))
        out.view(torch.int16).fill_(SENTINEL)
        g.replay()
        torch.cuda.synchronize()
        ref = oracle.grouped_gemv("w4a16", ids, wq, sfw, gw, act_bf16=x)
        routed = ~np.isnan(ref[..., 0])
        assert np.all(host_bf16_bits(out)[~routed] == SENTINEL)
        assert_float_parity(host_bf16_f64(out)[routed], ref[routed], what="graph replay")


@pytest.mark.parametrize("variant", ["auto", "tc"])
@pytest.mark.parametrize("path", ["grouping", "map"])
def test_gemv_w4a16_full_bf16_range(path, variant, monkeypatch):
    """W4A16 over bf16's whole range, in the decode variant (the plan's
    choice here) and the tensor-memory variant (its activations converted
    once into the workspace): tokens scaled by 2^-100 .. 2^115 (about 1e-30
    .. 4e34) and an outlier beyond fp16's largest value in an ordinary token.
    Each token's outputs, divided by its power of two, meet the stated
    tolerance against the oracle (the absolute floor alone would let tiny
    tokens pass trivially), and no range error is raised."""
    if variant != "auto":
        monkeypatch.setenv("MOE_GEMV_VARIANT", variant)
    cfg = wl.small_config("range_full", N=32, real=32, K=1024, E=4, top_k=2, N_out=64, seed=41)
    got, _ = moe.moe_grouped_gemv_plan(moe.MOE_W4A16, cfg.N, cfg.top_k, cfg.E, cfg.N_out, cfg.K,
                                       grouping_given=(path == "grouping"))
    assert got == (moe.MOE_GEMV_DECODE if variant == "auto" else moe.MOE_GEMV_TENSOR_MEMORY)
    xf = wl.bf16_bits_to_f32(wl.activations_bf16(cfg)).astype(np.float64)
    exps = np.linspace(-100, 115, cfg.N).round().astype(int)
    exps[3] = 0
    x = xf * np.exp2(exps)[:, None]
    x[3, 7] = 1.0e5                                   # beyond fp16 in an ordinary token
    xb = wl.f32_to_bf16_bits(x.astype(np.float32))
    ids = wl.routing(cfg)
    pipe = RoutingPipeline(cfg.N, cfg.K, cfg.E, cfg.top_k, cfg.N_out, dispatch=False)
    load_inputs(pipe, cfg, xb, ids, wl.router_weights(cfg))
    quantize_all_weights(pipe, cfg)
    moe.moe_get_device_error(clear=True)
    pipe.mask()
    pipe.create_indices()
    pipe.expert_out.view(torch.int16).fill_(SENTINEL)
    if path == "grouping":
        pipe.gemv()
    else:
        pipe.gemv_on_map()
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(clear=True) == 0
    wq, sfw, gw = oracle_weights(cfg, range(cfg.E))
    ref = oracle.grouped_gemv("w4a16", oracle.mask_padding(ids, cfg.real), wq, sfw, gw,
                              act_bf16=xb)
    got = host_bf16_f64(pipe.expert_out)
    scale = np.exp2(exps.astype(np.float64))[:, None, None]
    assert np.all(np.isfinite(got))
    assert_float_parity(got / scale, ref / scale, what="full bf16 range (per-token scaled)")


def test_gemv_activation_range_is_reported(monkeypatch):
    """Called with the grouping and no workspace, the tensor-memory variant
    converts W4A16 activations chunk by chunk without per-token offsets: a
    value beyond fp16's range is reported."""
    monkeypatch.setenv("MOE_GEMV_VARIANT", "tc")
    cfg = wl.small_config("range", N=4, real=4, K=128, E=2, top_k=1, N_out=16)
    x = wl.activations_bf16(cfg)
    x[1, 5] = wl.f32_to_bf16_bits(np.array([1.0e5], np.float32))[0]   # beyond fp16 range
    pipe = RoutingPipeline(cfg.N, cfg.K, cfg.E, cfg.top_k, cfg.N_out, dispatch=False)
    load_inputs(pipe, cfg, x, wl.routing(cfg), wl.router_weights(cfg))
    quantize_all_weights(pipe, cfg)
    assert moe.moe_get_device_error(clear=True) == 0
    pipe.mask()
    pipe.create_indices()
    moe.moe_grouped_gemv_nvfp4(moe.MOE_W4A16, pipe.x, None, 1.0, pipe.routing_map, cfg.N,
                               cfg.top_k, pipe.wq, pipe.sfw, pipe.w_global, cfg.E, cfg.N_out, cfg.K,
                               pipe.token_expert_order, pipe.expert_start_indices,
                               pipe.expert_ids, pipe.expert_usage_stats, pipe.expert_out)
    assert moe.moe_get_device_error(clear=True) & moe.MOE_DEVERR_ACT_RANGE


def test_gemv_all_slots_unrouted():
    cfg = wl.small_config("empty", N=8, real=0, K=128, E=4, top_k=2, N_out=32)
    pipe, x, ids = run_gemv_case(cfg, "w4a16")
    assert np.all(host_bf16_bits(pipe.expert_out) == SENTINEL)
    assert host_u32(pipe.expert_usage_stats).tolist() == [0, 0]


# ------------------------------------------------------------------ step 5
@pytest.mark.parametrize("epi,alpha", [("none", 1.0), ("identity", 1.0), ("scale", -0.625)])
@pytest.mark.parametrize("cfg", [wl.small_config(N=20, real=17, top_k=4, N_out=72, E=6),
                                 wl.small_config("wide", N=33, real=33, top_k=8, N_out=1000, E=9)])
def test_combine_parity(cfg, epi, alpha):
    y = wl.expert_outputs_bf16(cfg)
    w = wl.router_weights(cfg)
    ids = oracle.mask_padding(wl.routing(cfg), cfg.real)
    ids[0, 0] = cfg.E + 3                                   # out of range: routes nowhere
    out = torch.empty((cfg.N, cfg.N_out), dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(dev(y), dev(w), dev(ids), cfg.N, cfg.top_k, cfg.N_out, cfg.E,
                    {"none": 0, "identity": 1, "scale": 2}[epi], alpha, out)
    ref = oracle.combine(y, w, ids, cfg.E, epi, alpha)
    assert_float_parity(host_bf16_f64(out), ref, what=f"combine {epi}")
    assert np.all(host_bf16_f64(out)[cfg.real:] == 0.0)


def test_combine_one_hot_is_exact():
    cfg = wl.small_config(N=8, real=8, top_k=3, N_out=64, E=4)
    y = wl.expert_outputs_bf16(cfg)
    ids = np.tile(np.arange(3), (8, 1)).astype(np.int64)
    w = np.zeros((8, 3), np.float32)
    sel = np.random.default_rng(2).integers(0, 3, 8)
    w[np.arange(8), sel] = 1.0
    out = torch.empty((8, 64), dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(dev(y), dev(w), dev(ids), 8, 3, 64, cfg.E, 0, 1.0, out)
    np.testing.assert_array_equal(host_bf16_bits(out), y[np.arange(8), sel])


def test_combine_into_pinned_host_memory():
    """output_tokens may be pinned host memory: same bytes as a device buffer."""
    cfg = wl.config("decode_30b_a3b")
    y, w = dev(wl.expert_outputs_bf16(cfg)), dev(wl.router_weights(cfg))
    ids = dev(wl.routing(cfg))
    out_dev = torch.empty((cfg.N, cfg.N_out), dtype=torch.bfloat16, device="cuda")
    out_host = torch.full((cfg.N, cfg.N_out), 7.0, dtype=torch.bfloat16).pin_memory()
    moe.moe_combine(y, w, ids, cfg.N, cfg.top_k, cfg.N_out, cfg.E, 1, 1.0, out_dev)
    moe.moe_combine(y, w, ids, cfg.N, cfg.top_k, cfg.N_out, cfg.E, 1, 1.0, out_host)
    torch.cuda.synchronize()
    assert torch.equal(out_host.view(torch.int16), out_dev.cpu().view(torch.int16))


# ------------------------------------------------------------------ boundary
def test_invalid_arguments_launch_nothing():
    with pytest.raises(moe.MoeError) as e:
        moe.moe_grouped_gemv_nvfp4(0, 16, 0, 1.0, 16, 4, 2, 16, 16, 0, 4, 12, 64, 16, 16, 16, 16,
                                   16)
    assert e.value.status == 1
    with pytest.raises(moe.MoeError) as e:
        moe.moe_create_indices(16, 8, 4, 16, 16, 16, 16, 16, None, None, 0)
    assert e.value.status == 3
