"""Pins for the oracle's grouped NVFP4 GEMV and combine.

References: a dense float64 numpy matmul over weights decoded with
ml_dtypes (an independent decoder), one-hot inputs that reproduce single
elements exactly, W4A4 == W4A16 on activations that already sit on the NVFP4
grid, and the token-major identity "M = routed pairs, top_k = 1".
"""
import ml_dtypes
import numpy as np
import pytest

import oracle
import workloads as wl

F4 = ml_dtypes.float4_e2m1fn
F8 = ml_dtypes.float8_e4m3fn


def lib_decode(q, sf):
    K = q.shape[-1] * 2
    codes = np.empty(q.shape[:-1] + (K,), np.uint8)
    codes[..., 0::2] = q & 0xF
    codes[..., 1::2] = q >> 4
    return codes.view(F4).astype(np.float64) * np.repeat(sf.view(F8).astype(np.float64), 16, -1)


def make_problem(cfg):
    x = wl.activations_bf16(cfg)
    ids = oracle.mask_padding(wl.routing(cfg), cfg.real)
    w = wl.all_expert_weights_f32(cfg)
    wq, sfw, gw = oracle.quantize_weights_nvfp4(w)
    return x, ids, wq, sfw, gw


def dense_reference(a, ids, wq, sfw, gw, E):
    W = lib_decode(wq, sfw) * gw[:, None, None].astype(np.float64)   # [E, N, K]
    M, k = ids.shape
    y = np.full((M, k, wq.shape[1]), np.nan)
    for m in range(M):
        for j in range(k):
            e = ids[m, j]
            if 0 <= e < E:
                y[m, j] = W[e] @ a[m]
    return y


@pytest.mark.parametrize("cfg", [wl.config("tiny"), wl.small_config()])
def test_gemv_w4a16_matches_dense_matmul(cfg):
    x, ids, wq, sfw, gw = make_problem(cfg)
    y = oracle.grouped_gemv("w4a16", ids, wq, sfw, gw, act_bf16=x)
    ref = dense_reference(wl.bf16_bits_to_f32(x).astype(np.float64), ids, wq, sfw, gw, cfg.E)
    np.testing.assert_array_equal(np.isnan(y), np.isnan(ref))
    np.testing.assert_allclose(y[~np.isnan(y)], ref[~np.isnan(ref)], rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("cfg", [wl.config("tiny"), wl.small_config()])
def test_gemv_w4a4_matches_dense_matmul(cfg):
    x, ids, wq, sfw, gw = make_problem(cfg)
    ga = float(np.float32(0.37))   # the GEMV takes g_a as fp32
    xq, sfa = oracle.nvfp4_quantize_bf16(x, ga)
    y = oracle.grouped_gemv("w4a4", ids, wq, sfw, gw, xq=xq, sfa=sfa, g_a=ga)
    ref = dense_reference(lib_decode(xq, sfa) * ga, ids, wq, sfw, gw, cfg.E)
    np.testing.assert_allclose(y[~np.isnan(y)], ref[~np.isnan(ref)], rtol=1e-12, atol=1e-15)


def test_gemv_one_hot_weights_reproduce_activation_elements():
    cfg = wl.small_config(N=5, real=5, K=64, E=2, top_k=1, N_out=16)
    x = wl.activations_bf16(cfg)
    ids = np.array([[0], [1], [0], [-1], [1]])
    w = np.zeros((2, 16, 64), np.float32)
    cols = np.random.default_rng(0).integers(0, 64, (2, 16))
    for e in range(2):
        w[e, np.arange(16), cols[e]] = 6.0 * 448.0      # one nonzero per row, g_w = 1
    wq, sfw, gw = oracle.quantize_weights_nvfp4(w)
    assert np.all(gw == 1.0)
    y = oracle.grouped_gemv("w4a16", ids, wq, sfw, gw, act_bf16=x)
    xf = wl.bf16_bits_to_f32(x).astype(np.float64)
    for m in range(5):
        e = ids[m, 0]
        if e < 0:
            assert np.all(np.isnan(y[m, 0]))
        else:
            np.testing.assert_array_equal(y[m, 0], 2688.0 * xf[m, cols[e]])


def test_gemv_w4a4_equals_w4a16_on_grid_activations():
    cfg = wl.small_config(N=12, real=10, K=128, E=4, top_k=2, N_out=48)
    x, ids, wq, sfw, gw = make_problem(cfg)
    xq, sfa = oracle.nvfp4_quantize_bf16(x, 1.0)
    x_grid = wl.f32_to_bf16_bits(lib_decode(xq, sfa).astype(np.float32))
    assert np.array_equal(wl.bf16_bits_to_f32(x_grid).astype(np.float64), lib_decode(xq, sfa))
    a = oracle.grouped_gemv("w4a16", ids, wq, sfw, gw, act_bf16=x_grid)
    b = oracle.grouped_gemv("w4a4", ids, wq, sfw, gw, xq=xq, sfa=sfa)
    np.testing.assert_array_equal(a, b)


def test_gemv_token_major_equals_flattened_pairs():
    cfg = wl.small_config(N=9, real=9, K=96, E=5, top_k=3, N_out=40)
    x, ids, wq, sfw, gw = make_problem(cfg)
    y = oracle.grouped_gemv("w4a16", ids, wq, sfw, gw, act_bf16=x)
    xr = np.repeat(x, cfg.top_k, axis=0)               # M = routed pairs, one activation each
    y1 = oracle.grouped_gemv("w4a16", ids.reshape(-1, 1), wq, sfw, gw, act_bf16=xr)
    np.testing.assert_array_equal(y.reshape(-1, 1, cfg.N_out), y1)


def test_gemv_elements_match_full():
    cfg = wl.small_config()
    x, ids, wq, sfw, gw = make_problem(cfg)
    y = oracle.grouped_gemv("w4a16", ids, wq, sfw, gw, act_bf16=x)
    rng = np.random.default_rng(1)
    samples = [(int(rng.integers(cfg.N)), int(rng.integers(cfg.top_k)), int(rng.integers(cfg.N_out)))
               for _ in range(50)]
    s = oracle.gemv_elements("w4a16", ids, wq, sfw, gw, samples, act_bf16=x)
    ref = np.array([y[m, j, n] for m, j, n in samples])
    np.testing.assert_array_equal(s, ref)


# ------------------------------------------------------------------ combine
def test_combine_matches_einsum():
    cfg = wl.small_config(N=20, real=17, top_k=4, N_out=72, E=6)
    y = wl.expert_outputs_bf16(cfg)
    w = wl.router_weights(cfg)
    ids = oracle.mask_padding(wl.routing(cfg), cfg.real)
    ids[0, 1] = 99                                   # out-of-range id routes nowhere
    valid = ((ids >= 0) & (ids < cfg.E)).astype(np.float64)
    yf = wl.bf16_bits_to_f32(y).astype(np.float64)
    ref = np.einsum("tj,tjh->th", w.astype(np.float64) * valid, yf)
    for epi, alpha, f in (("none", 1.0, 1.0), ("identity", 1.0, 1.0), ("scale", -0.75, -0.75)):
        out = oracle.combine(y, w, ids, cfg.E, epi, alpha)
        np.testing.assert_allclose(out, f * ref, rtol=1e-13, atol=1e-300)
    assert np.all(oracle.combine(y, w, ids, cfg.E)[cfg.real:] == 0)   # epi(0) on empty rows


def test_combine_one_hot_and_equal_rows():
    cfg = wl.small_config(N=8, real=8, top_k=3, N_out=32, E=4)
    y = wl.expert_outputs_bf16(cfg)
    ids = np.tile(np.arange(3), (8, 1))
    w = np.zeros((8, 3), np.float32)
    sel = np.random.default_rng(2).integers(0, 3, 8)
    w[np.arange(8), sel] = 1.0
    out = oracle.combine(y, w, ids, cfg.E)
    np.testing.assert_array_equal(out, wl.bf16_bits_to_f32(y[np.arange(8), sel]))
    yeq = np.repeat(y[:, :1], 3, axis=1)
    weq = np.full((8, 3), np.float32(0.25))
    weq[:, 2] = 0.5
    np.testing.assert_array_equal(oracle.combine(yeq, weq, ids, cfg.E),
                                  wl.bf16_bits_to_f32(y[:, 0]))
