"""Pins for the oracle's FP4 / FP8 codecs (E2M1, E4M3, E8M0, MXFP4 rows, NVFP4 blocks).

Independent references: ml_dtypes' float4_e2m1fn / float8_e4m3fn casts
(round-to-nearest-even, saturating E2M1; E4M3 needs clamping to +-448 first
because ml_dtypes overflows to NaN), closed-form properties of the MX and
NVFP4 block scales, and exact round trips of on-grid values.
"""
import ml_dtypes
import numpy as np
import pytest

import oracle
from workloads import bf16_bits_to_f32, f32_to_bf16_bits

F4 = ml_dtypes.float4_e2m1fn
F8 = ml_dtypes.float8_e4m3fn


def lib_e2m1_code(v):
    return int(np.array([v], np.float32).astype(F4).view(np.uint8)[0]) & 0xF


def lib_e2m1_value(code):
    return float(np.array([code], np.uint8).view(F4).astype(np.float64)[0])


def lib_e4m3_code(v):
    v = np.clip(np.float32(v), -448.0, 448.0)
    return int(np.array([v], np.float32).astype(F8).view(np.uint8)[0])


def lib_e4m3_value(code):
    return float(np.array([code], np.uint8).view(F8).astype(np.float64)[0])


# ------------------------------------------------------------------ E2M1
def test_e2m1_values_match_library():
    for c in range(16):
        assert oracle.e2m1_value(c) == lib_e2m1_value(c), c
    mags = [oracle.e2m1_value(c) for c in range(8)]
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_encode_ties_and_saturation():
    # values on the decision boundaries: ties go to the even code
    expect = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6,
              6.0: 7, 7.0: 7, 1e30: 7, 0.2499999: 0, 0.2500001: 1}
    for v, c in expect.items():
        assert oracle.e2m1_encode(v) == c, v
        assert oracle.e2m1_encode(-v) == c | 8, -v
    assert oracle.e2m1_encode(0.0) == 0
    assert oracle.e2m1_encode(-0.0) == 8
    assert oracle.e2m1_encode(-0.1) == 8


def test_e2m1_encode_matches_library_dense_sweep():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        np.arange(-8 * 256, 8 * 256 + 1) / 256.0,          # fine grid incl. all ties
        rng.uniform(-10, 10, 4000),
        rng.standard_normal(2000) * 1e-3,
    ]).astype(np.float32)
    lib = vals.astype(F4).view(np.uint8) & 0xF
    ours = np.array([oracle.e2m1_encode(float(v)) for v in vals], np.uint8)
    np.testing.assert_array_equal(ours, lib)


# ------------------------------------------------------------------ E4M3
def test_e4m3_values_match_library():
    for c in range(256):
        a, b = oracle.e4m3_value(c), lib_e4m3_value(c)
        if np.isnan(b):
            assert np.isnan(a), c
        else:
            assert a == b, c
    assert oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0x01) == 2.0 ** -9


def test_e4m3_encode_matches_library_sweep():
    rng = np.random.default_rng(1)
    # every representable value, every midpoint between neighbours, random values
    reps = np.array([oracle.e4m3_value(c) for c in range(127)])
    mids = (reps[:-1] + reps[1:]) / 2
    vals = np.concatenate([reps, mids, rng.uniform(0, 500, 3000),
                           np.exp(rng.uniform(np.log(1e-5), np.log(600), 3000))]).astype(np.float32)
    ours = np.array([oracle.e4m3_encode(float(v)) for v in vals])
    lib = np.array([lib_e4m3_code(float(v)) for v in vals])
    np.testing.assert_array_equal(ours, lib)
    assert oracle.e4m3_encode(1e9) == 0x7E        # saturates to 448, never NaN


# ------------------------------------------------------------------ MXFP4
def decode_mxfp4_row(row, K):
    codes = np.empty(K, np.uint8)
    codes[0::2] = row[: K // 2] & 0xF
    codes[1::2] = row[: K // 2] >> 4
    vals = codes.view(F4).astype(np.float64)
    se = row[K // 2: K // 2 + K // 32].astype(np.int64) - 127
    return vals, se


@pytest.mark.parametrize("K", [32, 96, 256, 2048])
def test_mxfp4_row_properties(K):
    rng = np.random.default_rng(K)
    x = f32_to_bf16_bits(rng.standard_normal((6, K)).astype(np.float32) * np.float32(3.0))
    x[1, :32] = 0                                  # an all-zero block
    x[2, :32] = 0x8000                             # all negative zeros
    rows = oracle.mxfp4_encode_rows(x)
    stride = oracle.mxfp4_row_stride(K)
    assert rows.shape == (6, stride) and stride % 16 == 0
    assert stride == -(-(K // 2 + K // 32) // 16) * 16
    xf = bf16_bits_to_f32(x).astype(np.float64)
    for r in range(6):
        vals, se = decode_mxfp4_row(rows[r], K)
        assert np.all(rows[r, K // 2 + K // 32:] == 0)     # zero padding
        for b in range(K // 32):
            blk = xf[r, b * 32:(b + 1) * 32]
            amax = np.abs(blk).max()
            if amax == 0:
                assert se[b] == -127
                codes = np.concatenate([[c & 0xF, c >> 4] for c in rows[r, b * 16:(b + 1) * 16]])
                np.testing.assert_array_equal(codes, np.where(np.signbit(blk), 8, 0))
                continue
            # closed form: the shared scale is the largest power of two <= amax / 4
            assert 4.0 * 2.0 ** se[b] <= amax < 8.0 * 2.0 ** se[b]
            # element codes are the library's RNE of x / 2^se
            q = (blk / 2.0 ** se[b]).astype(np.float32).astype(F4).astype(np.float64)
            np.testing.assert_array_equal(vals[b * 32:(b + 1) * 32], q)
            # reconstruction: half a grid step inside [0, 6X]; values in (6X, 8X) clip to 6X
            X = 2.0 ** se[b]
            a = np.abs(blk) / X
            step = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
            bound = np.where(a <= 6, 0.5 * step * X, np.abs(blk) - 6 * X)
            err = np.abs(vals[b * 32:(b + 1) * 32] * X - blk)
            assert np.all(err <= bound)


def test_mxfp4_grid_roundtrip_and_nibble_order():
    K = 64
    rng = np.random.default_rng(3)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    se = np.array([-3, 5])
    vals = grid[rng.integers(0, 8, K)] * np.where(rng.random(K) < 0.5, -1, 1)
    vals[0], vals[32] = 6.0, -4.0        # block maxima at 6 and 4 times the scale
    x = vals * np.repeat(2.0 ** se, 32)
    xb = f32_to_bf16_bits(x.astype(np.float32))
    assert np.array_equal(bf16_bits_to_f32(xb), x.astype(np.float32))
    row = oracle.mxfp4_encode_rows(xb[None])[0]
    dec, se_out = decode_mxfp4_row(row, K)
    np.testing.assert_array_equal(se_out, se)
    np.testing.assert_array_equal(dec * np.repeat(2.0 ** se_out, 32), x)
    # element 0 (6.0 -> code 7) sits in the low nibble of byte 0
    assert row[0] & 0xF == 7


def test_mxfp4_extreme_exponents():
    # smallest bf16 subnormal block and the largest finite bf16
    x = np.zeros((2, 32), np.uint16)
    x[0, 0] = 0x0001                 # 2^-133
    x[1, 0] = 0x7F7F                 # ~3.39e38
    rows = oracle.mxfp4_encode_rows(x)
    assert rows[0, 16] == 0          # exponent clamped to -127
    assert rows[0, 0] & 0xF == 0     # 2^-133 / 2^-127 = 1/64 rounds to zero
    assert rows[1, 16] == 127 + 125  # floor(log2) = 127
    assert rows[1, 0] & 0xF == lib_e2m1_code(float(bf16_bits_to_f32(x[1, :1])[0] / 2.0 ** 125))


# ------------------------------------------------------------------ NVFP4
def decode_nvfp4(q, sf, K):
    codes = np.empty(q.shape[:-1] + (K,), np.uint8)
    codes[..., 0::2] = q & 0xF
    codes[..., 1::2] = q >> 4
    v = codes.view(F4).astype(np.float64)
    s = sf.view(F8).astype(np.float64)
    return v * np.repeat(s, 16, axis=-1)


def test_nvfp4_grid_roundtrip_exact():
    rng = np.random.default_rng(4)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    K = 64
    scales = np.array([lib_e4m3_value(c) for c in (0x08, 0x31, 0x52, 0x7E)])  # 2^-6 .. 448
    vals = grid[rng.integers(0, 8, (3, K))] * np.where(rng.random((3, K)) < .5, -1, 1)
    vals[:, ::16] = 6.0                       # every block reaches 6 * scale
    x = vals * np.repeat(scales, 16)[None]
    q, sf = oracle.nvfp4_quantize(x.astype(np.float32), 1.0)
    np.testing.assert_array_equal(sf.view(F8).astype(np.float64), np.tile(scales, (3, 1)))
    np.testing.assert_array_equal(decode_nvfp4(q, sf, K), x)


def test_nvfp4_scale_and_error_bounds():
    rng = np.random.default_rng(5)
    K = 256
    x = (rng.standard_normal((16, K)) * np.exp(rng.uniform(-8, 3, (16, 1)))).astype(np.float32)
    x[0, :16] = 0.0
    x[0, 16:32] = -0.0
    for g in (1.0, 0.0173):
        q, sf = oracle.nvfp4_quantize(x, g)
        s = sf.view(F8).astype(np.float64)
        blocks = x.reshape(16, K // 16, 16).astype(np.float64)
        amax = np.abs(blocks).max(-1)
        # the block scale is the library's E4M3 rounding of fl32(fl32(amax/6)/g)
        t = (amax.astype(np.float32) / np.float32(6)).astype(np.float32) / np.float32(g)
        lib_sc = np.array([[lib_e4m3_code(float(v)) for v in row] for row in t])
        np.testing.assert_array_equal(sf, lib_sc)
        dec = decode_nvfp4(q, sf, K).reshape(blocks.shape) * g
        sdec = (s * g)[..., None]
        nz = (sdec > 0)[..., 0]
        # element codes: library RNE of the fp32 quotient x / sdec
        sdec32 = (s.astype(np.float32) * np.float32(g))[..., None]
        quot = np.where(sdec32 > 0, blocks.astype(np.float32) / np.where(sdec32 > 0, sdec32, 1),
                        0).astype(np.float32)
        codes = np.empty(q.shape[:-1] + (K,), np.uint8)
        codes[..., 0::2] = q & 0xF
        codes[..., 1::2] = q >> 4
        codes = codes.reshape(blocks.shape)
        libc = (quot.astype(F4).view(np.uint8) & 0xF).reshape(blocks.shape)
        libc = np.where(nz[..., None], libc, np.where(np.signbit(blocks), 8, 0))
        np.testing.assert_array_equal(codes, libc)
        # error: at most half a grid step inside the range, bounded saturation above it
        err = np.abs(dec - blocks)
        step = np.where(np.abs(blocks) / np.where(sdec > 0, sdec, 1) >= 4, 2,
                        np.where(np.abs(blocks) / np.where(sdec > 0, sdec, 1) >= 2, 1, 0.5))
        bound = np.where(np.abs(blocks) <= 6 * sdec, 0.5 * step * sdec * (1 + 1e-6),
                         np.abs(blocks) - 6 * sdec + 1e-12)
        assert np.all(err[nz] <= bound[nz] + 1e-30)
        # all-zero blocks: zero scale and signed-zero codes
        assert sf[0, 0] == 0 and sf[0, 1] == 0
        assert np.all(codes[0, 0] == 0) and np.all(codes[0, 1] == 8)


def test_nvfp4_weight_global_uses_full_e4m3_range():
    rng = np.random.default_rng(6)
    w = (rng.standard_normal((3, 32, 128)) * 0.02).astype(np.float32)
    w[2] = 0
    wq, sfw, gw = oracle.quantize_weights_nvfp4(w)
    for e in range(2):
        amax = np.float32(np.abs(w[e]).max())
        assert gw[e] == np.float32(amax / np.float32(2688.0))
        # the block holding amax gets a scale at (or one step below) 448
        assert sfw[e].max() in (0x7E, 0x7D)
    assert gw[2] == 1.0 and np.all(sfw[2] == 0) and np.all(wq[2] == 0)


def test_nvfp4_bf16_entry_matches_f32_entry():
    rng = np.random.default_rng(7)
    xb = f32_to_bf16_bits(rng.standard_normal((5, 96)).astype(np.float32) * 4)
    a = oracle.nvfp4_quantize_bf16(xb, 0.5)
    b = oracle.nvfp4_quantize(bf16_bits_to_f32(xb), 0.5)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
