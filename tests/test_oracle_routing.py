"""Pins for the oracle's mask, create_indices and MXFP4 dispatch steps.

References: numpy slice assignment (mask), numpy's stable argsort, bincount
and cumsum (grouping, CSR offsets), permutation inversion, brute force on
tiny inputs, and the MXFP4 row encoder composed with the grouping (dispatch).
"""
import itertools

import numpy as np
import pytest

import oracle
import workloads as wl


# ------------------------------------------------------------------ mask
@pytest.mark.parametrize("N,k,real,tp", [(16, 2, 13, 0), (16, 2, 0, 0), (16, 2, -5, 0),
                                         (16, 2, 16, 0), (16, 2, 99, 0), (10, 3, 25, 2),
                                         (10, 3, 15, 1), (7, 8, 3, 0)])
def test_mask_matches_slice_assignment(N, k, real, tp):
    rng = np.random.default_rng(N * 100 + real)
    m = rng.integers(-3, 50, (N, k))
    ref = m.copy()
    first = min(max(real - tp * N, 0), N)    # first local row whose global row >= real
    ref[first:, :] = -1
    np.testing.assert_array_equal(oracle.mask_padding(m, real, tp), ref)


# ------------------------------------------------------------------ create_indices
def library_grouping(ids, E):
    ids = np.asarray(ids).reshape(-1)
    valid = (ids >= 0) & (ids < E)
    p = np.nonzero(valid)[0]
    order = p[np.argsort(ids[valid], kind="stable")]
    cnt = np.bincount(ids[valid], minlength=E)
    active = np.nonzero(cnt)[0]
    start = np.concatenate([[0], np.cumsum(cnt[active])])
    return order, cnt, active, start


def check_grouping(ids, E, out):
    ids = np.asarray(ids).reshape(-1)
    S = ids.size
    order, cnt, active, start = library_grouping(ids, E)
    R, A = order.size, active.size
    assert out["expert_usage_stats"].tolist() == [int(cnt.max()) if S else 0, A]
    np.testing.assert_array_equal(out["token_expert_order"][:R], order)
    assert np.all(out["token_expert_order"][R:] == 0xFFFFFFFF)
    np.testing.assert_array_equal(out["expert_ids"][:A], active)
    assert np.all(out["expert_ids"][A:] == -1)
    np.testing.assert_array_equal(out["expert_start_indices"][:A + 1], start)
    assert np.all(out["expert_start_indices"][A + 1:] == R)
    # restore is the inverse permutation on routed pairs
    rest = out["restore_token_order"]
    np.testing.assert_array_equal(rest[order], np.arange(R))
    invalid = np.setdiff1d(np.arange(S), order)
    assert np.all(rest[invalid] == 0xFFFFFFFF)
    # contiguous, ascending-id groups
    grp = ids[out["token_expert_order"][:R].astype(np.int64)]
    assert np.all(np.diff(grp) >= 0)
    # scales_offset: 128-aligned, each active expert gets its count rounded up
    so = out["scales_offset"].astype(np.int64)
    assert np.all(so % 128 == 0) and so[0] == 0
    np.testing.assert_array_equal(np.diff(so[:A + 1]), -(-cnt[active] // 128) * 128)
    assert np.all(so[:A + 1] >= start) and np.all(so[A + 1:] == so[A])


@pytest.mark.parametrize("S,E,lo", [(0, 4, 0), (1, 1, 0), (32, 8, -1), (257, 5, -2),
                                    (1024, 128, 0), (5000, 256, -1), (3000, 1024, -4)])
def test_create_indices_matches_library(S, E, lo):
    rng = np.random.default_rng(S + E)
    ids = rng.integers(lo, E + 2, S)
    check_grouping(ids, E, oracle.create_indices(ids, E))


def test_create_indices_brute_force_tiny():
    # every routing map of 4 slots over ids {-1, 0, 1, 2} with E = 3
    for ids in itertools.product([-1, 0, 1, 2], repeat=4):
        ids = np.array(ids)
        out = oracle.create_indices(ids, 3)
        pos = 0
        for e in range(3):
            for p in range(4):
                if ids[p] == e:
                    assert out["token_expert_order"][pos] == p
                    assert out["restore_token_order"][p] == pos
                    pos += 1


def test_masked_rows_route_nowhere():
    for name in ("tiny", "decode_large_expert"):
        cfg = wl.config(name)
        ids = oracle.mask_padding(wl.routing(cfg), cfg.real)
        out = oracle.create_indices(ids, cfg.E)
        R = out["expert_start_indices"][-1]
        assert R == cfg.real * cfg.top_k                  # counts sum to real * top_k
        assert np.all(out["token_expert_order"][:R] < cfg.real * cfg.top_k)
        # without the mask the padding rows' garbage ids would be routed
        raw = oracle.create_indices(wl.routing(cfg), cfg.E)
        assert raw["expert_start_indices"][-1] == cfg.N * cfg.top_k


# ------------------------------------------------------------------ dispatch
@pytest.mark.parametrize("cfg", [wl.config("tiny"), wl.small_config(K=96, N=9, real=7, E=5, top_k=2)])
def test_dispatch_rows_are_grouped_token_encodings(cfg):
    x = wl.activations_bf16(cfg)
    ids = oracle.mask_padding(wl.routing(cfg), cfg.real)
    idx = oracle.create_indices(ids, cfg.E)
    recv, counts = oracle.dispatch_mxfp4(x, cfg.top_k, cfg.E, idx, fill=0xA5)
    R = int(idx["expert_start_indices"][-1])
    enc = oracle.mxfp4_encode_rows(x)
    tok = idx["token_expert_order"][:R] // cfg.top_k
    np.testing.assert_array_equal(recv[:R], enc[tok])
    assert np.all(recv[R:] == 0xA5)                       # rows past R untouched
    valid = ids[(ids >= 0) & (ids < cfg.E)]
    np.testing.assert_array_equal(counts, np.bincount(valid, minlength=cfg.E))
    # each expert segment holds exactly the tokens routed to that expert
    st = idx["expert_start_indices"]
    for a, e in enumerate(idx["expert_ids"][: idx["expert_usage_stats"][1]]):
        seg = tok[st[a]:st[a + 1]]
        np.testing.assert_array_equal(seg, np.nonzero((ids == e).any(axis=1))[0])


def test_workloads_are_deterministic_and_shaped():
    cfg = wl.config("tiny")
    a, b = wl.routing(cfg), wl.routing(cfg)
    np.testing.assert_array_equal(a, b)
    assert a.shape == (16, 2) and a.dtype == np.int64
    for r in range(cfg.real):
        assert len(set(a[r])) == cfg.top_k            # distinct experts in real rows
    w = wl.router_weights(cfg)
    np.testing.assert_allclose(w.sum(1), 1, rtol=1e-6)
    z = wl.config("decode_large_expert")
    ids = wl.routing(z)
    cnt = np.bincount(ids[: z.real].ravel(), minlength=z.E)
    assert cnt.max() > 8 * cnt.mean()                 # Zipf skew is visible
