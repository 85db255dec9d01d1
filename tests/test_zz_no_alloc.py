"""The workspace-free grouping entry point, moe_create_indices_static.

Some callers of this library cannot allocate device memory at run time (plugin
hosts that pass only input and output tensors, serving loops with a frozen
memory plan).  For them moe_create_indices_static keeps its scratch in a fixed
array inside the library.  These tests call it through the C ABI and check
that its outputs equal those of the regular moe_create_indices (integer
outputs, so equality is exact), on two calls in a row that share the scratch,
and that a problem too large for the fixed scratch is refused up front.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import permute_fp4_dispatch_b200 as moe
from permute_fp4_dispatch_b200.build import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_library():
    build()
    moe.library()
    yield
    assert moe.moe_get_device_error(clear=True) == 0


def _outputs(S, E):
    i32 = dict(dtype=torch.int32, device="cuda")
    return dict(order=torch.full((max(S, 1),), -7, **i32), start=torch.full((E + 1,), -7, **i32),
                restore=torch.full((max(S, 1),), -7, **i32), eids=torch.full((E,), -7, **i32),
                stats=torch.full((2,), -7, **i32), soff=torch.full((E + 1,), -7, **i32))


def _regular(ids_t, S, E):
    o = _outputs(S, E)
    ws_bytes = moe.moe_create_indices_workspace_bytes(S, E)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device="cuda")
    moe.moe_create_indices(ids_t, S, E, o["order"], o["start"], o["restore"], o["eids"],
                           o["stats"], o["soff"], ws, ws_bytes)
    return o


def _static(ids_t, S, E):
    o = _outputs(S, E)
    moe.moe_create_indices_static(ids_t, S, E, o["order"], o["start"], o["restore"], o["eids"],
                                  o["stats"], o["soff"])
    return o


def _same(a, b):
    torch.cuda.synchronize()
    for k in a:
        assert torch.equal(a[k], b[k]), k


@pytest.mark.parametrize("S,E", [(40000, 64), (500000, 1024)])
def test_static_matches_regular_on_two_calls(S, E):
    # both cases take the tiled path, whose per-tile histograms live in the
    # fixed scratch; the second fills it almost to its limit
    assert S > 16384
    assert moe.moe_create_indices_workspace_bytes(S, E) <= moe.MOE_CREATE_INDICES_STATIC_SCRATCH
    rng = np.random.default_rng(S + E)
    first = torch.from_numpy(rng.integers(-1, E + 1, S).astype(np.int64)).cuda()
    second = torch.from_numpy(rng.integers(-1, E + 1, S).astype(np.int64)).cuda()
    # two calls in a row: the second reuses the scratch the first left behind
    s1 = _static(first, S, E)
    s2 = _static(second, S, E)
    _same(s1, _regular(first, S, E))
    _same(s2, _regular(second, S, E))


def test_static_rejects_problems_beyond_its_scratch():
    E = 1024
    S = 600 * 8192                           # needs 600 tiles x 1024 experts x 4 bytes
    assert moe.moe_create_indices_workspace_bytes(S, E) > moe.MOE_CREATE_INDICES_STATIC_SCRATCH
    o = _outputs(1, E)
    with pytest.raises(moe.MoeError) as err:
        moe.moe_create_indices_static(16, S, E, o["order"], o["start"], o["restore"], o["eids"],
                                      o["stats"], o["soff"])
    assert err.value.status == 3             # MOE_ERR_WORKSPACE: nothing was launched
    assert torch.all(o["start"] == -7)
