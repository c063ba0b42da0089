"""The allocation-free grouping entry point (moe_permute_noalloc).

Some callers cannot allocate device memory (a fixed pool owned by another
component, or a loop that may not take an allocation's device-wide
synchronisation), so they cannot hand the library a workspace.  This checks,
through the C ABI, that the variant whose scratch lives in the library's own
static device array gives exactly the grouping of moe_permute with a caller
workspace and of the oracle's counting sort, on two calls in a row, for both
the single-block (T <= 256) and the multi-block path, including the largest
case the array holds (T = 16384, E = 1024: all 64 x 1024 entries), and that
sizes beyond the array are refused.

This file is collected last so that a failure here does not stop a run that
stops at the first failure before every other test has run.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from oracle import moe_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_moe_layer_04_b200 as m
    return m


def _outs(T, E, k):
    return (torch.empty(E, dtype=torch.int32, device="cuda"),
            torch.empty(E + 1, dtype=torch.int32, device="cuda"),
            torch.empty(T * k, dtype=torch.int32, device="cuda"),
            torch.empty((T, k), dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("T,E,k", [(200, 256, 8), (3000, 256, 8), (16384, 64, 4), (777, 1024, 32),
                                   (16384, 1024, 8)])
def test_noalloc_matches_workspace_grouping_twice(moe, T, E, k):
    d = moe.dims(T=T, D=64, E=E, F=64, k=k)
    ws = moe.alloc_workspace(d)
    for call in range(2):
        idx = mi.synthetic_topk(T, E, k, call, f"noalloc{T}x{E}").cuda()
        ref = _outs(T, E, k)
        moe.moe_permute(idx, d, *ref, ws)
        got = _outs(T, E, k)
        for t in got:
            t.fill_(-7)
        moe.moe_permute_noalloc(idx, d, *got)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
        # and the oracle's counting sort of the same pairs, bit for bit
        counts, offsets, perm, inv = orc.group_by_expert(idx.cpu().numpy(), E)
        for a, b in zip(got, (counts, offsets, perm, inv)):
            assert np.array_equal(a.cpu().numpy(), b)


def test_noalloc_rejects_sizes_beyond_the_scratch(moe):
    d = moe.dims(T=16385, D=64, E=8, F=64, k=2)
    outs = _outs(16385, 8, 2)
    idx = torch.zeros((16385, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_permute_noalloc(idx, d, *outs)
    assert ei.value.code == moe.MOE_ERR_UNSUPPORTED and "static scratch" in str(ei.value)
