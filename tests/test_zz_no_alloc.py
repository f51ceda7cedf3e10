"""The allocation-free bucketing call against the workspace-based one.

moe_permute_noalloc serves callers that cannot allocate device memory (an
engine with a fixed memory plan, or a step that must not stall on an
allocation); its scratch is a static device array instead of a workspace.  It
must produce exactly what moe_permute produces (integer outputs, bit for bit),
and two calls in a row must not leave state that changes the second result.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_only_bit_route_b200 import moe

pytestmark = pytest.mark.gpu


def _ids(T, k, E, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)


def test_permute_noalloc_matches_workspace_permute():
    assert torch.cuda.is_available()
    cases = [(_ids(300, 8, 352, 1), 352), (_ids(37, 8, 32, 2), 32)]     # two calls in a row
    for ids_np, E in cases:
        ids = torch.from_numpy(ids_np).cuda()
        T, k = ids_np.shape
        ws = moe.workspace(T, 128, E, 128, k)
        off, rs, sr = moe.permute(ids, E, ws)
        off2, rs2, sr2 = moe.permute_noalloc(ids, E)
        torch.cuda.synchronize()
        assert torch.equal(off, off2)
        assert torch.equal(rs, rs2)
        assert torch.equal(sr, sr2)
        # and against the oracle's bucketing directly
        o_off, o_rs, o_sr = oracle.permute(ids_np, E)
        assert np.array_equal(off2.cpu().numpy(), o_off)
        assert np.array_equal(rs2.cpu().numpy(), o_rs)
        assert np.array_equal(sr2.cpu().numpy(), o_sr)


def test_permute_noalloc_rejects_oversize():
    ids = torch.zeros(65537, 1, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoEError):
        moe.permute_noalloc(ids, 8)
