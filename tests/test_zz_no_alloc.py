"""The routing entry point that allocates nothing (for callers that cannot
allocate device memory or pass a workspace) against the workspace-based
moe_route_permute: identical routing tables on two calls in a row, so the
scratch the calls share carries nothing over from one call to the next.
Collected last on purpose: a failure here never hides another test."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_route_b200 as moe
import synth

pytestmark = pytest.mark.gpu


def _with_ws(ids, E):
    T, k = ids.shape
    R = T * k
    m = torch.full((E + 1,), -5, dtype=torch.int32, device="cuda")
    p = torch.full((max(R, 1),), -5, dtype=torch.int32, device="cuda")
    ip = torch.full((max(R, 1),), -5, dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.moe_route_workspace_size(T, k, E), dtype=torch.uint8, device="cuda")
    moe.moe_route_permute(ids, E, m, p, ip, ws)
    return m, p, ip


def _no_alloc(ids, E):
    T, k = ids.shape
    R = T * k
    m = torch.full((E + 1,), -9, dtype=torch.int32, device="cuda")
    p = torch.full((max(R, 1),), -9, dtype=torch.int32, device="cuda")
    ip = torch.full((max(R, 1),), -9, dtype=torch.int32, device="cuda")
    moe.moe_route_permute_noalloc(ids, E, m, p, ip)
    return m, p, ip


def test_noalloc_route_matches_workspace_route_twice():
    assert torch.cuda.is_available()
    from fp8_block_scaled_route_b200 import build
    build.build()
    cases = [(8192, 8, 256, "zipf", 1), (300, 6, 1000, "normal", 2)]   # two calls in a row
    for T, k, E, routing, seed in cases:
        ids, _ = synth.make_routing(T, E, k, routing, torch.Generator().manual_seed(seed), "cpu")
        ids = ids.cuda()
        ref = _with_ws(ids, E)
        got = _no_alloc(ids, E)
        torch.cuda.synchronize()
        for r, g in zip(ref, got):
            assert torch.equal(r, g)
        assert int(got[0][-1]) == T * k


def test_noalloc_route_rejects_oversize():
    ids = torch.zeros(8193, 8, dtype=torch.int32, device="cuda")
    st = moe.moe_route_permute_noalloc(ids, 16, ids, ids, None, check=False)
    assert st == moe.MOE_ERR_INVALID_ARG
