"""The routing entry point that allocates nothing (for callers that cannot
allocate device memory or pass a workspace), called through the C ABI and
checked against the workspace-based moe_route_permute and against the
oracle's routing: identical tables on several calls in a row, so the scratch
the calls share carries nothing over from one call to the next.  The first
two calls take the three-launch path (more than 8 chunks of 1024 pairs),
whose per-chunk histograms live in the shared scratch; the third takes the
single-CTA path.  Collected last on purpose: a failure here never hides
another test."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_route_b200 as moe
import oracle as O
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


def test_noalloc_route_matches_workspace_route_and_oracle():
    assert torch.cuda.is_available()
    from fp8_block_scaled_route_b200 import build
    build.build()
    O.build()
    # calls in a row, each with a different (T, k, E): 65536 and 16000 pairs
    # (three-launch path), then 1800 pairs (single-CTA path)
    cases = [(8192, 8, 256, "zipf", 1), (2000, 8, 64, "normal", 2), (300, 6, 1000, "normal", 3)]
    for T, k, E, routing, seed in cases:
        ids, _ = synth.make_routing(T, E, k, routing, torch.Generator().manual_seed(seed), "cpu")
        got = _no_alloc(ids.cuda(), E)
        ref = _with_ws(ids.cuda(), E)
        torch.cuda.synchronize()
        for r, g in zip(ref, got):
            assert torch.equal(r, g), f"T={T} k={k} E={E}: differs from moe_route_permute"
        m_o, p_o, i_o, bad = O.route_permute(ids.numpy(), E)
        assert bad == 0
        assert np.array_equal(got[0].cpu().numpy(), m_o), f"T={T}: m_indptr"
        assert np.array_equal(got[1].cpu().numpy(), p_o), f"T={T}: perm"
        assert np.array_equal(got[2].cpu().numpy(), i_o), f"T={T}: inv_perm"
        assert int(got[0][-1]) == T * k


def test_noalloc_route_rejects_oversize():
    ids = torch.zeros(8193, 8, dtype=torch.int32, device="cuda")
    st = moe.moe_route_permute_noalloc(ids, 16, ids, ids, None, check=False)
    assert st == moe.MOE_ERR_INVALID_ARG
