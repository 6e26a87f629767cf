"""Parity of the device router (moe_router_topk) against the oracle's router,
through the C ABI: expert ids bit-exact, weights within a few fp32 ulps (expf
on the device and on the host may differ in the last bit).  B200 only."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_route_b200 as moe

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,E,k,seed", [(64, 256, 8, 0), (1000, 128, 8, 1), (33, 5, 5, 2),
                                        (257, 1024, 32, 3), (7, 300, 1, 4), (8192, 256, 8, 5)])
def test_router_topk(oracle, T, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    logits = torch.randn(T, E, generator=g)
    if T > 2 and E > 2:
        logits[0, 1] = logits[0, 0]          # ties inside and at the edge of the top-k
        logits[1, E - 1] = logits[1, 0]
        logits[2, :] = 0.5                   # all equal: ids 0..k-1, uniform weights
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    moe.moe_router_topk(logits.cuda(), ids, w)
    torch.cuda.synchronize()
    r_ids, r_w = oracle.router_topk(logits.numpy(), k)
    np.testing.assert_array_equal(ids.cpu().numpy(), r_ids)
    np.testing.assert_allclose(w.cpu().numpy(), r_w, rtol=1e-6, atol=1e-9)


def test_router_empty_and_bad_args():
    logits = torch.zeros(0, 16, device="cuda")
    ids = torch.zeros(0, 4, dtype=torch.int32, device="cuda")
    w = torch.zeros(0, 4, device="cuda")
    assert moe.moe_router_topk(logits, ids, w) == 0
    assert moe.moe_router_topk(logits, ids, w, dims=(0, 16, 17), check=False) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_router_topk(logits, ids, w, dims=(0, 64, 33), check=False) == moe.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("T,E,k,seed", [(64, 256, 8, 0), (1000, 128, 8, 1), (33, 5, 5, 2),
                                        (257, 1024, 4, 3), (2000, 64, 8, 6), (1, 3, 2, 7)])
def test_router_route_one_call(oracle, T, E, k, seed):
    """moe_router_route (router and grouping in one call; one launch up to 8192
    pairs) against the oracle's router and grouping: ids and tables
    bit-exact, weights within a few fp32 ulps."""
    g = torch.Generator().manual_seed(100 + seed)
    logits = torch.randn(T, E, generator=g)
    R = T * k
    ids = torch.full((T, k), -3, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    m = torch.full((E + 1,), -3, dtype=torch.int32, device="cuda")
    perm = torch.full((R,), -3, dtype=torch.int32, device="cuda")
    inv = torch.full((R,), -3, dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.moe_route_workspace_size(T, k, E), dtype=torch.uint8, device="cuda")
    moe.moe_router_route(logits.cuda(), k, ids, w, m, perm, inv, ws)
    assert moe.moe_get_device_status(ws) == moe.MOE_OK
    r_ids, r_w = oracle.router_topk(logits.numpy(), k)
    np.testing.assert_array_equal(ids.cpu().numpy(), r_ids)
    np.testing.assert_allclose(w.cpu().numpy(), r_w, rtol=1e-6, atol=1e-9)
    m_o, p_o, i_o, bad = oracle.route_permute(r_ids, E)
    assert bad == 0
    np.testing.assert_array_equal(m.cpu().numpy(), m_o)
    np.testing.assert_array_equal(perm.cpu().numpy(), p_o)
    np.testing.assert_array_equal(inv.cpu().numpy(), i_o)
