"""The tactic table on the GPU: tuning times every tile valid for K on the
caller's buffers, stores the fastest, and a tile_m = -1 call then runs that
tile (bit-identical to an explicit call with it).  B200 only."""
import pytest
import torch

import synth
import fp8_block_scaled_route_b200 as moe

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_table():
    moe.moe_tactic_clear()
    yield
    moe.moe_tactic_clear()


@pytest.mark.parametrize("R,N,K,E,gated", [
    (600, 512, 1024, 8, False),
    (96, 1024, 2048, 16, True),      # ~6 rows per expert
    (2048, 512, 7168, 4, False),     # 56 K blocks
])
def test_tune_then_auto_tile(R, N, K, E, gated):
    inp = synth.make_grouped_gemm_inputs(R, N, K, E, seed=R, device="cuda")
    out = torch.empty(R, N // 2 if gated else N, dtype=torch.bfloat16, device="cuda")
    tm = moe.moe_tactic_tune_gemm(inp["a"], inp["b"], inp["a_scale"], inp["b_scale"],
                                  inp["m_indptr"], out, "K", gated, iters=3)
    assert tm in (16, 32, 64, 128)
    assert moe.moe_tactic_lookup(R, N, K, E, gated) == tm
    auto = torch.empty_like(out)
    expl = torch.empty_like(out)
    moe.fp8_groupwise_moe_gemm(inp["a"], inp["b"], inp["a_scale"], inp["b_scale"], inp["m_indptr"],
                               auto, "K", (1, 128, 128), gated, -1)
    moe.fp8_groupwise_moe_gemm(inp["a"], inp["b"], inp["a_scale"], inp["b_scale"], inp["m_indptr"],
                               expl, "K", (1, 128, 128), gated, tm)
    torch.cuda.synchronize()
    rows = int(inp["m_indptr"][-1])
    assert torch.equal(auto[:rows].view(torch.int16), expl[:rows].view(torch.int16))
