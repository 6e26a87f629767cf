"""Failure detection on the GPU without a fault: a wait bound far shorter
than the pipeline's latency makes the grouped GEMM's bounded waits run out.
The kernel must report MOE_ERR_DEVICE_TIMEOUT through the status word,
return, and leave the context usable for the next, correct call."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_route_b200 as moe
import oracle as O
import synth
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu

DEFAULT_TIMEOUT_NS = 2_000_000_000


def _gemm(inp, out):
    return moe.fp8_groupwise_moe_gemm(inp["a"], inp["b"], inp["a_scale"], inp["b_scale"],
                                      inp["m_indptr"], out, "K", (1, 128, 128), True, -1, -1)


def test_wait_timeout_is_reported_and_context_survives():
    assert torch.cuda.is_available()
    inp = synth.make_grouped_gemm_inputs(0, 1024, 7168, 4, seed=3, group_sizes=[300, 7, 0, 90],
                                         device="cuda")
    R = int(inp["m_indptr"][-1])
    out = torch.zeros(R, 512, dtype=torch.bfloat16, device="cuda")
    moe.moe_set_wait_timeout_ns(1)
    try:
        _gemm(inp, out)
        assert moe.moe_get_device_status(None) == moe.MOE_ERR_DEVICE_TIMEOUT
    finally:
        moe.moe_set_wait_timeout_ns(DEFAULT_TIMEOUT_NS)
    torch.cuda.synchronize()          # the context is still healthy
    _gemm(inp, out)
    assert moe.moe_get_device_status(None) == moe.MOE_OK
    ref = O.groupwise_gemm_bf16(G.u8(inp["a"]), G.f32(inp["a_scale"]), G.u8(inp["b"]),
                                G.f32(inp["b_scale"]), G.i32(inp["m_indptr"]), True)
    G.compare_out(G.bf16_bits(out), ref, "after timeout")


def test_fused_layer_timeout_is_reported_and_context_survives():
    """The same through the fused layer at a shape with 128-row tiles: every
    kernel after the first one that gives up still ends and reports."""
    cfg = synth.MoEConfig("tiles128", 700, 512, 256, 4, 2)
    inp = synth.make_moe_inputs(cfg, seed=5, device="cuda")
    moe.moe_set_wait_timeout_ns(1)
    try:
        res = G.run_fused(inp, debug=False)
        assert res["status"] == moe.MOE_ERR_DEVICE_TIMEOUT
    finally:
        moe.moe_set_wait_timeout_ns(DEFAULT_TIMEOUT_NS)
    torch.cuda.synchronize()
    res = G.run_fused(inp, debug=False)
    assert res["status"] == moe.MOE_OK
    ref = O.moe_fused(*G.oracle_args(inp))
    G.compare_out(res["out"], ref["out"], "fused layer after timeout")
