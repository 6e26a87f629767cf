"""GPU parity of the fused-expert launch (gate/up GEMM, SwiGLU, FP8
requantisation and down GEMM in one kernel, the intermediate kept in shared
memory) against the CPU oracle, with fusion forced on; and the automatic
choice between it and the two-launch path."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_route_b200 as moe
import oracle as O
import synth
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_block_scaled_route_b200 import build
    build.build()
    moe.lib()
    O.build()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


@pytest.fixture
def fusion_on():
    moe.moe_set_expert_fusion(moe.MOE_FUSION_ON)
    yield
    moe.moe_set_expert_fusion(moe.MOE_FUSION_AUTO)


def _check(inp, what, debug=True):
    """Against the oracle through the debug entry point; with debug=False the
    plain entry point must then give the same output bits."""
    res = G.run_fused(inp, debug=True)
    assert res["status"] == moe.MOE_OK, what
    ref = O.moe_fused(*G.oracle_args(inp))
    assert np.array_equal(res["m_indptr"], ref["m_indptr"]), what
    assert np.array_equal(res["perm"], ref["perm"]), what
    G.compare_codes(res["hq"], ref["hq"], what + " intermediate codes")
    G.compare_scales(res["hs"], ref["hs"], what + " intermediate scales")
    G.compare_layer(res, ref, inp, what + " output")
    if not debug:
        plain = G.run_fused(inp, debug=False)
        assert plain["status"] == moe.MOE_OK, what
        assert np.array_equal(plain["out"], res["out"]), what + ": plain entry point differs"
    return res


@pytest.mark.parametrize("T,H,I,E,k,routing", [
    (16, 256, 128, 4, 2, "normal"),       # tiny: one tile per expert
    (100, 512, 256, 16, 4, "normal"),     # ragged groups
    (1, 256, 128, 4, 2, "normal"),        # a single token
    (40, 384, 384, 1, 1, "normal"),       # one expert; H = 3 x 128: last down tile half empty
    (24, 256, 128, 6, 6, "normal"),       # every expert chosen by every token
    (200, 256, 256, 64, 2, "zipf"),       # many empty experts
    (1000, 256, 128, 8, 2, "zipf"),       # ~250 rows per expert: several 64-row items each
    (300, 640, 640, 12, 3, "normal"),     # 5 intermediate blocks, H = 5 x 128
    (130, 1024, 768, 3, 2, "normal"),     # long K loops, ragged last item per expert
    (64, 2048, 768, 128, 8, "normal"),    # the mid workload's expert shape
    (600, 256, 128, 1024, 8, "zipf"),     # the largest expert count (item table of 1024)
    (48, 7168, 128, 16, 2, "normal"),     # the pages' H with a small I: 56 K blocks in phase 1
])
def test_fused_expert_parity(fusion_on, T, H, I, E, k, routing):
    cfg = synth.MoEConfig("case", T, H, I, E, k, routing)
    inp = synth.make_moe_inputs(cfg, seed=3 * T + E, device=DEV)
    _check(inp, f"fused expert T={T} H={H} I={I} E={E} k={k}")


def test_fused_expert_without_debug_outputs(fusion_on):
    """The plain entry point (intermediate never leaves the chip)."""
    inp = synth.make_moe_inputs(synth.MoEConfig("nd", 200, 512, 384, 16, 4), seed=9, device=DEV)
    _check(inp, "fused expert, no debug outputs", debug=False)


def test_fused_expert_matches_two_launch_path():
    """Both paths quantise the intermediate with the same arithmetic and
    sum each K block's partial products in the same order: bit-identical
    intermediate and output."""
    inp = synth.make_moe_inputs(synth.MoEConfig("ab", 256, 1024, 512, 32, 4), seed=2, device=DEV)
    try:
        moe.moe_set_expert_fusion(moe.MOE_FUSION_OFF)
        a = G.run_fused(inp, debug=True)
        moe.moe_set_expert_fusion(moe.MOE_FUSION_ON)
        b = G.run_fused(inp, debug=True)
    finally:
        moe.moe_set_expert_fusion(moe.MOE_FUSION_AUTO)
    assert a["status"] == moe.MOE_OK and b["status"] == moe.MOE_OK
    assert np.array_equal(a["perm"], b["perm"])
    assert np.array_equal(b["hq"], a["hq"])
    assert np.array_equal(b["hs"].view(np.uint32), a["hs"].view(np.uint32))
    assert np.array_equal(b["out"], a["out"])


def test_fused_expert_bad_ids_and_zero_tokens(fusion_on):
    inp = synth.make_moe_inputs(synth.MoEConfig("bad", 32, 256, 128, 8, 2), seed=4, device=DEV)
    inp["topk_ids"][3, 1] = -1
    inp["topk_ids"][10, 0] = 8
    res = G.run_fused(inp, debug=True)
    assert res["status"] == moe.MOE_ERR_BAD_EXPERT_ID
    ref = O.moe_fused(*G.oracle_args(inp))
    assert np.array_equal(res["m_indptr"], ref["m_indptr"])
    n = int(ref["m_indptr"][-1])
    assert np.array_equal(res["perm"][:n], ref["perm"])
    G.compare_layer(res, ref, inp, "fused expert, bad ids")
    empty = synth.make_moe_inputs(synth.MoEConfig("empty", 0, 256, 128, 4, 2), seed=1, device=DEV)
    res = G.run_fused(empty, debug=True)
    assert res["status"] == moe.MOE_OK and np.all(res["m_indptr"] == 0)


def test_fused_expert_too_large_falls_back():
    """I = 2048 does not fit on chip: fusion on still runs the two launches."""
    inp = synth.make_moe_inputs(synth.MoEConfig("big", 8, 256, 2048, 4, 2), seed=6, device=DEV)
    moe.moe_set_expert_fusion(moe.MOE_FUSION_ON)
    try:
        _check(inp, "I=2048 with fusion on")
    finally:
        moe.moe_set_expert_fusion(moe.MOE_FUSION_AUTO)


def test_fused_expert_timeout_is_reported_and_context_survives(fusion_on):
    inp = synth.make_moe_inputs(synth.MoEConfig("tmo", 300, 512, 256, 8, 2), seed=5, device=DEV)
    moe.moe_set_wait_timeout_ns(1)
    try:
        res = G.run_fused(inp, debug=False)
        assert res["status"] == moe.MOE_ERR_DEVICE_TIMEOUT
    finally:
        moe.moe_set_wait_timeout_ns(2_000_000_000)
    torch.cuda.synchronize()
    _check(inp, "fused expert after timeout", debug=False)



def test_plan_reports_the_path_taken():
    """moe_fp8_fused_plan: fusion where the rule picks it, never where the
    intermediate does not fit, always off when switched off."""
    try:
        moe.moe_set_expert_fusion(moe.MOE_FUSION_AUTO)
        assert moe.moe_fp8_fused_plan(512, 2048, 768, 128, 8)["fused"]       # the mid workload
        assert not moe.moe_fp8_fused_plan(64, 7168, 2048, 256, 8)["fused"]   # decode: does not fit
        assert not moe.moe_fp8_fused_plan(8192, 7168, 2048, 256, 8)["fused"]
        moe.moe_set_expert_fusion(moe.MOE_FUSION_ON)
        assert moe.moe_fp8_fused_plan(64, 7168, 896, 256, 8)["fused"]        # fits: forced on
        assert not moe.moe_fp8_fused_plan(64, 7168, 2048, 256, 8)["fused"]
        moe.moe_set_expert_fusion(moe.MOE_FUSION_OFF)
        assert not moe.moe_fp8_fused_plan(512, 2048, 768, 128, 8)["fused"]
    finally:
        moe.moe_set_expert_fusion(moe.MOE_FUSION_AUTO)
