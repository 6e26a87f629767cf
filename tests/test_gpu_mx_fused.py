"""Parity of the fused MXFP8 layer (moe_mxfp8_fused) against the oracle's
MXFP8 layer, called through the C ABI: routing bit-exact, the requantised
intermediate's codes and E8M0 scales, and the bf16 output with the
tolerances of tests/gpu_helpers.py.  B200 only."""
import numpy as np
import pytest
import torch

import synth
import fp8_block_scaled_route_b200 as moe
from gpu_helpers import bf16_bits, compare_codes, compare_out, f32, i32, u8

pytestmark = pytest.mark.gpu

# E8M0 scales of the intermediate: both sides take the amax of the same 32
# fp32 values up to the GEMM's accumulation order; a scale moves only when
# that amax sits within a few ulps of a power-of-two boundary.
SF_MATCH_MIN = 0.999


def _tile(sf):
    rows = sf.numel() // sf.shape[-1]
    flat = sf.reshape(rows, sf.shape[-1]).contiguous()
    out = torch.empty_like(flat)
    moe.mxfp8_tile_scales(flat, out)
    return out


def _run(inp):
    x = inp["x"]
    T, H = x.shape
    E, I2, _ = inp["w13"].shape
    I = I2 // 2
    k = inp["topk_ids"].shape[1]
    R = T * k
    ws = torch.empty(moe.moe_workspace_size(T, H, I, E, k), dtype=torch.uint8, device="cuda")
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    m_indptr = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(max(R, 1), dtype=torch.int32, device="cuda")
    hq = torch.empty(max(R, 1), I, dtype=torch.uint8, device="cuda")
    hsf = torch.empty(I // 128, max(R, 1), 4, dtype=torch.uint8, device="cuda")
    moe.moe_mxfp8_fused_debug(x, inp["topk_ids"], inp["topk_w"], inp["w13"], _tile(inp["w13_sf"]),
                              inp["w2"], _tile(inp["w2_sf"]), out, ws, m_indptr, perm, hq, hsf)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    Rg = int(m_indptr[-1])
    hsf_rm = hsf[:, :Rg, :].permute(1, 0, 2).reshape(Rg, I // 32)
    return (bf16_bits(out), i32(m_indptr), i32(perm[:Rg]), u8(hq[:Rg]), u8(hsf_rm))


def _check(oracle, inp, what):
    got = _run(inp)
    ref = oracle.moe_mx_fused(bf16_bits(inp["x"]), i32(inp["topk_ids"]), f32(inp["topk_w"]),
                              u8(inp["w13"]), u8(inp["w13_sf"]), u8(inp["w2"]), u8(inp["w2_sf"]),
                              want_dump=True)
    out, m_indptr, perm, hq, hsf = got
    r_out, r_m, r_perm, r_hq, r_hsf = ref
    np.testing.assert_array_equal(m_indptr, r_m, err_msg=f"{what}: m_indptr")
    np.testing.assert_array_equal(perm, r_perm, err_msg=f"{what}: perm")
    if r_hq.size:
        frac = float((hsf == r_hsf).mean())
        assert frac >= SF_MATCH_MIN, f"{what}: {frac:.5f} of E8M0 scales identical"
        assert int(np.abs(hsf.astype(int) - r_hsf.astype(int)).max()) <= 1, what
        same = hsf == r_hsf  # codes are comparable where the block scale agrees
        blk = np.repeat(same, 32, axis=1)
        compare_codes(hq[blk], r_hq[blk], f"{what}: intermediate codes")
    compare_out(out, r_out, f"{what}: output")


def test_mx_fused_tiny(oracle):
    _check(oracle, synth.make_mx_moe_inputs(synth.CONFIGS["tiny"], seed=0, device="cuda"), "tiny")


@pytest.mark.parametrize("T,H,I,E,k,routing", [
    (33, 256, 256, 5, 3, "normal"),     # ragged tiles, odd group sizes
    (200, 512, 384, 16, 4, "zipf"),     # skewed groups, I not a multiple of 256
    (300, 384, 256, 8, 2, "normal"),    # GEMM2 with an odd number of 128-column blocks
])
def test_mx_fused_shapes(oracle, T, H, I, E, k, routing):
    cfg = synth.MoEConfig("mx_case", T, H, I, E, k, routing)
    _check(oracle, synth.make_mx_moe_inputs(cfg, seed=T, device="cuda"), f"T={T}")


def test_mx_fused_zero_tokens():
    cfg = synth.MoEConfig("mx_zero", 0, 256, 128, 4, 2)
    inp = synth.make_mx_moe_inputs(cfg, seed=0, device="cuda")
    out = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(moe.moe_workspace_size(0, 256, 128, 4, 2), dtype=torch.uint8, device="cuda")
    assert moe.moe_mxfp8_fused(inp["x"], inp["topk_ids"], inp["topk_w"], inp["w13"],
                               _tile(inp["w13_sf"]), inp["w2"], _tile(inp["w2_sf"]), out, ws) == 0


def _compact_mx(inp, tokens):
    """Host copies of only the experts the listed tokens use (MXFP8 weights and
    row-major scales), with their routing renumbered into the compact list."""
    dev = inp["topk_ids"].device
    sel = torch.as_tensor(tokens, device=dev)
    ids = inp["topk_ids"][sel]
    used = torch.unique(ids).to(torch.long)
    remap = torch.full((inp["w13"].shape[0],), -1, dtype=torch.int32, device=dev)
    remap[used] = torch.arange(len(used), dtype=torch.int32, device=dev)
    return dict(x=bf16_bits(inp["x"][sel]), topk_ids=i32(remap[ids]), topk_w=f32(inp["topk_w"][sel]),
                w13=u8(inp["w13"][used]), w13_sf=u8(inp["w13_sf"][used]),
                w2=u8(inp["w2"][used]), w2_sf=u8(inp["w2_sf"][used]))


def _check_mx_sampled(oracle, inp, tokens, what):
    out, m_indptr, perm, hq, hsf = _run(inp)
    E = inp["w13"].shape[0]
    m_o, p_o, i_o, _ = oracle.route_permute(i32(inp["topk_ids"]), E)
    np.testing.assert_array_equal(m_indptr, m_o, err_msg=what)
    np.testing.assert_array_equal(perm, p_o, err_msg=what)
    sub = _compact_mx(inp, tokens)
    out_o, hq_o, hsf_o = oracle.moe_mx_tokens(sub["x"], sub["topk_ids"], sub["topk_w"], sub["w13"],
                                              sub["w13_sf"], sub["w2"], sub["w2_sf"],
                                              np.arange(len(tokens), dtype=np.int32), want_h=True)
    k = inp["topk_ids"].shape[1]
    rows = np.array([[i_o[t * k + j] for j in range(k)] for t in tokens]).ravel()
    got_sf, ref_sf = hsf[rows], hsf_o.reshape(len(rows), -1)
    assert float((got_sf == ref_sf).mean()) >= SF_MATCH_MIN, what
    same = np.repeat(got_sf == ref_sf, 32, axis=1)
    compare_codes(hq[rows][same], hq_o.reshape(len(rows), -1)[same], what + " codes")
    compare_out(out[tokens], out_o, what + " output")


def test_mx_fused_decode_full_size_sampled(oracle):
    inp = synth.make_mx_moe_inputs(synth.CONFIGS["decode"], seed=0, device="cuda")
    _check_mx_sampled(oracle, inp, [0, 17, 42, 63], "mx decode")
    del inp
    torch.cuda.empty_cache()


def test_mx_fused_prefill_full_size_sampled(oracle):
    inp = synth.make_mx_moe_inputs(synth.CONFIGS["prefill"], seed=0, device="cuda")
    ids = inp["topk_ids"]
    counts = torch.bincount(ids.flatten().long(), minlength=256)
    big = int(torch.argmax(counts))
    nz = torch.nonzero(counts).flatten()
    small = int(nz[torch.argmin(counts[nz])])
    t_big = int(torch.nonzero((ids == big).any(1)).flatten()[0])
    t_small = int(torch.nonzero((ids == small).any(1)).flatten()[0])
    _check_mx_sampled(oracle, inp, sorted({0, t_big, t_small, 8191}), "mx prefill")
    del inp
    torch.cuda.empty_cache()
