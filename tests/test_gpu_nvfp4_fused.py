"""Parity of the NVFP4 path against the oracle, called through the C ABI: the
quantiser (nvfp4_quantize) bit-exact, and the fused NVFP4 layer
(moe_nvfp4_fused): routing bit-exact, the requantised intermediate's E4M3
scales and E2M1 codes, and the bf16 output with the tolerances of
tests/gpu_helpers.py.  B200 only."""
import numpy as np
import pytest
import torch

import synth
import fp8_block_scaled_route_b200 as moe
from gpu_helpers import OUT_MAX_ABS_RMS, OUT_REL_L2, bf16_bits, bits_to_f64, f32, i32, u8

pytestmark = pytest.mark.gpu

# E4M3 scales of the intermediate: both sides take the amax of the same 16
# fp32 values up to the GEMM's accumulation order; a scale moves only when
# amax * g / 6 sits within a few ulps of a rounding midpoint.
SF_MATCH_MIN = 0.999
CODE_MATCH_MIN = 0.999


def _unpack(packed):
    """[rows, n/2] bytes -> [rows, n] codes, element 2i from the low nibble."""
    p = np.asarray(packed, np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def _rank(codes):
    """Signed E2M1 magnitude rank (+0 and -0 share rank 0)."""
    c = np.asarray(codes, np.int64)
    return np.where(c & 8, -(c & 7), c & 7)


def _compare_e2m1(got, ref, what):
    got, ref = _rank(got).ravel(), _rank(ref).ravel()
    if got.size == 0:
        return
    frac = float((got == ref).mean())
    assert frac >= CODE_MATCH_MIN, f"{what}: only {frac:.5f} of codes identical"
    assert int(np.abs(got - ref).max()) <= 1, f"{what}: a code differs by more than one step"


@pytest.mark.parametrize("M,K", [(300, 1024), (37, 384)])  # 384: a warp's last 8 lanes idle
def test_nvfp4_quantize_bit_exact(oracle, M, K):
    """Codes and scales identical to the oracle's on the exact fp32 values of
    bf16 rows (x N(0,1) with per-16 magnitudes 2^U{-3..3}, a few all-zero
    blocks and values past the saturation point).  +0 and -0 codes are
    treated as equal (both decode to 0)."""
    g = torch.Generator().manual_seed(K)
    x = torch.randn(M, K, generator=g)
    u = torch.randint(-3, 4, (M, K // 16), generator=g).float()
    x = (x.view(M, K // 16, 16) * torch.exp2(u)[:, :, None]).view(M, K)
    x[5, 32:48] = 0.0
    x[7, :16] *= 1e4
    xb = x.to(torch.bfloat16)
    gs = 448.0 * 6.0 / 64.0
    q = torch.empty(M, K // 2, dtype=torch.uint8, device="cuda")
    sf = torch.empty(M, K // 16, dtype=torch.uint8, device="cuda")
    moe.nvfp4_quantize(xb.cuda(), gs, q, sf)
    torch.cuda.synchronize()
    ref_q, ref_sf = oracle.quant_rows_nvfp4(xb.float().numpy(), gs)
    np.testing.assert_array_equal(u8(sf), ref_sf)
    np.testing.assert_array_equal(_rank(_unpack(u8(q))), _rank(ref_q))


def _tile(sf, rows_k16):
    rows, nsf = rows_k16
    out = torch.empty(rows, nsf, dtype=torch.uint8, device=sf.device)
    moe.nvfp4_tile_scales(sf.reshape(rows, nsf).contiguous(), out)
    return out


def _alphas(inp):
    a13 = (1.0 / (inp["a1_g"] * inp["w13_g"].double())).float()
    a2 = (1.0 / (inp["a2_g"] * inp["w2_g"].double())).float()
    return a13, a2


def _run(inp):
    x = inp["x"]
    T, H = x.shape
    E, I2, _ = inp["w13_packed"].shape
    I = I2 // 2
    k = inp["topk_ids"].shape[1]
    R = T * k
    dev = x.device
    ws = torch.empty(moe.moe_workspace_size(T, H, I, E, k), dtype=torch.uint8, device=dev)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    m_indptr = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(max(R, 1), dtype=torch.int32, device=dev)
    hq = torch.empty(max(R, 1), I // 2, dtype=torch.uint8, device=dev)
    hsf = torch.empty(I // 64, max(R, 1), 4, dtype=torch.uint8, device=dev)  # K-block-major
    a13, a2 = _alphas(inp)
    moe.moe_nvfp4_fused_debug(x, inp["topk_ids"], inp["topk_w"], inp["w13_packed"],
                              _tile(inp["w13_sf"], (E * 2 * I, H // 16)), a13,
                              inp["w2_packed"], _tile(inp["w2_sf"], (E * H, I // 16)), a2,
                              inp["a1_g"], inp["a2_g"], out, ws, m_indptr, perm, hq, hsf)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    Rg = int(m_indptr[-1])
    hsf_rm = hsf[:, :Rg, :].permute(1, 0, 2).reshape(Rg, I // 16)
    return bf16_bits(out), i32(m_indptr), i32(perm[:Rg]), _unpack(u8(hq[:Rg])), u8(hsf_rm)


# The output is checked twice, with the layer's bounds each time (relative
# L2 <= 1e-2, max abs <= 2e-2 rms):
#  * against the oracle's GEMM2 + combine run on the GPU's own intermediate
#    (codes and block scales), on every token row: this checks the second
#    GEMM and the combine without the first GEMM's rounding;
#  * against the oracle's whole layer: relative L2 on all rows, max abs on
#    the token rows whose k intermediate rows match the oracle's exactly.
# A token row whose intermediate differs (a code or a block scale on the
# other side of a rounding midpoint, the GEMM1 sums differing in
# accumulation order; the intermediate itself is compared above) can move by
# one E2M1 step of a block, up to a third of its maximum, which no
# element-wise bound on the end-to-end output could absorb.
def _out_errors(gpu_bits, ref_bits):
    g, r = bits_to_f64(gpu_bits), bits_to_f64(ref_bits)
    assert np.all(np.isfinite(g)), "non-finite output"
    rms = float(np.sqrt(np.mean(r * r)))
    rel_l2 = float(np.linalg.norm(g - r) / np.linalg.norm(r))
    return rel_l2, np.abs(g - r).max(axis=1) / rms


def _compare_out(gpu_bits, ref_bits, cond_bits, exact_rows, what):
    if np.asarray(ref_bits).size == 0:
        return
    rel, err = _out_errors(gpu_bits, cond_bits)
    assert rel <= OUT_REL_L2, f"{what}: relative L2 {rel:.3e} against GEMM2 on the GPU intermediate"
    assert err.max() <= OUT_MAX_ABS_RMS, \
        f"{what}: max abs {err.max():.3e} x rms against GEMM2 on the GPU intermediate"
    rel, err = _out_errors(gpu_bits, ref_bits)
    assert rel <= OUT_REL_L2, f"{what}: relative L2 {rel:.3e}"
    exact_rows = np.asarray(exact_rows, bool)
    if exact_rows.any():
        assert err[exact_rows].max() <= OUT_MAX_ABS_RMS, \
            f"{what}: max abs {err[exact_rows].max():.3e} x rms on rows with identical intermediates"


def _gemm2_on(oracle, hq, hsf, row_expert, w2, w2_sf, w2_g, topk_w, a2_g):
    """Oracle GEMM2 + combine on a given intermediate: hq [n, I] codes and
    hsf [n, I/16] of the n = T*k pairs in pair order (row t*k + j), row_expert
    [n] their experts (compact ids into w2).  Returns bf16 bits [T, H]."""
    order = np.argsort(row_expert, kind="stable")
    E = w2.shape[0]
    m = np.concatenate([[0], np.cumsum(np.bincount(row_expert, minlength=E))]).astype(np.int32)
    y = oracle.nvfp4_grouped_gemm(np.ascontiguousarray(hq[order]), np.ascontiguousarray(hsf[order]),
                                  a2_g, w2, w2_sf, w2_g, m)
    inv = np.empty(len(order), np.int32)
    inv[order] = np.arange(len(order), dtype=np.int32)
    return oracle.combine(y, inv, topk_w)


def _exact_tokens(hq, hsf, r_hq, r_hsf, pair_of_row, T, k):
    """Tokens all of whose k intermediate rows (codes and scales) match."""
    row_same = (_rank(hq) == _rank(r_hq)).all(axis=1) & (hsf == r_hsf).all(axis=1)
    tok_ok = np.ones(T, bool)
    for r, pair in enumerate(pair_of_row):
        if not row_same[r]:
            tok_ok[pair // k] = False
    return tok_ok


def _check_h(hq, hsf, r_hq, r_hsf, what):
    if r_hq.size == 0:
        return
    frac = float((hsf == r_hsf).mean())
    assert frac >= SF_MATCH_MIN, f"{what}: {frac:.5f} of E4M3 scales identical"
    same = np.repeat(hsf == r_hsf, 16, axis=1)  # codes are comparable where the block scale agrees
    _compare_e2m1(hq[same], r_hq[same], f"{what}: intermediate codes")


def _check(oracle, inp, what):
    out, m_indptr, perm, hq, hsf = _run(inp)
    ref = oracle.moe_nvfp4_fused(bf16_bits(inp["x"]), i32(inp["topk_ids"]), f32(inp["topk_w"]),
                                 u8(inp["w13"]), u8(inp["w13_sf"]), f32(inp["w13_g"]),
                                 u8(inp["w2"]), u8(inp["w2_sf"]), f32(inp["w2_g"]),
                                 inp["a1_g"], inp["a2_g"], want_dump=True)
    r_out, r_m, r_perm, r_hq, r_hsf = ref
    np.testing.assert_array_equal(m_indptr, r_m, err_msg=f"{what}: m_indptr")
    np.testing.assert_array_equal(perm, r_perm, err_msg=f"{what}: perm")
    _check_h(hq, hsf, r_hq, r_hsf, what)
    T, k = inp["topk_ids"].shape
    exact = _exact_tokens(hq, hsf, r_hq, r_hsf, perm, T, k)
    # the GPU's intermediate in pair order (all ids are valid here)
    hq_p = np.empty_like(hq)
    hsf_p = np.empty_like(hsf)
    hq_p[perm] = hq
    hsf_p[perm] = hsf
    cond = _gemm2_on(oracle, hq_p, hsf_p, i32(inp["topk_ids"]).ravel(), u8(inp["w2"]),
                     u8(inp["w2_sf"]), f32(inp["w2_g"]), f32(inp["topk_w"]), inp["a2_g"])
    _compare_out(out, r_out, cond, exact, f"{what}: output")


def test_nvfp4_fused_tiny(oracle):
    cfg = synth.MoEConfig("nv_tiny", 16, 256, 256, 4, 2)
    _check(oracle, synth.make_nvfp4_moe_inputs(cfg, seed=0, device="cuda"), "tiny")


@pytest.mark.parametrize("T,H,I,E,k,routing", [
    (33, 256, 256, 5, 3, "normal"),     # ragged tiles, odd group sizes
    (200, 512, 512, 16, 4, "zipf"),     # skewed groups
    (300, 768, 256, 8, 2, "normal"),    # GEMM2 with three 256-column tiles
    (20, 8192, 256, 4, 2, "normal"),    # I < H/16: x's scales scattered K-block-major directly
])
def test_nvfp4_fused_shapes(oracle, T, H, I, E, k, routing):
    cfg = synth.MoEConfig("nv_case", T, H, I, E, k, routing)
    _check(oracle, synth.make_nvfp4_moe_inputs(cfg, seed=T, device="cuda"), f"T={T}")


def test_nvfp4_fused_zero_tokens_and_bad_args():
    cfg = synth.MoEConfig("nv_zero", 0, 256, 256, 4, 2)
    inp = synth.make_nvfp4_moe_inputs(cfg, seed=0, device="cuda")
    out = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(moe.moe_workspace_size(0, 256, 256, 4, 2), dtype=torch.uint8, device="cuda")
    a13, a2 = _alphas(inp)
    args = (inp["x"], inp["topk_ids"], inp["topk_w"], inp["w13_packed"],
            _tile(inp["w13_sf"], (4 * 512, 16)), a13, inp["w2_packed"],
            _tile(inp["w2_sf"], (4 * 256, 16)), a2)
    assert moe.moe_nvfp4_fused(*args, inp["a1_g"], inp["a2_g"], out, ws) == 0
    # a global scale must be positive; I must be a multiple of 256
    assert moe.moe_nvfp4_fused(*args, 0.0, inp["a2_g"], out, ws, check=False) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_nvfp4_fused(*args, inp["a1_g"], inp["a2_g"], out, ws, dims=(0, 256, 128, 4, 2),
                               check=False) == moe.MOE_ERR_INVALID_ARG


def _compact(inp, tokens):
    """Host copies of only the experts the listed tokens use, with their
    routing renumbered into the compact list."""
    dev = inp["topk_ids"].device
    sel = torch.as_tensor(tokens, device=dev)
    ids = inp["topk_ids"][sel]
    used = torch.unique(ids).to(torch.long)
    remap = torch.full((inp["w13_packed"].shape[0],), -1, dtype=torch.int32, device=dev)
    remap[used] = torch.arange(len(used), dtype=torch.int32, device=dev)
    return dict(x=bf16_bits(inp["x"][sel]), topk_ids=i32(remap[ids]), topk_w=f32(inp["topk_w"][sel]),
                w13=u8(inp["w13"][used]), w13_sf=u8(inp["w13_sf"][used]), w13_g=f32(inp["w13_g"][used]),
                w2=u8(inp["w2"][used]), w2_sf=u8(inp["w2_sf"][used]), w2_g=f32(inp["w2_g"][used]))


def _check_sampled(oracle, inp, tokens, what):
    out, m_indptr, perm, hq, hsf = _run(inp)
    E = inp["w13_packed"].shape[0]
    m_o, p_o, i_o, _ = oracle.route_permute(i32(inp["topk_ids"]), E)
    np.testing.assert_array_equal(m_indptr, m_o, err_msg=what)
    np.testing.assert_array_equal(perm, p_o, err_msg=what)
    sub = _compact(inp, tokens)
    out_o, hq_o, hsf_o = oracle.moe_nvfp4_tokens(
        sub["x"], sub["topk_ids"], sub["topk_w"], sub["w13"], sub["w13_sf"], sub["w13_g"],
        sub["w2"], sub["w2_sf"], sub["w2_g"], inp["a1_g"], inp["a2_g"],
        np.arange(len(tokens), dtype=np.int32), want_h=True)
    k = inp["topk_ids"].shape[1]
    rows = np.array([[i_o[t * k + j] for j in range(k)] for t in tokens]).ravel()
    r_hq, r_hsf = hq_o.reshape(len(rows), -1), hsf_o.reshape(len(rows), -1)
    _check_h(hq[rows], hsf[rows], r_hq, r_hsf, what)
    # sampled row n holds slot n % k of sampled token n // k
    exact = _exact_tokens(hq[rows], hsf[rows], r_hq, r_hsf, np.arange(len(rows)), len(tokens), k)
    cond = _gemm2_on(oracle, hq[rows], hsf[rows], sub["topk_ids"].ravel(), sub["w2"], sub["w2_sf"],
                     sub["w2_g"], sub["topk_w"], inp["a2_g"])
    _compare_out(out[tokens], out_o, cond, exact, what + " output")


def test_nvfp4_fused_decode_full_size_sampled(oracle):
    inp = synth.make_nvfp4_moe_inputs(synth.CONFIGS["decode"], seed=0, device="cuda")
    _check_sampled(oracle, inp, [0, 17, 42, 63], "nvfp4 decode")
    del inp
    torch.cuda.empty_cache()


def test_nvfp4_fused_prefill_full_size_sampled(oracle):
    inp = synth.make_nvfp4_moe_inputs(synth.CONFIGS["prefill"], seed=0, device="cuda")
    ids = inp["topk_ids"]
    counts = torch.bincount(ids.flatten().long(), minlength=256)
    big = int(torch.argmax(counts))
    nz = torch.nonzero(counts).flatten()
    small = int(nz[torch.argmin(counts[nz])])
    t_big = int(torch.nonzero((ids == big).any(1)).flatten()[0])
    t_small = int(torch.nonzero((ids == small).any(1)).flatten()[0])
    _check_sampled(oracle, inp, sorted({0, t_big, t_small, 8191}), "nvfp4 prefill")
    del inp
    torch.cuda.empty_cache()
