"""Parity of the NVFP4 grouped GEMM (packed E2M1 operands, E4M3 scales per 16
K elements, per-expert alpha = 1 / (g_a g_b[e])) against the oracle's NVFP4
GEMM, called through the C ABI.  B200 only."""
import numpy as np
import pytest
import torch

import synth
import fp8_block_scaled_route_b200 as moe

pytestmark = pytest.mark.gpu


def _tiled(sf_rowmajor):
    rows = sf_rowmajor.numel() // sf_rowmajor.shape[-1]
    flat = sf_rowmajor.reshape(rows, sf_rowmajor.shape[-1]).contiguous().view(torch.uint8)
    tiled = torch.empty_like(flat)
    moe.nvfp4_tile_scales(flat, tiled)
    return tiled


def _alpha(inp):
    return (1.0 / (inp["ga"] * inp["gb"].double())).float()


def _mn(a_sf):
    """[R, K/16] -> [K/64, R, 4] (the four scales of a 64-wide K block together)."""
    R, nsf = a_sf.shape
    return a_sf.view(R, nsf // 4, 4).permute(1, 0, 2).contiguous()


def _run(inp, is_gated, a_mn=False):
    a, b = inp["a_packed"], inp["b_packed"]
    R = a.shape[0]
    E, N, _ = b.shape
    out = torch.full((R, N // 2 if is_gated else N), float("nan"), dtype=torch.bfloat16,
                     device=a.device)
    a_sf = inp["a_sf"].view(torch.uint8)
    moe.nvfp4_moe_gemm(a, b, _mn(a_sf) if a_mn else a_sf, _tiled(inp["b_sf"]),
                       _alpha(inp).to(a.device), inp["m_indptr"], out, is_gated,
                       "MN" if a_mn else "K")
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(None) == 0
    return out.cpu()


def _oracle(oracle, inp, is_gated):
    h = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in inp.items()}
    bits = oracle.nvfp4_gemm_bf16(h["a"].numpy(), h["a_sf"].view(torch.uint8).numpy(), float(h["ga"]),
                                  h["b"].numpy(), h["b_sf"].view(torch.uint8).numpy(),
                                  h["gb"].numpy(), h["m_indptr"].numpy(), is_gated)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


def _compare(got, ref, rows):
    g = got[:rows].float()
    r = ref[:rows].float()
    assert torch.isfinite(g).all()
    rms = r.pow(2).mean().sqrt().item() + 1e-30
    diff = (g - r).abs()
    # both sides round an fp32 value to bf16; the fp32 values differ by the
    # order of the tensor core's accumulation and by alpha being an fp32
    # reciprocal (~1e-6 relative)
    bound = r.abs() * 2.0 ** -7 + 1e-3 * rms
    bad = (diff > bound).sum().item()
    assert bad == 0, f"{bad} elements off; max diff {diff.max().item()} rms {rms}"
    rel = ((g - r).pow(2).sum() / r.pow(2).sum().clamp_min(1e-30)).sqrt().item()
    assert rel <= 2e-3, rel


def _exact_inputs(R, N, K, E, sizes, seed):
    """Random E2M1 codes, unit block scales (E4M3 1.0 = 0x38), unit global
    scales: every product is a multiple of 0.25 and every partial sum is exact
    in fp32, so both sides round the same value to bf16."""
    g = torch.Generator().manual_seed(seed)
    a = torch.randint(0, 16, (R, K), generator=g, dtype=torch.uint8)
    b = torch.randint(0, 16, (E, N, K), generator=g, dtype=torch.uint8)
    m = torch.zeros(E + 1, dtype=torch.int32)
    m[1:] = torch.cumsum(torch.tensor(sizes), 0).to(torch.int32)
    return dict(a=a, a_packed=synth.pack_e2m1(a), b=b,
                b_packed=synth.pack_e2m1(b.view(E * N, K)).view(E, N, K // 2),
                a_sf=torch.full((R, K // 16), 0x38, dtype=torch.uint8),
                b_sf=torch.full((E, N, K // 16), 0x38, dtype=torch.uint8),
                ga=1.0, gb=torch.ones(E), m_indptr=m)


def _cuda(inp):
    return {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}


@pytest.mark.parametrize("gated", [False, True])
def test_nvfp4_gemm_exact_small_values(oracle, gated):
    R, N, K, E = 300, 512, 512, 3
    inp = _exact_inputs(R, N, K, E, [77, 0, 213], seed=0)
    got = _run(_cuda(inp), gated)
    ref = _oracle(oracle, inp, gated)
    rows = 290
    if gated:  # silu: both sides in fp32, different exp implementations
        _compare(got, ref, rows)
    else:
        assert torch.equal(got[:rows].view(torch.int16), ref[:rows].view(torch.int16))
    assert torch.isnan(got[rows:].float()).all()  # rows outside every group untouched


@pytest.mark.parametrize("R,N,K,E,gated,sizes", [
    (256, 256, 256, 1, False, None),          # one tile, one K block
    (200, 512, 512, 4, True, None),           # gated, ragged groups
    (517, 384, 256, 5, False, [0, 130, 1, 0, 386]),  # odd number of 128-column blocks, empty experts
    (1000, 1024, 1024, 8, True, None),
    (640, 512, 7168, 3, False, None),         # 28 K blocks
    (64, 512, 2048, 8, True, None),           # small groups
    (130, 128, 256, 64, False, None),         # one 128-column block, most experts empty
])
def test_nvfp4_gemm_random(oracle, R, N, K, E, gated, sizes):
    inp = synth.make_nvfp4_gemm_inputs(R, N, K, E, seed=R + K, group_sizes=sizes)
    rows = int(inp["m_indptr"][-1])
    ref = _oracle(oracle, inp, gated)
    dev = _cuda(inp)
    _compare(_run(dev, gated), ref, rows)
    _compare(_run(dev, gated, a_mn=True), ref, rows)


def test_nvfp4_gemm_scale_placement(oracle):
    """One 16-wide block scale of one row of A and one of B set far above the
    others (E4M3 16.0): a scale read from the wrong row, column or K block
    shows up as a large error on the touched outputs."""
    R, N, K, E = 256, 256, 512, 1
    inp = synth.make_nvfp4_gemm_inputs(R, N, K, E, seed=7, group_sizes=[R])
    a_sf = inp["a_sf"].view(torch.uint8)
    b_sf = inp["b_sf"].view(torch.uint8)
    a_sf[37, 21] = 0x58
    b_sf[0, 200, 6] = 0x58
    ref = _oracle(oracle, inp, False)
    for a_mn in (False, True):
        _compare(_run(_cuda(inp), False, a_mn), ref, R)


def test_nvfp4_tile_scales_layout():
    """Tiled byte (r % 32) * 16 + ((r / 32) % 4) * 4 + j of atom (r / 128, kb)
    = row-major scale [r, 4 kb + j] (one atom per 64 K elements); bit-exact."""
    rows, K = 384, 512
    rm = torch.randint(0, 256, (rows, K // 16), dtype=torch.uint8)
    got = _tiled(rm.cuda()).cpu().numpy().reshape(rows // 128, K // 64, 512)
    r = np.arange(rows)[:, None]
    j = np.arange(K // 16)[None, :]
    kb, jj = j // 4, j % 4
    ref = np.zeros_like(got)
    ref[r // 128, kb, (r % 32) * 16 + ((r // 32) % 4) * 4 + jj] = rm.numpy()
    np.testing.assert_array_equal(got, ref)


def test_nvfp4_gemm_empty_and_bad_args():
    a = torch.zeros(0, 128, dtype=torch.uint8, device="cuda")
    b = torch.zeros(2, 256, 128, dtype=torch.uint8, device="cuda")
    a_sf = torch.zeros(0, 16, dtype=torch.uint8, device="cuda")
    b_sf = torch.zeros(2 * 256 * 16, dtype=torch.uint8, device="cuda")
    alpha = torch.ones(2, device="cuda")
    m = torch.zeros(3, dtype=torch.int32, device="cuda")
    out = torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda")
    assert moe.nvfp4_moe_gemm(a, b, a_sf, b_sf, alpha, m, out, False) == 0
    # K not a multiple of 256
    assert moe.nvfp4_moe_gemm(a, b, a_sf, b_sf, alpha, m, out, False, dims=(0, 256, 192, 2),
                              check=False) == moe.MOE_ERR_INVALID_ARG
    assert moe.nvfp4_moe_gemm(a, b, a_sf, b_sf, alpha, m, out, False, 2,
                              check=False) == moe.MOE_ERR_INVALID_ARG
