"""Parity of the MXFP8 grouped GEMM (block-scaled tensor core path) against
the oracle's MXFP8 GEMM, called through the C ABI.  B200 only."""
import numpy as np
import pytest
import torch

import synth
import fp8_block_scaled_route_b200 as moe

pytestmark = pytest.mark.gpu


def _tiled(sf_rowmajor):
    rows = sf_rowmajor.numel() // sf_rowmajor.shape[-1]
    flat = sf_rowmajor.reshape(rows, sf_rowmajor.shape[-1]).contiguous()
    tiled = torch.empty_like(flat)
    moe.mxfp8_tile_scales(flat, tiled)
    return tiled


def _mn(a_sf):
    """[R, K/32] -> [K/128, R, 4] (the four scales of a K block together)."""
    R, nsf = a_sf.shape
    return a_sf.view(R, nsf // 4, 4).permute(1, 0, 2).contiguous()


def _run(inp, is_gated, a_mn=False):
    a, b = inp["a"], inp["b"]
    R = a.shape[0]
    E, N, _ = b.shape
    out = torch.full((R, N // 2 if is_gated else N), float("nan"), dtype=torch.bfloat16,
                     device=a.device)
    a_sf = _mn(inp["a_sf"]) if a_mn else inp["a_sf"]
    moe.mxfp8_moe_gemm(a, b, a_sf, _tiled(inp["b_sf"]), inp["m_indptr"], out, is_gated,
                       "MN" if a_mn else "K")
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(None) == 0
    return out.cpu()


def _oracle(oracle, inp, is_gated):
    h = {k: v.cpu() for k, v in inp.items()}
    bits = oracle.mx_gemm_bf16(h["a"].view(torch.uint8).numpy(), h["a_sf"].numpy(),
                               h["b"].view(torch.uint8).numpy(), h["b_sf"].numpy(),
                               h["m_indptr"].numpy(), is_gated)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


def _compare(got, ref, rows):
    g = got[:rows].float()
    r = ref[:rows].float()
    assert torch.isfinite(g).all()
    rms = r.pow(2).mean().sqrt().item() + 1e-30
    diff = (g - r).abs()
    # both sides round an fp32 value to bf16; the fp32 values differ only by
    # the order of the tensor core's accumulation (~1e-6 relative)
    bound = r.abs() * 2.0 ** -7 + 1e-3 * rms
    bad = (diff > bound).sum().item()
    assert bad == 0, f"{bad} elements off; max diff {diff.max().item()} rms {rms}"
    rel = ((g - r).pow(2).sum() / r.pow(2).sum().clamp_min(1e-30)).sqrt().item()
    assert rel <= 2e-3, rel


def test_mx_gemm_exact_small_integers(oracle):
    """Integer operands with unit scales: the fp32 accumulator is exact, so the
    bf16 outputs are bit-identical to the oracle's."""
    torch.manual_seed(0)
    R, N, K, E = 300, 384, 512, 3
    table = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float()
    ints = {int(v): c for c, v in enumerate(table.tolist()) if v == v and v == int(v) and abs(v) <= 4}
    lut = torch.tensor([ints[v] for v in range(-4, 5)], dtype=torch.uint8)
    a = lut[torch.randint(0, 9, (R, K))].view(torch.float8_e4m3fn)
    b = lut[torch.randint(0, 9, (E, N, K))].view(torch.float8_e4m3fn)
    inp = dict(a=a, b=b, a_sf=torch.full((R, K // 32), 127, dtype=torch.uint8),
               b_sf=torch.full((E, N, K // 32), 127, dtype=torch.uint8),
               m_indptr=torch.tensor([0, 77, 77, 290], dtype=torch.int32))
    dev = {k: v.cuda() for k, v in inp.items()}
    got = _run(dev, False)
    ref = _oracle(oracle, inp, False)
    rows = 290
    assert torch.equal(got[:rows].view(torch.int16), ref[:rows].view(torch.int16))
    assert torch.isnan(got[rows:].float()).all()  # rows outside every group untouched


@pytest.mark.parametrize("R,N,K,E,gated,sizes", [
    (256, 256, 128, 1, False, None),          # one tile, one K block
    (200, 512, 384, 4, True, None),           # gated, ragged groups
    (517, 384, 256, 5, False, [0, 130, 1, 0, 386]),  # odd number of 128-column blocks, empty experts
    (1000, 1024, 1024, 8, True, None),
    (640, 512, 7168, 3, False, None),         # 56 K blocks
    (64, 512, 256, 8, True, None),            # small groups: 32-token swapped tiles
    (100, 384, 512, 5, False, [0, 40, 1, 0, 59]),  # swapped, groups over one token tile
    (48, 256, 7168, 6, False, None),          # swapped, 56 K blocks
])
def test_mx_gemm_random(oracle, R, N, K, E, gated, sizes):
    inp = synth.make_mx_gemm_inputs(R, N, K, E, seed=R + K, group_sizes=sizes)
    rows = int(inp["m_indptr"][-1])
    dev = {k: v.cuda() for k, v in inp.items()}
    ref = _oracle(oracle, inp, gated)
    _compare(_run(dev, gated), ref, rows)
    _compare(_run(dev, gated, a_mn=True), ref, rows)


def test_mx_gemm_exact_small_integers_swapped(oracle):
    """As above on the swapped (32-token) tile: groups of at most 32 rows."""
    torch.manual_seed(1)
    R, N, K, E = 60, 256, 256, 3
    table = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float()
    ints = {int(v): c for c, v in enumerate(table.tolist()) if v == v and v == int(v) and abs(v) <= 4}
    lut = torch.tensor([ints[v] for v in range(-4, 5)], dtype=torch.uint8)
    inp = dict(a=lut[torch.randint(0, 9, (R, K))].view(torch.float8_e4m3fn),
               b=lut[torch.randint(0, 9, (E, N, K))].view(torch.float8_e4m3fn),
               a_sf=torch.full((R, K // 32), 127, dtype=torch.uint8),
               b_sf=torch.full((E, N, K // 32), 127, dtype=torch.uint8),
               m_indptr=torch.tensor([0, 20, 21, 57], dtype=torch.int32))
    got = _run({k: v.cuda() for k, v in inp.items()}, False)
    ref = _oracle(oracle, inp, False)
    assert torch.equal(got[:57].view(torch.int16), ref[:57].view(torch.int16))
    assert torch.isnan(got[57:].float()).all()


def test_mx_gemm_scale_placement(oracle):
    """One 32-wide scale step per block of one row of A and one row of B, set
    far from the others: a scale read from the wrong row, column or K step
    shows up as an error of 2^8 on the touched outputs."""
    R, N, K, E = 256, 256, 256, 1
    inp = synth.make_mx_gemm_inputs(R, N, K, E, seed=7, group_sizes=[R], spread=0)
    inp["a_sf"][37, 5] += 8
    inp["b_sf"][0, 200, 2] += 8
    ref = _oracle(oracle, inp, False)
    for a_mn in (False, True):
        got = _run({k: v.cuda() for k, v in inp.items()}, False, a_mn)
        _compare(got, ref, R)


def test_mx_tile_scales_layout():
    """Tiled byte (r % 32) * 16 + ((r / 32) % 4) * 4 + j of block (r / 128, kb)
    = row-major scale [r, 4 kb + j]; bit-exact."""
    rows, K = 384, 512
    rm = torch.randint(0, 256, (rows, K // 32), dtype=torch.uint8)
    got = _tiled(rm.cuda()).cpu().numpy().reshape(rows // 128, K // 128, 512)
    r = np.arange(rows)[:, None]
    j = np.arange(K // 32)[None, :]
    kb, jj = j // 4, j % 4
    ref = np.zeros_like(got)
    ref[r // 128, kb, (r % 32) * 16 + ((r // 32) % 4) * 4 + jj] = rm.numpy()
    np.testing.assert_array_equal(got, ref)


def test_mx_gemm_empty_and_bad_args():
    a = torch.zeros(0, 128, dtype=torch.float8_e4m3fn, device="cuda")
    b = torch.zeros(2, 256, 128, dtype=torch.float8_e4m3fn, device="cuda")
    a_sf = torch.zeros(0, 4, dtype=torch.uint8, device="cuda")
    b_sf = torch.zeros(2, 256, 4, dtype=torch.uint8, device="cuda")
    m = torch.zeros(3, dtype=torch.int32, device="cuda")
    out = torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda")
    assert moe.mxfp8_moe_gemm(a, b, a_sf, b_sf, m, out, False) == 0
    # K not a multiple of 128
    assert moe.mxfp8_moe_gemm(a, b, a_sf, b_sf, m, out, False, dims=(0, 256, 96, 2),
                              check=False) == moe.MOE_ERR_INVALID_ARG
