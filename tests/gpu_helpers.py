"""Shared helpers of the GPU parity tests: run the CUDA path through the C
ABI, convert tensors for the oracle and compare results with the tolerances
the layer's acceptance rules fix.

Tolerances (one place, used by every GPU test):
  * routing tables, m_indptr and permutations: bit-exact.
  * FP8 codes of the requantised intermediate and of SwiGLU+MXFP8: at least
    99.9% identical; every other code adjacent (neighbouring representable
    value, same sign) to the oracle's.
  * fp32 block scales of the intermediate: relative difference <= 2^-20.
    Both sides take amax/448 with an IEEE divide of the same fp32 values up
    to the GEMM's accumulation order (56 block partials of up to 128 exact
    products each, promoted in a different order) and the kernel's SiLU
    (hardware exp2 and reciprocal, about 2 ulp): amax moves by a few fp32
    ulps.  The largest difference over every GPU test is 6.8e-7 (0.71 of
    the bound).
  * final bf16 output: relative L2 error <= 1e-2 and max abs error
    <= 2e-2 * rms(reference).
"""
from __future__ import annotations

import numpy as np
import torch

import fp8_block_scaled_route_b200 as moe

CODE_MATCH_MIN = 0.999
SCALE_RTOL = 2.0 ** -20
OUT_REL_L2 = 1e-2
OUT_MAX_ABS_RMS = 2e-2

# Worst values seen by the comparisons of this test session (written out by
# tests/conftest.py when MOE_PARITY_STATS names a file).
STATS = {"scale_rel_max": 0.0, "code_match_min": 1.0, "out_rel_l2_max": 0.0,
         "out_max_abs_rms_max": 0.0, "calls": 0}

# Guard bytes after every output buffer the helpers hand to the library: any
# write past the end of a buffer changes them.
GUARD_BYTES = 4096
GUARD_FILL = 0xA5


def guarded_empty(shape, dtype, device, fill=None):
    """A tensor of `shape` at the start of a larger buffer whose tail
    (GUARD_BYTES) holds GUARD_FILL; returns (tensor, guard view)."""
    n = 1
    for d in shape:
        n *= int(d)
    esize = torch.empty((), dtype=dtype).element_size()
    raw = torch.empty(n * esize + GUARD_BYTES, dtype=torch.uint8, device=device)
    raw[n * esize:].fill_(GUARD_FILL)
    t = raw[:n * esize].view(dtype).view(*shape)
    if fill is not None:
        t.fill_(fill)
    return t, raw[n * esize:]


def check_guards(guards: dict, what: str):
    for name, g in guards.items():
        bad = int((g != GUARD_FILL).sum())
        assert bad == 0, f"{what}: {bad} guard bytes after {name} were overwritten"


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16) \
        .to(torch.float64).numpy()


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.uint8).numpy()


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().to(torch.float32).numpy()


def i32(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().to(torch.int32).numpy()


# rank of every E4M3 code in signed value order (+0 and -0 share a rank)
def _code_rank():
    vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    order = np.unique(vals[~np.isnan(vals)])
    rank = np.full(256, -10**6, np.int64)
    for c in range(256):
        if not np.isnan(vals[c]):
            rank[c] = int(np.searchsorted(order, vals[c]))
    return rank


CODE_RANK = _code_rank()


def compare_codes(gpu: np.ndarray, ref: np.ndarray, what: str):
    gpu = np.asarray(gpu, np.uint8).ravel()
    ref = np.asarray(ref, np.uint8).ravel()
    assert gpu.shape == ref.shape, what
    if gpu.size == 0:
        return 1.0
    same = gpu == ref
    frac = float(same.mean())
    STATS["code_match_min"] = min(STATS["code_match_min"], frac)
    dist = np.abs(CODE_RANK[gpu] - CODE_RANK[ref])
    assert frac >= CODE_MATCH_MIN, f"{what}: only {frac:.5f} of codes identical"
    assert int(dist.max()) <= 1, f"{what}: a code differs by {int(dist.max())} steps"
    return frac


def compare_scales(gpu: np.ndarray, ref: np.ndarray, what: str, rtol: float = SCALE_RTOL):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    rel = np.abs(gpu - ref) / np.maximum(np.abs(ref), 1e-30)
    STATS["scale_rel_max"] = max(STATS["scale_rel_max"], float(rel.max(initial=0.0)))
    assert float(rel.max(initial=0.0)) <= rtol, f"{what}: scale rel diff {rel.max():.3e}"


def compare_out(gpu_bits: np.ndarray, ref_bits: np.ndarray, what: str):
    g = bits_to_f64(gpu_bits)
    r = bits_to_f64(ref_bits)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    if rms == 0.0:
        assert np.array_equal(g, r), what
        return 0.0, 0.0
    rel_l2 = float(np.linalg.norm(g - r) / np.linalg.norm(r))
    max_abs = float(np.abs(g - r).max() / rms)
    STATS["out_rel_l2_max"] = max(STATS["out_rel_l2_max"], rel_l2)
    STATS["out_max_abs_rms_max"] = max(STATS["out_max_abs_rms_max"], max_abs)
    STATS["calls"] += 1
    assert rel_l2 <= OUT_REL_L2, f"{what}: relative L2 {rel_l2:.3e}"
    assert max_abs <= OUT_MAX_ABS_RMS, f"{what}: max abs {max_abs:.3e} x rms"
    return rel_l2, max_abs


def oracle_args(inp: dict):
    return (bf16_bits(inp["x"]), i32(inp["topk_ids"]), f32(inp["topk_w"]), u8(inp["w13"]),
            f32(inp["w13_scale"]), u8(inp["w2"]), f32(inp["w2_scale"]))


def run_fused(inp: dict, debug: bool = True):
    """Runs moe_fp8_fused(_debug) on device tensors; returns host arrays.
    The workspace and every output buffer are followed by guard bytes that
    are checked after the call."""
    x = inp["x"]
    T, H = x.shape
    E, I2, _ = inp["w13"].shape
    I = I2 // 2
    k = inp["topk_ids"].shape[1]
    R = T * k
    dev = x.device
    guards = {}
    ws, guards["ws"] = guarded_empty((moe.moe_workspace_size(T, H, I, E, k),), torch.uint8, dev)
    out, guards["out"] = guarded_empty((T, H), torch.bfloat16, dev)
    res = {}
    if debug:
        m_indptr, guards["m_indptr"] = guarded_empty((E + 1,), torch.int32, dev)
        perm, guards["perm"] = guarded_empty((max(R, 1),), torch.int32, dev)
        hq, guards["hq"] = guarded_empty((max(R, 1), I), torch.uint8, dev)
        hs, guards["hs"] = guarded_empty((I // 128, max(R, 1)), torch.float32, dev)
        moe.moe_fp8_fused_debug(x, inp["topk_ids"], inp["topk_w"], inp["w13"], inp["w13_scale"],
                                inp["w2"], inp["w2_scale"], out, ws, m_indptr, perm, hq, hs,
                                ws_bytes=moe.moe_workspace_size(T, H, I, E, k))
        st = moe.moe_get_device_status(ws)
        res.update(m_indptr=i32(m_indptr), perm=i32(perm)[:R], hq=u8(hq)[:R],
                   hs=f32(hs)[:, :R].T.copy())
    else:
        moe.moe_fp8_fused(x, inp["topk_ids"], inp["topk_w"], inp["w13"], inp["w13_scale"],
                          inp["w2"], inp["w2_scale"], out, ws,
                          ws_bytes=moe.moe_workspace_size(T, H, I, E, k))
        st = moe.moe_get_device_status(ws)
    check_guards(guards, "fused layer")
    res["status"] = st
    res["out"] = bf16_bits(out)
    return res
