"""Seeded synthetic inputs for the fused W8A8 MoE layer and the standalone
SwiGLU+MXFP8 op.

This module is shared by the CUDA path's tests/benchmark and by the CPU
oracle's tests.  It holds none of the layer's own arithmetic: it draws router
logits, picks top-k experts and softmax weights (the router is the step
*before* the layer; its outputs are the layer's inputs), draws bf16
activations, and produces FP8 E4M3 weights with fp32 128x128 block scales by
torch's own fp32 -> float8_e4m3fn cast (weights reach the layer already
quantised, so weight quantisation is input preparation, not a layer step).

Workloads (sizes from the method's pages' MoE settings):
  tiny     T=16,   H=256,  I=128,  E=4,   top-2, logits ~N(0,1)
  mid      T=512,  H=2048, I=768,  E=128, top-8, logits ~N(0,1)
  decode   T=64,   H=7168, I=2048, E=256, top-8, logits ~N(0,1)
  prefill  T=8192, H=7168, I=2048, E=256, top-8, logits ~N(0,1) plus a
           per-expert bias -1.2*ln(rank), ranks a seeded permutation of 1..E
           (Zipf(1.2)-shaped popularity)
Weights: w13 [E,2I,H] ~ N(0, 1/sqrt(H)), w2 [E,H,I] ~ N(0, 1/sqrt(I)).
Draw order for one seed: logits, (Zipf ranks), x, then w13 and w2 expert by
expert.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    routing: str = "normal"   # "normal" or "zipf"

    @property
    def R(self) -> int:
        return self.T * self.k


CONFIGS = {
    "tiny": MoEConfig("tiny", 16, 256, 128, 4, 2),
    "mid": MoEConfig("mid", 512, 2048, 768, 128, 8),
    "decode": MoEConfig("decode", 64, 7168, 2048, 256, 8),
    "prefill": MoEConfig("prefill", 8192, 7168, 2048, 256, 8, "zipf"),
}

SWIGLU_SHAPES = ((128, 128), (1024, 2048), (8192, 7168))
ZIPF_S = 1.2


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def quantize_weight_blocks(w: torch.Tensor):
    """[N, K] fp32 -> (float8_e4m3fn [N, K], fp32 scales [N/128, K/128]) with
    scale = blockwise amax / 448 and torch's float8 cast of w / scale."""
    N, K = w.shape
    blocks = w.view(N // 128, 128, K // 128, 128)
    amax = blocks.abs().amax(dim=(1, 3))
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    q = (blocks / scale[:, None, :, None]).to(torch.float8_e4m3fn)
    return q.view(N, K), scale.contiguous()


def _expert_weights(E: int, N: int, K: int, sigma: float, g, device):
    q = torch.empty(E, N, K, dtype=torch.float8_e4m3fn, device=device)
    s = torch.empty(E, N // 128, K // 128, dtype=torch.float32, device=device)
    for e in range(E):
        w = torch.randn(N, K, generator=g, device=device, dtype=torch.float32) * sigma
        q[e], s[e] = quantize_weight_blocks(w)
    return q, s


def make_routing(T: int, E: int, k: int, routing: str, g, device):
    logits = torch.randn(T, E, generator=g, device=device, dtype=torch.float32)
    if routing == "zipf":
        ranks = torch.randperm(E, generator=g, device=device).to(torch.float32) + 1.0
        logits = logits + (-ZIPF_S) * torch.log(ranks)[None, :]
    elif routing != "normal":
        raise ValueError(routing)
    top_v, top_i = torch.topk(logits, k, dim=1, largest=True, sorted=True)
    topk_w = torch.softmax(top_v, dim=1).to(torch.float32)
    return top_i.to(torch.int32).contiguous(), topk_w.contiguous()


def make_moe_inputs(cfg: MoEConfig, seed: int = 0, device="cpu", weights: bool = True):
    """Returns a dict of tensors on `device`: x (bf16 [T,H]), topk_ids (int32
    [T,k]), topk_w (fp32 [T,k]), w13 (fp8 [E,2I,H]), w13_scale (fp32
    [E,2I/128,H/128]), w2 (fp8 [E,H,I]), w2_scale (fp32 [E,H/128,I/128])."""
    g = _gen(seed, device)
    topk_ids, topk_w = make_routing(cfg.T, cfg.E, cfg.k, cfg.routing, g, device)
    x = torch.randn(cfg.T, cfg.H, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    out = dict(x=x, topk_ids=topk_ids, topk_w=topk_w)
    if weights:
        out["w13"], out["w13_scale"] = _expert_weights(cfg.E, 2 * cfg.I, cfg.H,
                                                       1.0 / math.sqrt(cfg.H), g, device)
        out["w2"], out["w2_scale"] = _expert_weights(cfg.E, cfg.H, cfg.I,
                                                     1.0 / math.sqrt(cfg.I), g, device)
    return out


def _host(t: torch.Tensor, dtype) -> "np.ndarray":
    return t.detach().contiguous().cpu().view(dtype).numpy()


def compact_experts(inp: dict, tokens):
    """Host copies (numpy) of the listed tokens' inputs and of only the
    experts they use, with their routing renumbered into that compact expert
    list: x as bf16 bits, topk_ids int32, topk_w fp32, weights as FP8 codes and
    fp32 scales.  Lets a per-token check of a full-size workload move a few
    experts to the host instead of all of them.  Ids outside [0, E) are kept
    as they are."""
    E = inp["w13"].shape[0]
    sel = torch.as_tensor(tokens, device=inp["topk_ids"].device)
    ids = inp["topk_ids"][sel]
    valid = (ids >= 0) & (ids < E)
    used = torch.unique(ids[valid]).to(torch.long)
    remap = torch.full((E,), -1, dtype=torch.int32, device=ids.device)
    remap[used] = torch.arange(len(used), dtype=torch.int32, device=ids.device)
    local = torch.where(valid, remap[ids.clamp(0, E - 1)], ids)
    return dict(
        x=_host(inp["x"][sel.to(inp["x"].device)], torch.int16).view(np.uint16),
        topk_ids=_host(local, torch.int32), topk_w=_host(inp["topk_w"][sel], torch.float32),
        w13=_host(inp["w13"][used], torch.uint8), w13_scale=_host(inp["w13_scale"][used], torch.float32),
        w2=_host(inp["w2"][used], torch.uint8), w2_scale=_host(inp["w2_scale"][used], torch.float32))


def make_swiglu_input(M: int, K: int, variant: str = "normal", seed: int = 0, device="cpu"):
    """bf16 [M, 2K] (gate | up halves) ~ N(0,1); variant "block_scaled"
    multiplies each 32-column block by 2^u, u ~ U{-8..8} (integers)."""
    g = _gen(seed, device)
    x = torch.randn(M, 2 * K, generator=g, device=device, dtype=torch.float32)
    if variant == "block_scaled":
        u = torch.randint(-8, 9, (M, 2 * K // 32), generator=g, device=device).to(torch.float32)
        x = (x.view(M, 2 * K // 32, 32) * torch.exp2(u)[:, :, None]).view(M, 2 * K)
    elif variant != "normal":
        raise ValueError(variant)
    return x.to(torch.bfloat16).contiguous()


def make_grouped_gemm_inputs(R: int, N: int, K: int, E: int, seed: int = 0, device="cpu",
                             group_sizes=None):
    """Inputs for the standalone grouped GEMM: activations already quantised
    per row per 128 (drawn as bf16 N(0,1), cast the same way as weights but
    with 1x128 blocks), B [E,N,K] fp8 with 128x128 scales, m_indptr from
    `group_sizes` (default: a seeded multinomial split of R over E)."""
    g = _gen(seed, device)
    if group_sizes is None:
        idx = torch.randint(0, E, (R,), generator=g, device=device)
        group_sizes = torch.bincount(idx, minlength=E)
    group_sizes = torch.as_tensor(group_sizes, device=device, dtype=torch.int64)
    m_indptr = torch.zeros(E + 1, dtype=torch.int32, device=device)
    m_indptr[1:] = torch.cumsum(group_sizes, 0).to(torch.int32)
    R = int(m_indptr[-1])
    a32 = torch.randn(R, K, generator=g, device=device, dtype=torch.float32)
    blocks = a32.view(R, K // 128, 128)
    amax = blocks.abs().amax(dim=2)
    a_scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    a = (blocks / a_scale[:, :, None]).to(torch.float8_e4m3fn).view(R, K)
    b, b_scale = _expert_weights(E, N, K, 1.0 / math.sqrt(K), g, device)
    return dict(a=a.contiguous(), a_scale=a_scale.contiguous(), b=b, b_scale=b_scale,
                m_indptr=m_indptr)


def quantize_mx_rows(x: torch.Tensor):
    """[rows, cols] fp32 -> (float8_e4m3fn [rows, cols], uint8 E8M0 codes
    [rows, cols/32]): per 32 consecutive values the smallest power of two 2^s
    with amax <= 448 * 2^s (code s + 127, all-zero blocks code 0), then
    torch's float8 cast of x / 2^s (exact power-of-two scaling)."""
    rows, cols = x.shape
    blocks = x.view(rows, cols // 32, 32)
    amax = blocks.abs().amax(dim=2).to(torch.float64)
    s = torch.ceil(torch.log2(torch.clamp(amax, min=1e-300) / 448.0))
    s = torch.where(amax > torch.ldexp(torch.full_like(amax, 448.0), s), s + 1, s)
    s = torch.where(amax <= torch.ldexp(torch.full_like(amax, 448.0), s - 1), s - 1, s)
    code = torch.clamp(s + 127, 0, 254)
    code = torch.where(amax > 0, code, torch.zeros_like(code))
    X = torch.ldexp(torch.ones_like(amax), (code - 127).to(torch.int64)).to(torch.float32)
    q = (blocks / X[:, :, None]).to(torch.float8_e4m3fn).view(rows, cols)
    return q.contiguous(), code.to(torch.uint8).contiguous()


def make_mx_gemm_inputs(R: int, N: int, K: int, E: int, seed: int = 0, device="cpu",
                        group_sizes=None, spread: int = 4):
    """Inputs for the MXFP8 grouped GEMM: activations N(0,1) and weights
    N(0, 1/K), each 32-wide K block of a row multiplied by 2^u with u uniform
    in [-spread, spread] (so the scales differ from block to block), then
    quantised to MXFP8 (quantize_mx_rows); m_indptr as in
    make_grouped_gemm_inputs."""
    g = _gen(seed, device)
    if group_sizes is None:
        idx = torch.randint(0, E, (R,), generator=g, device=device)
        group_sizes = torch.bincount(idx, minlength=E)
    group_sizes = torch.as_tensor(group_sizes, device=device, dtype=torch.int64)
    m_indptr = torch.zeros(E + 1, dtype=torch.int32, device=device)
    m_indptr[1:] = torch.cumsum(group_sizes, 0).to(torch.int32)
    R = int(m_indptr[-1])

    def spread_blocks(x):
        u = torch.randint(-spread, spread + 1, (x.shape[0], x.shape[1] // 32), generator=g,
                          device=device).to(torch.float32)
        return (x.view(x.shape[0], -1, 32) * torch.exp2(u)[:, :, None]).view(x.shape)

    a32 = spread_blocks(torch.randn(R, K, generator=g, device=device, dtype=torch.float32))
    a, a_sf = quantize_mx_rows(a32)
    b = torch.empty(E, N, K, dtype=torch.float8_e4m3fn, device=device)
    b_sf = torch.empty(E, N, K // 32, dtype=torch.uint8, device=device)
    for e in range(E):
        w = spread_blocks(torch.randn(N, K, generator=g, device=device, dtype=torch.float32)
                          / math.sqrt(K))
        b[e], b_sf[e] = quantize_mx_rows(w)
    return dict(a=a, a_sf=a_sf, b=b, b_sf=b_sf, m_indptr=m_indptr)


def make_mx_moe_inputs(cfg: MoEConfig, seed: int = 0, device="cpu"):
    """The fused layer's inputs with MXFP8 weights: routing and x as in
    make_moe_inputs; w13 [E,2I,H] and w2 [E,H,I] drawn N(0, 1/fan_in) and
    quantised per row per 32 (quantize_mx_rows); scales row-major
    w13_sf [E,2I,H/32], w2_sf [E,H,I/32]."""
    base = make_moe_inputs(cfg, seed, device, weights=False)
    g = _gen(seed + 7919, device)
    E, H, I = cfg.E, cfg.H, cfg.I
    w13 = torch.empty(E, 2 * I, H, dtype=torch.float8_e4m3fn, device=device)
    w13_sf = torch.empty(E, 2 * I, H // 32, dtype=torch.uint8, device=device)
    w2 = torch.empty(E, H, I, dtype=torch.float8_e4m3fn, device=device)
    w2_sf = torch.empty(E, H, I // 32, dtype=torch.uint8, device=device)
    for e in range(E):
        w13[e], w13_sf[e] = quantize_mx_rows(
            torch.randn(2 * I, H, generator=g, device=device) / math.sqrt(H))
        w2[e], w2_sf[e] = quantize_mx_rows(
            torch.randn(H, I, generator=g, device=device) / math.sqrt(I))
    base.update(w13=w13, w13_sf=w13_sf, w2=w2, w2_sf=w2_sf)
    return base


E2M1_VALUES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def _e2m1_codes(v: torch.Tensor) -> torch.Tensor:
    """Nearest E2M1 code (sign bit 8, magnitude code 0..7), ties to the even
    code, saturating at 6: the magnitude code counts the midpoints between
    neighbouring values that |v| passes (a midpoint below an odd code needs
    |v| strictly above it, one below an even code |v| at or above it)."""
    a = v.abs()
    code = torch.zeros(v.shape, dtype=torch.uint8, device=v.device)
    for i, mid in enumerate((0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)):
        code += ((a > mid) if i % 2 == 0 else (a >= mid)).to(torch.uint8)
    return code | ((v < 0).to(torch.uint8) * 8)


def quantize_nvfp4_rows(x: torch.Tensor, g: float):
    """[rows, cols] fp32, global scale g -> (E2M1 codes [rows, cols] one per
    byte, E4M3 block scales [rows, cols/16] as float8_e4m3fn): per 16 values
    c = E4M3(amax * g / 6) (torch's float8 cast), codes E2M1(x * g / dec(c))."""
    rows, cols = x.shape
    blocks = x.view(rows, cols // 16, 16)
    amax = blocks.abs().amax(dim=2)
    sc = (amax * g / 6.0).to(torch.float8_e4m3fn)
    dec = sc.to(torch.float32)
    scaled = torch.where(dec[:, :, None] > 0, blocks * g / dec[:, :, None].clamp(min=1e-30),
                         torch.zeros_like(blocks))
    return _e2m1_codes(scaled).view(rows, cols), sc.contiguous()


def pack_e2m1(codes: torch.Tensor) -> torch.Tensor:
    """[rows, cols] codes -> [rows, cols/2] bytes, element 2i in the low nibble."""
    c = codes.view(codes.shape[0], -1, 2).to(torch.uint8)
    return (c[..., 0] | (c[..., 1] << 4)).contiguous()


def make_nvfp4_gemm_inputs(R: int, N: int, K: int, E: int, seed: int = 0, device="cpu",
                           group_sizes=None):
    """Inputs for the NVFP4 grouped GEMM: activations N(0,1) and weights
    N(0,1/K), with per-16 magnitudes 2^U{-3..3}; global scales 448*6/amax of
    the activations and of each expert's weights; codes unpacked (one per
    byte, for the oracle) and packed (two per byte)."""
    g = _gen(seed, device)
    if group_sizes is None:
        idx = torch.randint(0, E, (R,), generator=g, device=device)
        group_sizes = torch.bincount(idx, minlength=E)
    group_sizes = torch.as_tensor(group_sizes, device=device, dtype=torch.int64)
    m_indptr = torch.zeros(E + 1, dtype=torch.int32, device=device)
    m_indptr[1:] = torch.cumsum(group_sizes, 0).to(torch.int32)
    R = int(m_indptr[-1])

    def spread(x):
        u = torch.randint(-3, 4, (x.shape[0], x.shape[1] // 16), generator=g, device=device)
        return (x.view(x.shape[0], -1, 16) * torch.exp2(u.float())[:, :, None]).view(x.shape)

    a32 = spread(torch.randn(max(R, 1), K, generator=g, device=device))[:R]
    ga = 448.0 * 6.0 / max(float(a32.abs().max()) if R else 1.0, 1e-30)
    a, a_sf = quantize_nvfp4_rows(a32, ga)
    b = torch.empty(E, N, K, dtype=torch.uint8, device=device)
    b_sf = torch.empty(E, N, K // 16, dtype=torch.float8_e4m3fn, device=device)
    gb = torch.empty(E, dtype=torch.float32, device=device)
    for e in range(E):
        w = spread(torch.randn(N, K, generator=g, device=device) / math.sqrt(K))
        gb[e] = 448.0 * 6.0 / float(w.abs().max())
        b[e], b_sf[e] = quantize_nvfp4_rows(w, float(gb[e]))
    return dict(a=a, a_packed=pack_e2m1(a) if R else a.view(0, K // 2), a_sf=a_sf, ga=ga,
                b=b, b_packed=pack_e2m1(b.view(E * N, K)).view(E, N, K // 2), b_sf=b_sf, gb=gb,
                m_indptr=m_indptr)


# Calibrated global scales of the NVFP4 layer's activations: 448*6 / the
# assumed bound of |x| (8; x ~ N(0,1)) and of |silu(gate) * up| (16).
NVFP4_A1_GSCALE = 448.0 * 6.0 / 8.0
NVFP4_A2_GSCALE = 448.0 * 6.0 / 16.0


def make_nvfp4_moe_inputs(cfg: MoEConfig, seed: int = 0, device="cpu", keep_codes=True):
    """The fused layer's inputs with NVFP4 weights: routing and x as in
    make_moe_inputs; w13 [E,2I,H] and w2 [E,H,I] drawn N(0, 1/fan_in),
    per-expert global scales 448*6/amax, quantised per row per 16
    (quantize_nvfp4_rows).  Returns packed codes (w13_packed [E,2I,H/2],
    w2_packed [E,H,I/2]), the codes one per byte when keep_codes (w13, w2),
    E4M3 scales as uint8 (w13_sf [E,2I,H/16], w2_sf [E,H,I/16]), global
    scales w13_g, w2_g [E] and the activations' a1_g, a2_g."""
    base = make_moe_inputs(cfg, seed, device, weights=False)
    g = _gen(seed + 7919, device)
    E, H, I = cfg.E, cfg.H, cfg.I
    out = dict(w13_packed=torch.empty(E, 2 * I, H // 2, dtype=torch.uint8, device=device),
               w13_sf=torch.empty(E, 2 * I, H // 16, dtype=torch.uint8, device=device),
               w13_g=torch.empty(E, dtype=torch.float32, device=device),
               w2_packed=torch.empty(E, H, I // 2, dtype=torch.uint8, device=device),
               w2_sf=torch.empty(E, H, I // 16, dtype=torch.uint8, device=device),
               w2_g=torch.empty(E, dtype=torch.float32, device=device))
    if keep_codes:
        out["w13"] = torch.empty(E, 2 * I, H, dtype=torch.uint8, device=device)
        out["w2"] = torch.empty(E, H, I, dtype=torch.uint8, device=device)
    for name, rows, cols in (("w13", 2 * I, H), ("w2", H, I)):
        for e in range(E):
            w = torch.randn(rows, cols, generator=g, device=device) / math.sqrt(cols)
            ge = 448.0 * 6.0 / float(w.abs().max())
            q, sf = quantize_nvfp4_rows(w, ge)
            out[name + "_g"][e] = ge
            out[name + "_sf"][e] = sf.view(torch.uint8)
            out[name + "_packed"][e] = pack_e2m1(q)
            if keep_codes:
                out[name][e] = q
    base.update(out)
    base.update(a1_g=NVFP4_A1_GSCALE, a2_g=NVFP4_A2_GSCALE)
    return base
