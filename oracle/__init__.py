"""CPU oracle for the fused W8A8 block-scaled MoE expert computation.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference leg of ``bench.py`` use it.  It shares no code with the CUDA
library; the arithmetic lives in ``moe_oracle.c`` (plain C, fp32, one
rounding per operation) and this module only marshals numpy arrays into it.

The tile-size selector (``select_tile_m``) is written here in plain Python,
straight from the wave+residue description on the page "FlashInfer SM120 MoE
GEMM 최적화: 웨이브+잔여물 비용 모델 도입" (flashinfer PR #4318, "코드 분석 2."
and "리뷰 피드백 반영"), re-parameterised for the tile menu of the sm_100a
kernels (token tiles 16/32/64 on the swapped path, 128 on the direct path).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        P = ctypes.c_void_p
        i = ctypes.c_int
        L.oracle_e4m3_decode.restype = ctypes.c_float
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e8m0_decode.restype = ctypes.c_float
        L.oracle_e8m0_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e8m0_scale_code.restype = ctypes.c_uint8
        L.oracle_e8m0_scale_code.argtypes = [ctypes.c_float]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_router_topk.restype = None
        L.oracle_router_topk.argtypes = [P, i, i, i, P, P]
        L.oracle_route_permute.restype = i
        L.oracle_route_permute.argtypes = [P, i, i, i, P, P, P]
        L.oracle_quant_rows_128.restype = None
        L.oracle_quant_rows_128.argtypes = [P, i, i, P, P]
        L.oracle_quant_rows_128_bf16.restype = None
        L.oracle_quant_rows_128_bf16.argtypes = [P, i, i, P, P]
        L.oracle_grouped_gemm.restype = None
        L.oracle_grouped_gemm.argtypes = [P, P, P, P, P, i, i, i, i, P]
        L.oracle_swiglu.restype = None
        L.oracle_swiglu.argtypes = [P, i, i, P]
        L.oracle_moe_fused.restype = i
        L.oracle_moe_fused.argtypes = [P] * 8 + [i] * 5 + [P] * 4
        L.oracle_moe_tokens.restype = None
        L.oracle_moe_tokens.argtypes = [P] * 7 + [i] * 5 + [P, i, P, P, P]
        L.oracle_groupwise_gemm_bf16.restype = None
        L.oracle_groupwise_gemm_bf16.argtypes = [P, P, P, P, P, i, i, i, i, i, P]
        L.oracle_swiglu_mxfp8.restype = None
        L.oracle_swiglu_mxfp8.argtypes = [P, i, i, P, P]
        L.oracle_quant_rows_mx_bf16.restype = None
        L.oracle_quant_rows_mx_bf16.argtypes = [P, i, i, P, P]
        L.oracle_mx_grouped_gemm.restype = None
        L.oracle_mx_grouped_gemm.argtypes = [P, P, P, P, P, i, i, i, i, P]
        L.oracle_mx_gemm_bf16.restype = None
        L.oracle_mx_gemm_bf16.argtypes = [P, P, P, P, P, i, i, i, i, i, P]
        L.oracle_e2m1_decode.restype = ctypes.c_float
        L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_encode.restype = ctypes.c_uint8
        L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        L.oracle_quant_rows_nvfp4.restype = None
        L.oracle_quant_rows_nvfp4.argtypes = [P, i, i, ctypes.c_float, P, P]
        L.oracle_nvfp4_grouped_gemm.restype = None
        L.oracle_nvfp4_grouped_gemm.argtypes = [P, P, ctypes.c_float, P, P, P, P, i, i, i, i, P]
        L.oracle_nvfp4_gemm_bf16.restype = None
        L.oracle_moe_nvfp4_fused.restype = i
        L.oracle_moe_nvfp4_fused.argtypes = [P] * 9 + [ctypes.c_float] * 2 + [P] + [i] * 5 + [P] * 4
        L.oracle_moe_nvfp4_tokens.restype = None
        L.oracle_moe_nvfp4_tokens.argtypes = ([P] * 9 + [ctypes.c_float] * 2 + [i] * 5 +
                                              [P, i, P, P, P])
        L.oracle_nvfp4_gemm_bf16.argtypes = [P, P, ctypes.c_float, P, P, P, P, i, i, i, i, i, P]
        L.oracle_moe_mx_tokens.restype = None
        L.oracle_moe_mx_tokens.argtypes = [P] * 7 + [i] * 5 + [P, i, P, P, P]
        L.oracle_moe_mx_fused.restype = i
        L.oracle_moe_mx_fused.argtypes = [P] * 8 + [i] * 5 + [P] * 4
        L.oracle_combine.restype = None
        L.oracle_combine.argtypes = [P, P, P, i, i, i, P]
        L.oracle_num_threads.restype = i
        L.oracle_num_threads.argtypes = []
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _u8(a):
    return np.ascontiguousarray(np.asarray(a).view(np.uint8) if np.asarray(a).dtype != np.uint8 else a)


def _c(a, dt):
    return np.ascontiguousarray(np.asarray(a, dtype=dt))


def num_threads() -> int:
    return int(lib().oracle_num_threads())


# ---------------------------------------------------------------- codecs
def e4m3_decode(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    table = np.array([lib().oracle_e4m3_decode(c) for c in range(256)], dtype=np.float32)
    return table[codes]


def e4m3_encode(values) -> np.ndarray:
    v = np.asarray(values, dtype=np.float32)
    f = lib().oracle_e4m3_encode
    return np.array([f(float(x)) for x in v.ravel()], dtype=np.uint8).reshape(v.shape)


def e8m0_decode(code: int) -> float:
    return float(lib().oracle_e8m0_decode(code))


def e8m0_scale_code(amax: float) -> int:
    return int(lib().oracle_e8m0_scale_code(float(amax)))


def f32_to_bf16_bits(values) -> np.ndarray:
    v = np.asarray(values, dtype=np.float32)
    f = lib().oracle_f32_to_bf16
    return np.array([f(float(x)) for x in v.ravel()], dtype=np.uint16).reshape(v.shape)


# ---------------------------------------------------------------- stages
def router_topk(logits, k: int):
    """logits fp32 [T, E] -> (ids int32 [T, k], weights fp32 [T, k])."""
    l = _c(logits, np.float32)
    T, E = l.shape
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    lib().oracle_router_topk(_p(l), T, E, k, _p(ids), _p(w))
    return ids, w


def route_permute(topk_ids, E: int):
    """Stage a1.  Returns (m_indptr[E+1], perm[R], inv_perm[R], n_bad)."""
    ids = _c(topk_ids, np.int32)
    T, k = ids.shape
    R = T * k
    m_indptr = np.zeros(E + 1, np.int32)
    perm = np.full(max(R, 1), -1, np.int32)
    inv_perm = np.full(max(R, 1), -1, np.int32)
    bad = lib().oracle_route_permute(_p(ids), T, k, E, _p(m_indptr), _p(perm), _p(inv_perm))
    return m_indptr, perm[:R], inv_perm[:R], int(bad)


def quant_rows_128(x):
    """Stages a2/a5 on fp32 rows.  Returns (codes [rows, cols], scale [rows, cols/128])."""
    x = _c(x, np.float32)
    rows, cols = x.shape
    q = np.zeros((rows, cols), np.uint8)
    s = np.zeros((rows, cols // 128), np.float32)
    lib().oracle_quant_rows_128(_p(x), rows, cols, _p(q), _p(s))
    return q, s


def quant_rows_128_bf16(x_bits):
    """Stage a2 on bf16 rows given as uint16 bit patterns."""
    x = _c(x_bits, np.uint16)
    rows, cols = x.shape
    q = np.zeros((rows, cols), np.uint8)
    s = np.zeros((rows, cols // 128), np.float32)
    lib().oracle_quant_rows_128_bf16(_p(x), rows, cols, _p(q), _p(s))
    return q, s


def grouped_gemm(a, a_scale, b, b_scale, m_indptr):
    """Stages a3/a6.  a [R,K] codes, a_scale [R,K/128], b [E,N,K] codes,
    b_scale [E,N/128,K/128] -> fp32 [R,N] (rows outside m_indptr are 0)."""
    a = _u8(a); b = _u8(b)
    a_scale = _c(a_scale, np.float32); b_scale = _c(b_scale, np.float32)
    m_indptr = _c(m_indptr, np.int32)
    R, K = a.shape
    E, N, _ = b.shape
    out = np.zeros((R, N), np.float32)
    lib().oracle_grouped_gemm(_p(a), _p(a_scale), _p(b), _p(b_scale), _p(m_indptr),
                              R, N, K, E, _p(out))
    return out


def swiglu(g):
    g = _c(g, np.float32)
    rows, n2 = g.shape
    h = np.zeros((rows, n2 // 2), np.float32)
    lib().oracle_swiglu(_p(g), rows, n2 // 2, _p(h))
    return h


def moe_fused(x_bits, topk_ids, topk_w, w13, w13_scale, w2, w2_scale):
    """Whole layer, grouped form.  Returns dict with out (bf16 bits [T,H]),
    m_indptr, perm, hq [R,I] codes, hs [R,I/128] (grouped-row order), n_bad."""
    x = _c(x_bits, np.uint16)
    ids = _c(topk_ids, np.int32)
    tw = _c(topk_w, np.float32)
    w13 = _u8(w13); w2 = _u8(w2)
    w13_scale = _c(w13_scale, np.float32); w2_scale = _c(w2_scale, np.float32)
    T, H = x.shape
    k = ids.shape[1]
    E, I2, _ = w13.shape
    I = I2 // 2
    R = T * k
    out = np.zeros((T, H), np.uint16)
    m_indptr = np.zeros(E + 1, np.int32)
    perm = np.zeros(max(R, 1), np.int32)
    hq = np.zeros((max(R, 1), I), np.uint8)
    hs = np.zeros((max(R, 1), I // 128), np.float32)
    bad = lib().oracle_moe_fused(_p(x), _p(ids), _p(tw), _p(w13), _p(w13_scale), _p(w2),
                                 _p(w2_scale), _p(out), T, H, I, E, k, _p(m_indptr), _p(perm),
                                 _p(hq), _p(hs))
    Rg = int(m_indptr[E])
    return dict(out=out, m_indptr=m_indptr, perm=perm[:Rg], hq=hq[:Rg], hs=hs[:Rg], n_bad=int(bad))


def moe_tokens(x_bits, topk_ids, topk_w, w13, w13_scale, w2, w2_scale, tokens, want_h=False):
    """Whole layer, per-token form, for the listed tokens only.
    Returns out [n,H] bf16 bits (and hq [n,k,I], hs [n,k,I/128] if want_h)."""
    x = _c(x_bits, np.uint16)
    ids = _c(topk_ids, np.int32)
    tw = _c(topk_w, np.float32)
    w13 = _u8(w13); w2 = _u8(w2)
    w13_scale = _c(w13_scale, np.float32); w2_scale = _c(w2_scale, np.float32)
    tokens = _c(tokens, np.int32)
    T, H = x.shape
    k = ids.shape[1]
    E, I2, _ = w13.shape
    I = I2 // 2
    n = len(tokens)
    out = np.zeros((n, H), np.uint16)
    hq = np.zeros((n, k, I), np.uint8) if want_h else None
    hs = np.zeros((n, k, I // 128), np.float32) if want_h else None
    lib().oracle_moe_tokens(_p(x), _p(ids), _p(tw), _p(w13), _p(w13_scale), _p(w2), _p(w2_scale),
                            T, H, I, E, k, _p(tokens), n, _p(out),
                            _p(hq) if want_h else None, _p(hs) if want_h else None)
    return (out, hq, hs) if want_h else out


def combine(y, inv_perm, topk_w):
    """Stage 5 alone: out [T, H] bf16 bits = bf16(sum_j topk_w[t, j] *
    y[inv_perm[t*k + j]]) in fp32, ascending j, pairs with inv_perm < 0
    skipped.  y [rows, H] fp32 (grouped rows), inv_perm [T*k], topk_w [T, k]."""
    y = _c(y, np.float32)
    w = _c(topk_w, np.float32)
    T, k = w.shape
    inv = _c(inv_perm, np.int32).reshape(T * k)
    H = y.shape[1]
    assert int(inv.max(initial=-1)) < y.shape[0]
    out = np.zeros((T, H), np.uint16)
    lib().oracle_combine(_p(y), _p(inv), _p(w), T, k, H, _p(out))
    return out


def groupwise_gemm_bf16(a, a_scale_kmajor, b, b_scale, m_indptr, is_gated: bool):
    a = _u8(a); b = _u8(b)
    a_scale_kmajor = _c(a_scale_kmajor, np.float32); b_scale = _c(b_scale, np.float32)
    m_indptr = _c(m_indptr, np.int32)
    R, K = a.shape
    E, N, _ = b.shape
    out = np.zeros((R, N // 2 if is_gated else N), np.uint16)
    lib().oracle_groupwise_gemm_bf16(_p(a), _p(a_scale_kmajor), _p(b), _p(b_scale), _p(m_indptr),
                                     R, N, K, E, int(bool(is_gated)), _p(out))
    return out


def swiglu_mxfp8(in_bits):
    """Stage a10.  in [M, 2K] bf16 bits -> (codes [M,K], e8m0 [M,K/32])."""
    x = _c(in_bits, np.uint16)
    M, K2 = x.shape
    K = K2 // 2
    out = np.zeros((M, K), np.uint8)
    sc = np.zeros((M, K // 32), np.uint8)
    lib().oracle_swiglu_mxfp8(_p(x), M, K, _p(out), _p(sc))
    return out, sc


# ---------------------------------------------------------------- MXFP8 variant
def quant_rows_mx_bf16(x_bits):
    """[rows, cols] bf16 bits -> (E4M3 codes [rows, cols], E8M0 codes [rows, cols/32])."""
    x = _c(x_bits, np.uint16)
    rows, cols = x.shape
    q = np.zeros((rows, cols), np.uint8)
    sf = np.zeros((rows, cols // 32), np.uint8)
    lib().oracle_quant_rows_mx_bf16(_p(x), rows, cols, _p(q), _p(sf))
    return q, sf


def mx_grouped_gemm(a, a_sf, b, b_sf, m_indptr):
    """fp32 [R, N]: per 32-wide K block, 2^(sa-127) 2^(sb-127) times the block dot."""
    a = _u8(a); b = _u8(b); a_sf = _u8(a_sf); b_sf = _u8(b_sf)
    m_indptr = _c(m_indptr, np.int32)
    R, K = a.shape
    E, N, _ = b.shape
    out = np.zeros((R, N), np.float32)
    lib().oracle_mx_grouped_gemm(_p(a), _p(a_sf), _p(b), _p(b_sf), _p(m_indptr), R, N, K, E,
                                 _p(out))
    return out


def mx_gemm_bf16(a, a_sf, b, b_sf, m_indptr, is_gated: bool):
    a = _u8(a); b = _u8(b); a_sf = _u8(a_sf); b_sf = _u8(b_sf)
    m_indptr = _c(m_indptr, np.int32)
    R, K = a.shape
    E, N, _ = b.shape
    out = np.zeros((R, N // 2 if is_gated else N), np.uint16)
    lib().oracle_mx_gemm_bf16(_p(a), _p(a_sf), _p(b), _p(b_sf), _p(m_indptr), R, N, K, E,
                              int(bool(is_gated)), _p(out))
    return out


def moe_mx_fused(x_bits, topk_ids, topk_w, w13, w13_sf, w2, w2_sf, want_dump=False):
    """The fused layer with MXFP8 operands.  x_bits [T,H] bf16 bits; w13 [E,2I,H]
    codes, w13_sf [E,2I,H/32]; w2 [E,H,I] codes, w2_sf [E,H,I/32].  Returns bf16
    bits [T,H] (and m_indptr, perm, hq [R,I], hsf [R,I/32] when want_dump)."""
    x = _c(x_bits, np.uint16)
    ids = _c(topk_ids, np.int32)
    w = _c(topk_w, np.float32)
    w13 = _u8(w13); w2 = _u8(w2); w13_sf = _u8(w13_sf); w2_sf = _u8(w2_sf)
    T, H = x.shape
    k = ids.shape[1]
    E, I2, _ = w13.shape
    I = I2 // 2
    R = T * k
    out = np.zeros((T, H), np.uint16)
    m_indptr = np.zeros(E + 1, np.int32)
    perm = np.zeros(max(R, 1), np.int32)
    hq = np.zeros((max(R, 1), I), np.uint8)
    hsf = np.zeros((max(R, 1), I // 32), np.uint8)
    lib().oracle_moe_mx_fused(_p(x), _p(ids), _p(w), _p(w13), _p(w13_sf), _p(w2), _p(w2_sf),
                              _p(out), T, H, I, E, k, _p(m_indptr), _p(perm), _p(hq), _p(hsf))
    if want_dump:
        Rg = int(m_indptr[E])
        return out, m_indptr, perm[:Rg], hq[:Rg], hsf[:Rg]
    return out


def moe_mx_tokens(x_bits, topk_ids, topk_w, w13, w13_sf, w2, w2_sf, tokens, want_h=False):
    """Per-token form of moe_mx_fused for the listed tokens: bf16 bits [n, H]
    (and hq [n, k, I], hsf [n, k, I/32] when want_h)."""
    x = _c(x_bits, np.uint16)
    ids = _c(topk_ids, np.int32)
    w = _c(topk_w, np.float32)
    w13 = _u8(w13); w2 = _u8(w2); w13_sf = _u8(w13_sf); w2_sf = _u8(w2_sf)
    tok = _c(tokens, np.int32)
    T, H = x.shape
    k = ids.shape[1]
    E, I2, _ = w13.shape
    I = I2 // 2
    n = len(tok)
    out = np.zeros((n, H), np.uint16)
    hq = np.zeros((n, k, I), np.uint8)
    hsf = np.zeros((n, k, I // 32), np.uint8)
    lib().oracle_moe_mx_tokens(_p(x), _p(ids), _p(w), _p(w13), _p(w13_sf), _p(w2), _p(w2_sf),
                               T, H, I, E, k, _p(tok), n, _p(out), _p(hq), _p(hsf))
    return (out, hq, hsf) if want_h else out


# ---------------------------------------------------------------- NVFP4 variant
def e2m1_decode(codes) -> np.ndarray:
    return np.array([lib().oracle_e2m1_decode(int(c)) for c in np.asarray(codes).ravel()],
                    np.float32).reshape(np.shape(codes))


def e2m1_encode(values) -> np.ndarray:
    return np.array([lib().oracle_e2m1_encode(float(v)) for v in np.asarray(values).ravel()],
                    np.uint8).reshape(np.shape(values))


def quant_rows_nvfp4(x, g: float):
    """[rows, cols] fp32 -> (E2M1 codes [rows, cols], E4M3 block scales [rows, cols/16])."""
    x = _c(x, np.float32)
    rows, cols = x.shape
    q = np.zeros((rows, cols), np.uint8)
    sf = np.zeros((rows, cols // 16), np.uint8)
    lib().oracle_quant_rows_nvfp4(_p(x), rows, cols, float(g), _p(q), _p(sf))
    return q, sf


def nvfp4_grouped_gemm(a, a_sf, ga, b, b_sf, gb, m_indptr):
    a = _u8(a); b = _u8(b); a_sf = _u8(a_sf); b_sf = _u8(b_sf)
    gb = _c(gb, np.float32); m_indptr = _c(m_indptr, np.int32)
    R, K = a.shape
    E, N, _ = b.shape
    out = np.zeros((R, N), np.float32)
    lib().oracle_nvfp4_grouped_gemm(_p(a), _p(a_sf), float(ga), _p(b), _p(b_sf), _p(gb),
                                    _p(m_indptr), R, N, K, E, _p(out))
    return out


def nvfp4_gemm_bf16(a, a_sf, ga, b, b_sf, gb, m_indptr, is_gated: bool):
    """bf16 bits of the NVFP4 GEMM: [R, N], or gated [R, N/2] = silu(gate) * up."""
    a = _u8(a); b = _u8(b); a_sf = _u8(a_sf); b_sf = _u8(b_sf)
    gb = _c(gb, np.float32); m_indptr = _c(m_indptr, np.int32)
    R, K = a.shape
    E, N, _ = b.shape
    out = np.zeros((R, N // 2 if is_gated else N), np.uint16)
    lib().oracle_nvfp4_gemm_bf16(_p(a), _p(a_sf), float(ga), _p(b), _p(b_sf), _p(gb),
                                 _p(m_indptr), R, N, K, E, int(bool(is_gated)), _p(out))
    return out


def moe_nvfp4_fused(x_bits, topk_ids, topk_w, w13, w13_sf, w13_g, w2, w2_sf, w2_g, a1_g, a2_g,
                    want_dump=False):
    """The fused layer with NVFP4 operands.  x_bits [T,H] bf16 bits; w13 [E,2I,H]
    E2M1 codes (one per byte), w13_sf [E,2I,H/16] E4M3, w13_g [E]; w2 [E,H,I],
    w2_sf [E,H,I/16], w2_g [E]; a1_g, a2_g the activations' global scales.
    Returns bf16 bits [T,H] (and m_indptr, perm, hq [R,I], hsf [R,I/16] when
    want_dump)."""
    x = _c(x_bits, np.uint16)
    ids = _c(topk_ids, np.int32)
    w = _c(topk_w, np.float32)
    w13 = _u8(w13); w2 = _u8(w2); w13_sf = _u8(w13_sf); w2_sf = _u8(w2_sf)
    w13_g = _c(w13_g, np.float32); w2_g = _c(w2_g, np.float32)
    T, H = x.shape
    k = ids.shape[1]
    E, I2, _ = w13.shape
    I = I2 // 2
    R = T * k
    out = np.zeros((T, H), np.uint16)
    m_indptr = np.zeros(E + 1, np.int32)
    perm = np.zeros(max(R, 1), np.int32)
    hq = np.zeros((max(R, 1), I), np.uint8)
    hsf = np.zeros((max(R, 1), I // 16), np.uint8)
    lib().oracle_moe_nvfp4_fused(_p(x), _p(ids), _p(w), _p(w13), _p(w13_sf), _p(w13_g), _p(w2),
                                 _p(w2_sf), _p(w2_g), float(a1_g), float(a2_g), _p(out), T, H, I,
                                 E, k, _p(m_indptr), _p(perm), _p(hq), _p(hsf))
    if want_dump:
        Rg = int(m_indptr[E])
        return out, m_indptr, perm[:Rg], hq[:Rg], hsf[:Rg]
    return out


def moe_nvfp4_tokens(x_bits, topk_ids, topk_w, w13, w13_sf, w13_g, w2, w2_sf, w2_g, a1_g, a2_g,
                     tokens, want_h=False):
    """Per-token form of moe_nvfp4_fused for the listed tokens: bf16 bits [n, H]
    (and hq [n, k, I], hsf [n, k, I/16] when want_h)."""
    x = _c(x_bits, np.uint16)
    ids = _c(topk_ids, np.int32)
    w = _c(topk_w, np.float32)
    w13 = _u8(w13); w2 = _u8(w2); w13_sf = _u8(w13_sf); w2_sf = _u8(w2_sf)
    w13_g = _c(w13_g, np.float32); w2_g = _c(w2_g, np.float32)
    tok = _c(tokens, np.int32)
    T, H = x.shape
    k = ids.shape[1]
    E, I2, _ = w13.shape
    I = I2 // 2
    n = len(tok)
    out = np.zeros((n, H), np.uint16)
    hq = np.zeros((n, k, I), np.uint8)
    hsf = np.zeros((n, k, I // 16), np.uint8)
    lib().oracle_moe_nvfp4_tokens(_p(x), _p(ids), _p(w), _p(w13), _p(w13_sf), _p(w13_g), _p(w2),
                                  _p(w2_sf), _p(w2_g), float(a1_g), float(a2_g), T, H, I, E, k,
                                  _p(tok), n, _p(out), _p(hq), _p(hsf))
    return (out, hq, hsf) if want_h else out


# ---------------------------------------------------------------- tile selection
# Tile menu of the sm_100a grouped GEMM: token tiles of 16/32/64 rows run with
# the weights as the 128-row MMA operand ("swap-AB"), 128-row token tiles run
# with the tokens as the MMA M operand.  Every tile covers 256 weight rows
# (gated: 128 gate + 128 up rows -> 128 output columns; plain: 256 columns).
TILE_MENU = (16, 32, 64, 128)
# Per-tile cost that does not shrink with the token tile (streaming the
# 256-row weight tile, pipeline fill, epilogue), in token-row equivalents.
TILE_OVERHEAD_ROWS = 32


def balanced_max_rows(total_rows: int, E: int) -> int:
    """Largest per-expert row count if rows spread evenly (remainder included)."""
    return -(-total_rows // E) if E > 0 else 0


def balanced_tile_count(total_rows: int, n_out: int, E: int, tile_m: int, tile_n: int) -> int:
    """Tiles over all experts when rows spread evenly: r experts get q+1 rows,
    E-r get q rows, with q = total_rows // E and r = total_rows % E."""
    q, r = divmod(total_rows, E)
    m_tiles = r * (-(-(q + 1) // tile_m)) + (E - r) * (-(-q // tile_m))
    return m_tiles * (-(-n_out // tile_n))


def select_tile_m(total_rows: int, n: int, k: int, E: int, num_sms: int, is_gated: bool):
    """Returns (tile_m, tile_n) with tile_n counted in output columns."""
    n_out = n // 2 if is_gated else n
    tile_n = 128 if is_gated else 256
    if E <= 0 or total_rows <= 0:
        return 16, tile_n
    max_m = balanced_max_rows(total_rows, E)

    def tiles(tm):
        return balanced_tile_count(total_rows, n_out, E, tm, tile_n)

    if max_m <= 16 or (tiles(32) < num_sms // 2 and tiles(16) <= num_sms):
        return 16, tile_n
    if max_m <= 32:
        return 32, tile_n
    if k <= 2048:
        return (64 if max_m < 192 else 128), tile_n

    def cost(tm):
        waves = -(-tiles(tm) // num_sms)
        return waves * (tm + TILE_OVERHEAD_ROWS)

    return (64 if cost(64) < cost(128) else 128), tile_n
