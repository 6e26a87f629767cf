"""Python binding of libmoefp8.so, the sm_100a fused W8A8 block-scaled MoE
library (C ABI in include/moefp8.h).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  PyTorch supplies device memory and streams.  The
binding raises if the compiled library is missing; there is no fallback.

Functions keep the C names:
  moe_route_permute, moe_fp8_fused, moe_fp8_fused_debug,
  fp8_groupwise_moe_gemm, swiglu_mxfp8_quant, moe_select_tile_m,
  moe_workspace_size, moe_route_workspace_size, moe_get_device_status,
  moe_set_wait_timeout_ns, moe_set_expert_fusion, moe_status_string.
Tensor arguments may be torch tensors (their data_ptr is passed) or raw
integer device addresses.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "MoEError", "lib", "lib_path", "EXPORTS",
    "moe_route_permute", "moe_fp8_fused", "moe_fp8_fused_debug", "fp8_groupwise_moe_gemm",
    "swiglu_mxfp8_quant", "moe_select_tile_m", "moe_workspace_size", "moe_route_workspace_size",
    "moe_get_device_status", "moe_set_wait_timeout_ns", "moe_status_string",
    "moe_set_stage_events", "moe_route_permute_noalloc", "mxfp8_moe_gemm",
    "mxfp8_tile_scales", "moe_mxfp8_fused", "moe_mxfp8_fused_debug", "moe_router_topk",
    "nvfp4_moe_gemm", "nvfp4_tile_scales", "moe_nvfp4_fused", "moe_nvfp4_fused_debug",
    "nvfp4_quantize", "moe_tactic_tune_gemm", "moe_tactic_lookup", "moe_tactic_store",
    "moe_tactic_clear", "moe_ep_workspace_size", "moe_ep_plan", "moe_ep_pack",
    "moe_fp8_expert_rows_workspace_size", "moe_fp8_expert_rows", "moe_combine", "moe_router_route",
    "moe_set_expert_fusion", "moe_fp8_fused_plan",
    "MOE_FUSION_AUTO", "MOE_FUSION_ON", "MOE_FUSION_OFF",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoefp8.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_CUDA = 3
MOE_ERR_NO_TILE_CONFIG = 4
MOE_ERR_DEVICE_TIMEOUT = 5
MOE_ERR_BAD_EXPERT_ID = 6

MOE_FUSION_AUTO = 0
MOE_FUSION_ON = 1
MOE_FUSION_OFF = 2

# Every symbol declared in include/moefp8.h.
EXPORTS = (
    "moe_status_string", "moe_route_workspace_size", "moe_route_permute", "moe_workspace_size",
    "moe_fp8_fused", "moe_fp8_fused_debug", "fp8_groupwise_moe_gemm", "moe_select_tile_m",
    "swiglu_mxfp8_quant", "moe_get_device_status", "moe_set_wait_timeout_ns",
    "moe_set_stage_events", "moe_route_permute_noalloc", "mxfp8_moe_gemm", "mxfp8_tile_scales",
    "moe_mxfp8_fused", "moe_mxfp8_fused_debug", "moe_router_topk", "nvfp4_moe_gemm",
    "nvfp4_tile_scales", "moe_nvfp4_fused", "moe_nvfp4_fused_debug", "nvfp4_quantize",
    "moe_tactic_tune_gemm", "moe_tactic_lookup", "moe_tactic_store", "moe_tactic_clear",
    "moe_ep_workspace_size", "moe_ep_plan", "moe_ep_pack", "moe_fp8_expert_rows_workspace_size",
    "moe_fp8_expert_rows", "moe_combine", "moe_router_route", "moe_set_expert_fusion",
    "moe_fp8_fused_plan",
)

_lib = None


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = int(status)
        super().__init__(f"{where}: {moe_status_string(status)} ({status})")


def lib_path() -> str:
    return LIB_PATH


def lib():
    """Loads libmoefp8.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m fp8_block_scaled_route_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, Z, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_status_string.argtypes = [I]
    L.moe_route_workspace_size.restype = Z
    L.moe_route_workspace_size.argtypes = [I, I, I]
    L.moe_route_permute.restype = I
    L.moe_route_permute.argtypes = [P, I, I, I, P, P, P, P, Z, P]
    L.moe_workspace_size.restype = Z
    L.moe_workspace_size.argtypes = [I] * 5
    L.moe_fp8_fused.restype = I
    L.moe_fp8_fused.argtypes = [P] * 8 + [I] * 5 + [P, Z, P]
    L.moe_fp8_fused_debug.restype = I
    L.moe_fp8_fused_debug.argtypes = [P] * 8 + [I] * 5 + [P, Z, P] + [P] * 4
    L.fp8_groupwise_moe_gemm.restype = I
    L.fp8_groupwise_moe_gemm.argtypes = [P] * 6 + [I] * 11 + [P]
    L.moe_select_tile_m.restype = I
    L.moe_select_tile_m.argtypes = [I] * 6 + [ctypes.POINTER(I), ctypes.POINTER(I)]
    L.swiglu_mxfp8_quant.restype = I
    L.swiglu_mxfp8_quant.argtypes = [P, P, P, I, I, P]
    L.mxfp8_moe_gemm.restype = I
    L.mxfp8_moe_gemm.argtypes = [P] * 6 + [I] * 6 + [P]
    L.moe_router_topk.restype = I
    L.moe_router_topk.argtypes = [P, I, I, I, P, P, P]
    L.mxfp8_tile_scales.restype = I
    L.mxfp8_tile_scales.argtypes = [P, P, I, I, P]
    L.nvfp4_moe_gemm.restype = I
    L.nvfp4_moe_gemm.argtypes = [P] * 7 + [I] * 6 + [P]
    L.nvfp4_tile_scales.restype = I
    L.nvfp4_tile_scales.argtypes = [P, P, I, I, P]
    F = ctypes.c_float
    L.moe_tactic_tune_gemm.restype = I
    L.moe_tactic_tune_gemm.argtypes = [P] * 6 + [I] * 7 + [P, ctypes.POINTER(I)]
    L.moe_tactic_lookup.restype = I
    L.moe_tactic_lookup.argtypes = [I] * 5 + [ctypes.POINTER(I)]
    L.moe_tactic_store.restype = I
    L.moe_tactic_store.argtypes = [I] * 6
    L.moe_tactic_clear.restype = None
    L.moe_tactic_clear.argtypes = []
    L.nvfp4_quantize.restype = I
    L.nvfp4_quantize.argtypes = [P, F, P, P, I, I, P]
    L.moe_nvfp4_fused.restype = I
    L.moe_nvfp4_fused.argtypes = [P] * 9 + [F, F, P] + [I] * 5 + [P, ctypes.c_size_t, P]
    L.moe_nvfp4_fused_debug.restype = I
    L.moe_nvfp4_fused_debug.argtypes = ([P] * 9 + [F, F, P] + [I] * 5 +
                                        [P, ctypes.c_size_t, P] + [P] * 4)
    L.moe_mxfp8_fused.restype = I
    L.moe_mxfp8_fused.argtypes = [P] * 8 + [I] * 5 + [P, ctypes.c_size_t, P]
    L.moe_mxfp8_fused_debug.restype = I
    L.moe_mxfp8_fused_debug.argtypes = [P] * 8 + [I] * 5 + [P, ctypes.c_size_t, P] + [P] * 4
    L.moe_get_device_status.restype = I
    L.moe_get_device_status.argtypes = [P, P]
    L.moe_set_wait_timeout_ns.restype = None
    L.moe_set_wait_timeout_ns.argtypes = [U64]
    L.moe_set_expert_fusion.restype = I
    L.moe_set_expert_fusion.argtypes = [I]
    L.moe_fp8_fused_plan.restype = I
    L.moe_fp8_fused_plan.argtypes = [I] * 5 + [P] * 3
    L.moe_route_permute_noalloc.restype = I
    L.moe_route_permute_noalloc.argtypes = [P, I, I, I, P, P, P, P]
    L.moe_set_stage_events.restype = I
    L.moe_set_stage_events.argtypes = [ctypes.POINTER(P), I]
    L.moe_ep_workspace_size.restype = Z
    L.moe_ep_workspace_size.argtypes = [I, I, I]
    L.moe_ep_plan.restype = I
    L.moe_ep_plan.argtypes = [P, I, I, I, I, P, P, P, P, Z, P]
    L.moe_ep_pack.restype = I
    L.moe_ep_pack.argtypes = [P, P, P] + [I] * 6 + [P, P, P, P]
    L.moe_fp8_expert_rows_workspace_size.restype = Z
    L.moe_fp8_expert_rows_workspace_size.argtypes = [I] * 4
    L.moe_fp8_expert_rows.restype = I
    L.moe_fp8_expert_rows.argtypes = [P, P, P, I, P, P, P, P, P, I, I, I, P, Z, P]
    L.moe_combine.restype = I
    L.moe_combine.argtypes = [P, P, P, I, I, I, P, P]
    L.moe_router_route.restype = I
    L.moe_router_route.argtypes = [P, I, I, I, P, P, P, P, P, P, Z, P]
    _lib = L
    return L


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, where: str, check: bool) -> int:
    if check and status != MOE_OK:
        raise MoEError(status, where)
    return status


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def moe_set_wait_timeout_ns(ns: int) -> None:
    lib().moe_set_wait_timeout_ns(int(ns))


def moe_set_expert_fusion(mode: int) -> None:
    """MOE_FUSION_AUTO, MOE_FUSION_ON or MOE_FUSION_OFF (process-wide)."""
    _check(lib().moe_set_expert_fusion(int(mode)), "moe_set_expert_fusion", True)


def moe_fp8_fused_plan(T: int, H: int, I: int, E: int, k: int) -> dict:
    """Launch plan of moe_fp8_fused on the current device:
    {"tile_m1", "tile_m2", "fused"}."""
    a, b, c = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().moe_fp8_fused_plan(T, H, I, E, k, ctypes.byref(a), ctypes.byref(b),
                                    ctypes.byref(c)), "moe_fp8_fused_plan", True)
    return {"tile_m1": a.value, "tile_m2": b.value, "fused": bool(c.value)}


def moe_workspace_size(T: int, H: int, I: int, E: int, k: int) -> int:
    return int(lib().moe_workspace_size(T, H, I, E, k))


def moe_route_workspace_size(T: int, k: int, E: int) -> int:
    return int(lib().moe_route_workspace_size(T, k, E))


def moe_select_tile_m(total_rows: int, n: int, k: int, E: int, num_sms: int, is_gated: bool):
    tm, tn = ctypes.c_int(0), ctypes.c_int(0)
    st = lib().moe_select_tile_m(total_rows, n, k, E, num_sms, int(bool(is_gated)),
                                 ctypes.byref(tm), ctypes.byref(tn))
    _check(st, "moe_select_tile_m", True)
    return tm.value, tn.value


def moe_route_permute(topk_ids, E: int, m_indptr, perm, inv_perm, ws, ws_bytes=None, *,
                      T=None, k=None, stream=None, check=True) -> int:
    if T is None or k is None:
        T, k = topk_ids.shape
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    st = lib().moe_route_permute(_ptr(topk_ids), T, k, E, _ptr(m_indptr), _ptr(perm),
                                 _ptr(inv_perm), _ptr(ws), ws_bytes, _stream(stream))
    return _check(st, "moe_route_permute", check)


def moe_router_route(logits, k: int, topk_ids, topk_w, m_indptr, perm, inv_perm, ws, ws_bytes=None,
                     *, dims=None, stream=None, check=True) -> int:
    """moe_router_topk + moe_route_permute in one call (one launch for up to
    8192 pairs); dims = (T, E) when raw addresses are passed."""
    T, E = dims if dims is not None else logits.shape
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    st = lib().moe_router_route(_ptr(logits), T, E, k, _ptr(topk_ids), _ptr(topk_w),
                                _ptr(m_indptr), _ptr(perm), _ptr(inv_perm), _ptr(ws), ws_bytes,
                                _stream(stream))
    return _check(st, "moe_router_route", check)


def moe_route_permute_noalloc(topk_ids, E: int, m_indptr, perm, inv_perm, *, T=None, k=None,
                              stream=None, check=True) -> int:
    """moe_route_permute without a workspace: the scratch is a device array
    inside the library, shared by every call (T*k <= 65536)."""
    if T is None or k is None:
        T, k = topk_ids.shape
    st = lib().moe_route_permute_noalloc(_ptr(topk_ids), T, k, E, _ptr(m_indptr), _ptr(perm),
                                         _ptr(inv_perm), _stream(stream))
    return _check(st, "moe_route_permute_noalloc", check)


def _fused_dims(x, topk_ids, w13):
    T, H = x.shape
    k = topk_ids.shape[1]
    E, I2, _ = w13.shape
    return T, H, I2 // 2, E, k


def moe_fp8_fused(x, topk_ids, topk_w, w13, w13_scale, w2, w2_scale, out, ws, ws_bytes=None, *,
                  dims=None, stream=None, check=True) -> int:
    """dims = (T, H, I, E, k) when raw addresses are passed."""
    T, H, I, E, k = dims if dims is not None else _fused_dims(x, topk_ids, w13)
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    st = lib().moe_fp8_fused(_ptr(x), _ptr(topk_ids), _ptr(topk_w), _ptr(w13), _ptr(w13_scale),
                             _ptr(w2), _ptr(w2_scale), _ptr(out), T, H, I, E, k, _ptr(ws),
                             ws_bytes, _stream(stream))
    return _check(st, "moe_fp8_fused", check)


def moe_fp8_fused_debug(x, topk_ids, topk_w, w13, w13_scale, w2, w2_scale, out, ws,
                        m_indptr=None, perm=None, h_fp8=None, h_scale=None, ws_bytes=None, *,
                        dims=None, stream=None, check=True) -> int:
    T, H, I, E, k = dims if dims is not None else _fused_dims(x, topk_ids, w13)
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    st = lib().moe_fp8_fused_debug(_ptr(x), _ptr(topk_ids), _ptr(topk_w), _ptr(w13),
                                   _ptr(w13_scale), _ptr(w2), _ptr(w2_scale), _ptr(out), T, H, I,
                                   E, k, _ptr(ws), ws_bytes, _stream(stream), _ptr(m_indptr),
                                   _ptr(perm), _ptr(h_fp8), _ptr(h_scale))
    return _check(st, "moe_fp8_fused_debug", check)


def fp8_groupwise_moe_gemm(a, b, a_scale, b_scale, m_indptr, out, scale_major_mode="K",
                           scale_granularity=(1, 128, 128), is_gated=False, tile_m=-1, tile_n=-1,
                           *, dims=None, stream=None, check=True) -> int:
    """scale_major_mode "K": a_scale [R, K/128]; "MN": [K/128, R].
    dims = (R, N, K, E) when raw addresses are passed."""
    if dims is None:
        R, K = a.shape
        E, N, _ = b.shape
    else:
        R, N, K, E = dims
    mode = {"K": 0, "MN": 1}.get(scale_major_mode, scale_major_mode)
    sg_m, sg_n, sg_k = scale_granularity
    st = lib().fp8_groupwise_moe_gemm(_ptr(a), _ptr(b), _ptr(a_scale), _ptr(b_scale),
                                      _ptr(m_indptr), _ptr(out), R, N, K, E, mode, sg_m, sg_n,
                                      sg_k, int(bool(is_gated)), tile_m, tile_n, _stream(stream))
    return _check(st, "fp8_groupwise_moe_gemm", check)


def mxfp8_moe_gemm(a, b, a_sf, b_sf, m_indptr, out, is_gated=False, a_sf_major="K", *,
                   dims=None, stream=None, check=True) -> int:
    """a [R,K] fp8, b [E,N,K] fp8, a_sf [R,K/32] uint8 E8M0 row-major, b_sf the
    weight scales tiled by mxfp8_tile_scales, out bf16 [R, N/2 if gated else N].  dims = (R, N, K, E) when raw addresses
    are passed."""
    if dims is None:
        R, K = a.shape
        E, N, _ = b.shape
    else:
        R, N, K, E = dims
    mode = {"K": 0, "MN": 1}.get(a_sf_major, a_sf_major)
    st = lib().mxfp8_moe_gemm(_ptr(a), _ptr(b), _ptr(a_sf), _ptr(b_sf), _ptr(m_indptr), _ptr(out),
                              R, N, K, E, mode, int(bool(is_gated)), _stream(stream))
    return _check(st, "mxfp8_moe_gemm", check)


def moe_router_topk(logits, topk_ids, topk_w, *, dims=None, stream=None, check=True) -> int:
    """logits fp32 [T, E] -> topk_ids int32 [T, k], topk_w fp32 [T, k].
    dims = (T, E, k) when raw addresses are passed."""
    if dims is None:
        T, E = logits.shape
        k = topk_ids.shape[1]
    else:
        T, E, k = dims
    st = lib().moe_router_topk(_ptr(logits), T, E, k, _ptr(topk_ids), _ptr(topk_w), _stream(stream))
    return _check(st, "moe_router_topk", check)


def moe_mxfp8_fused(x, topk_ids, topk_w, w13, w13_sf, w2, w2_sf, out, ws, ws_bytes=None, *,
                    dims=None, stream=None, check=True) -> int:
    """w13_sf / w2_sf: weight scales tiled by mxfp8_tile_scales.  dims = (T, H, I, E, k)
    when raw addresses are passed."""
    T, H, I, E, k = dims if dims is not None else _fused_dims(x, topk_ids, w13)
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    st = lib().moe_mxfp8_fused(_ptr(x), _ptr(topk_ids), _ptr(topk_w), _ptr(w13), _ptr(w13_sf),
                               _ptr(w2), _ptr(w2_sf), _ptr(out), T, H, I, E, k, _ptr(ws), ws_bytes,
                               _stream(stream))
    return _check(st, "moe_mxfp8_fused", check)


def moe_mxfp8_fused_debug(x, topk_ids, topk_w, w13, w13_sf, w2, w2_sf, out, ws, m_indptr=None,
                          perm=None, h_fp8=None, h_sf=None, ws_bytes=None, *, dims=None,
                          stream=None, check=True) -> int:
    T, H, I, E, k = dims if dims is not None else _fused_dims(x, topk_ids, w13)
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    st = lib().moe_mxfp8_fused_debug(_ptr(x), _ptr(topk_ids), _ptr(topk_w), _ptr(w13),
                                     _ptr(w13_sf), _ptr(w2), _ptr(w2_sf), _ptr(out), T, H, I, E,
                                     k, _ptr(ws), ws_bytes, _stream(stream), _ptr(m_indptr),
                                     _ptr(perm), _ptr(h_fp8), _ptr(h_sf))
    return _check(st, "moe_mxfp8_fused_debug", check)


def mxfp8_tile_scales(sf_rowmajor, sf_tiled, *, dims=None, stream=None, check=True) -> int:
    """sf_rowmajor uint8 [rows, K/32] -> sf_tiled uint8 (rows * K/32 bytes, tiled).
    dims = (rows, K) when raw addresses are passed."""
    if dims is None:
        rows = sf_rowmajor.shape[0] if sf_rowmajor.dim() == 2 else sf_rowmajor.shape[0] * sf_rowmajor.shape[1]
        K = sf_rowmajor.shape[-1] * 32
    else:
        rows, K = dims
    st = lib().mxfp8_tile_scales(_ptr(sf_rowmajor), _ptr(sf_tiled), rows, K, _stream(stream))
    return _check(st, "mxfp8_tile_scales", check)


def nvfp4_moe_gemm(a, b, a_sf, b_sf, alpha, m_indptr, out, is_gated=False, a_sf_major="K", *,
                   dims=None, stream=None, check=True) -> int:
    """a uint8 [R, K/2] packed E2M1, b uint8 [E, N, K/2], a_sf uint8 E4M3
    [R, K/16] ("K") or [K/64, R, 4] ("MN"), b_sf the weight scales tiled by
    nvfp4_tile_scales, alpha fp32 [E], out bf16 [R, N/2 if gated else N].
    dims = (R, N, K, E) when raw addresses are passed."""
    if dims is None:
        R = a.shape[0]
        K = a.shape[1] * 2
        E, N = b.shape[0], b.shape[1]
    else:
        R, N, K, E = dims
    mode = {"K": 0, "MN": 1}.get(a_sf_major, a_sf_major)
    st = lib().nvfp4_moe_gemm(_ptr(a), _ptr(b), _ptr(a_sf), _ptr(b_sf), _ptr(alpha), _ptr(m_indptr),
                              _ptr(out), R, N, K, E, mode, int(bool(is_gated)), _stream(stream))
    return _check(st, "nvfp4_moe_gemm", check)


def moe_tactic_tune_gemm(a, b, a_scale, b_scale, m_indptr, out, scale_major="K",
                         is_gated=False, iters=5, *, dims=None, stream=None) -> int:
    """Times fp8_groupwise_moe_gemm at every tile_m valid for K on these
    buffers (out is overwritten), stores the fastest in the tactic table and
    returns it.  dims = (R, N, K, E) when raw addresses are passed."""
    if dims is None:
        R, K = a.shape
        E, N, _ = b.shape
    else:
        R, N, K, E = dims
    mode = {"K": 0, "MN": 1}.get(scale_major, scale_major)
    tm = ctypes.c_int(0)
    st = lib().moe_tactic_tune_gemm(_ptr(a), _ptr(b), _ptr(a_scale), _ptr(b_scale), _ptr(m_indptr),
                                    _ptr(out), R, N, K, E, mode, int(bool(is_gated)), int(iters),
                                    _stream(stream), ctypes.byref(tm))
    _check(st, "moe_tactic_tune_gemm", True)
    return tm.value


def moe_tactic_lookup(R, N, K, E, is_gated=False):
    """Stored tile_m of the shape class, or None (host only)."""
    tm = ctypes.c_int(0)
    st = lib().moe_tactic_lookup(R, N, K, E, int(bool(is_gated)), ctypes.byref(tm))
    if st == MOE_ERR_NO_TILE_CONFIG:
        return None
    _check(st, "moe_tactic_lookup", True)
    return tm.value


def moe_tactic_store(R, N, K, E, is_gated, tile_m, *, check=True) -> int:
    """Sets the shape class's tile_m (host only)."""
    return _check(lib().moe_tactic_store(R, N, K, E, int(bool(is_gated)), tile_m),
                  "moe_tactic_store", check)


def moe_tactic_clear() -> None:
    lib().moe_tactic_clear()


def nvfp4_quantize(x, gscale, q, sf, *, dims=None, stream=None, check=True) -> int:
    """x bf16 [M, K] -> q uint8 [M, K/2] packed E2M1, sf uint8 [M, K/16] E4M3.
    dims = (M, K) when raw addresses are passed."""
    M, K = dims if dims is not None else x.shape
    st = lib().nvfp4_quantize(_ptr(x), float(gscale), _ptr(q), _ptr(sf), M, K, _stream(stream))
    return _check(st, "nvfp4_quantize", check)


def _nv_fused_dims(x, topk_ids, w13):
    T, H = x.shape
    return T, H, w13.shape[1] // 2, w13.shape[0], topk_ids.shape[1]


def moe_nvfp4_fused(x, topk_ids, topk_w, w13, w13_sf, w13_alpha, w2, w2_sf, w2_alpha, a1_gscale,
                    a2_gscale, out, ws, ws_bytes=None, *, dims=None, stream=None,
                    check=True) -> int:
    """w13 / w2 packed E2M1 [E, 2I, H/2] / [E, H, I/2]; w13_sf / w2_sf tiled by
    nvfp4_tile_scales; *_alpha fp32 [E]; a1_gscale / a2_gscale floats.
    dims = (T, H, I, E, k) when raw addresses are passed."""
    T, H, I, E, k = dims if dims is not None else _nv_fused_dims(x, topk_ids, w13)
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    st = lib().moe_nvfp4_fused(_ptr(x), _ptr(topk_ids), _ptr(topk_w), _ptr(w13), _ptr(w13_sf),
                               _ptr(w13_alpha), _ptr(w2), _ptr(w2_sf), _ptr(w2_alpha),
                               float(a1_gscale), float(a2_gscale), _ptr(out), T, H, I, E, k,
                               _ptr(ws), ws_bytes, _stream(stream))
    return _check(st, "moe_nvfp4_fused", check)


def moe_nvfp4_fused_debug(x, topk_ids, topk_w, w13, w13_sf, w13_alpha, w2, w2_sf, w2_alpha,
                          a1_gscale, a2_gscale, out, ws, m_indptr=None, perm=None, h_fp4=None,
                          h_sf=None, ws_bytes=None, *, dims=None, stream=None, check=True) -> int:
    T, H, I, E, k = dims if dims is not None else _nv_fused_dims(x, topk_ids, w13)
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    st = lib().moe_nvfp4_fused_debug(_ptr(x), _ptr(topk_ids), _ptr(topk_w), _ptr(w13),
                                     _ptr(w13_sf), _ptr(w13_alpha), _ptr(w2), _ptr(w2_sf),
                                     _ptr(w2_alpha), float(a1_gscale), float(a2_gscale),
                                     _ptr(out), T, H, I, E, k, _ptr(ws), ws_bytes,
                                     _stream(stream), _ptr(m_indptr), _ptr(perm), _ptr(h_fp4),
                                     _ptr(h_sf))
    return _check(st, "moe_nvfp4_fused_debug", check)


def nvfp4_tile_scales(sf_rowmajor, sf_tiled, *, dims=None, stream=None, check=True) -> int:
    """sf_rowmajor uint8 [rows, K/16] E4M3 -> sf_tiled uint8 (rows * K/16 bytes, tiled).
    dims = (rows, K) when raw addresses are passed."""
    if dims is None:
        rows = sf_rowmajor.numel() // sf_rowmajor.shape[-1]
        K = sf_rowmajor.shape[-1] * 16
    else:
        rows, K = dims
    st = lib().nvfp4_tile_scales(_ptr(sf_rowmajor), _ptr(sf_tiled), rows, K, _stream(stream))
    return _check(st, "nvfp4_tile_scales", check)


def swiglu_mxfp8_quant(inp, out, scale, *, dims=None, stream=None, check=True) -> int:
    if dims is None:
        M, K2 = inp.shape
        K = K2 // 2
    else:
        M, K = dims
    st = lib().swiglu_mxfp8_quant(_ptr(inp), _ptr(out), _ptr(scale), M, K, _stream(stream))
    return _check(st, "swiglu_mxfp8_quant", check)


def moe_set_stage_events(events) -> int:
    """events: six torch.cuda.Event (timing enabled, already created on the
    device; None entries are not recorded) or None to switch stage timing off."""
    if events is None:
        return _check(lib().moe_set_stage_events(None, 0), "moe_set_stage_events", True)
    handles = (ctypes.c_void_p * len(events))(
        *[ctypes.c_void_p(e.cuda_event if e is not None else None) for e in events])
    return _check(lib().moe_set_stage_events(handles, len(events)), "moe_set_stage_events", True)


def moe_get_device_status(ws=None, *, stream=None) -> int:
    return int(lib().moe_get_device_status(_ptr(ws), _stream(stream)))


# ---------------------------------------------------------------- expert parallelism
def moe_ep_workspace_size(T: int, k: int, G: int) -> int:
    return int(lib().moe_ep_workspace_size(T, k, G))


def moe_ep_plan(topk_ids, E: int, G: int, send_indptr, send_pair, slot_of_pair, ws, ws_bytes=None,
                *, T=None, k=None, stream=None, check=True) -> int:
    if T is None or k is None:
        T, k = topk_ids.shape
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    st = lib().moe_ep_plan(_ptr(topk_ids), T, k, E, G, _ptr(send_indptr), _ptr(send_pair),
                           _ptr(slot_of_pair), _ptr(ws), ws_bytes, _stream(stream))
    return _check(st, "moe_ep_plan", check)


def moe_ep_pack(x, topk_ids, slot_of_pair, E: int, G: int, S: int, xq_send, xs_send, eid_send, *,
                dims=None, stream=None, check=True) -> int:
    """dims = (T, H, k) when raw addresses are passed."""
    if dims is None:
        T, H = x.shape
        k = topk_ids.shape[1]
    else:
        T, H, k = dims
    st = lib().moe_ep_pack(_ptr(x), _ptr(topk_ids), _ptr(slot_of_pair), T, H, k, E, G, S,
                           _ptr(xq_send), _ptr(xs_send), _ptr(eid_send), _stream(stream))
    return _check(st, "moe_ep_pack", check)


def moe_fp8_expert_rows_workspace_size(n: int, H: int, I: int, E: int) -> int:
    return int(lib().moe_fp8_expert_rows_workspace_size(n, H, I, E))


def moe_fp8_expert_rows(xq, xs, eid, w13, w13_scale, w2, w2_scale, y, ws, ws_bytes=None, *,
                        dims=None, stream=None, check=True) -> int:
    """dims = (n, H, I, E) when raw addresses are passed."""
    if dims is None:
        n, H = xq.shape
        E, I2, _ = w13.shape
        I = I2 // 2
    else:
        n, H, I, E = dims
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    st = lib().moe_fp8_expert_rows(_ptr(xq), _ptr(xs), _ptr(eid), n, _ptr(w13), _ptr(w13_scale),
                                   _ptr(w2), _ptr(w2_scale), _ptr(y), H, I, E, _ptr(ws), ws_bytes,
                                   _stream(stream))
    return _check(st, "moe_fp8_expert_rows", check)


def moe_combine(y, row_of_pair, topk_w, out, *, dims=None, stream=None, check=True) -> int:
    """dims = (T, k, H) when raw addresses are passed."""
    if dims is None:
        T, k = topk_w.shape
        H = out.shape[1]
    else:
        T, k, H = dims
    st = lib().moe_combine(_ptr(y), _ptr(row_of_pair), _ptr(topk_w), T, k, H, _ptr(out),
                           _stream(stream))
    return _check(st, "moe_combine", check)
