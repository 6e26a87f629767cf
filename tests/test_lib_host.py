"""Host-side checks of the C-ABI library that need no GPU: it loads, exports
every declared symbol, its tile selector equals the oracle's, and argument
validation rejects bad calls before touching a device."""
import os
import re

import numpy as np
import pytest

import fp8_block_scaled_route_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from fp8_block_scaled_route_b200 import build
    build.build()
    return moe.lib()


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(\w+)\s*\(", txt))
    return names


def test_exports_every_declared_symbol(L):
    declared = _declared_symbols()
    assert declared == set(moe.EXPORTS)
    for name in declared:
        assert hasattr(L, name), name


def _declared_arg_counts():
    """name -> number of parameters, from the MOE_API declarations."""
    counts = {}
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", fn)).read(),
                         flags=re.S)
            for m in re.finditer(r"MOE_API\s+[\w\s\*]+?\b(\w+)\s*\(([^)]*)\)", txt):
                args = m.group(2).strip()
                counts[m.group(1)] = 0 if args in ("", "void") else args.count(",") + 1
    return counts


def test_binding_signatures_match_header(L):
    """Every ctypes prototype the binding sets has as many parameters as the
    header declares (a missing or extra argument would shift every later one)."""
    for name, n in _declared_arg_counts().items():
        argtypes = getattr(L, name).argtypes
        assert argtypes is not None, f"{name}: no ctypes prototype"
        assert len(argtypes) == n, f"{name}: {len(argtypes)} ctypes arguments, header has {n}"


def test_status_strings(L):
    for code, name in [(0, "MOE_OK"), (1, "MOE_ERR_INVALID_ARG"), (4, "MOE_ERR_NO_TILE_CONFIG"),
                       (5, "MOE_ERR_DEVICE_TIMEOUT"), (6, "MOE_ERR_BAD_EXPERT_ID")]:
        assert moe.moe_status_string(code) == name


def test_stage_event_setter_validation(L):
    import ctypes
    six_null = (ctypes.c_void_p * 6)()
    assert L.moe_set_stage_events(six_null, 6) == moe.MOE_ERR_INVALID_ARG   # nothing to record
    assert L.moe_set_stage_events(six_null, 5) == moe.MOE_ERR_INVALID_ARG   # wrong count
    assert L.moe_set_stage_events(None, 0) == moe.MOE_OK                    # timing off


def test_expert_fusion_mode_setter(L):
    assert L.moe_set_expert_fusion(moe.MOE_FUSION_OFF) == moe.MOE_OK
    assert L.moe_set_expert_fusion(moe.MOE_FUSION_ON) == moe.MOE_OK
    assert L.moe_set_expert_fusion(7) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_set_expert_fusion(-1) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_set_expert_fusion(moe.MOE_FUSION_AUTO) == moe.MOE_OK
    with pytest.raises(moe.MoEError):
        moe.moe_set_expert_fusion(3)


def test_tile_selector_matches_oracle(L, oracle):
    rng = np.random.default_rng(0)
    for _ in range(3000):
        E = int(rng.integers(1, 1025))
        R = int(rng.choice([rng.integers(0, 64), rng.integers(0, 5000), rng.integers(0, 200000)]))
        gated = bool(rng.integers(0, 2))
        n = int(rng.choice([256, 512, 1536, 4096, 7168, 14336]))
        k = int(rng.choice([128, 768, 2048, 4096, 7168]))
        sms = int(rng.choice([148, 132, 8]))
        assert moe.moe_select_tile_m(R, n, k, E, sms, gated) == \
            oracle.select_tile_m(R, n, k, E, sms, gated)


def test_workspace_sizes(L):
    assert moe.moe_workspace_size(0, 256, 128, 4, 2) > 0
    a = moe.moe_workspace_size(16, 256, 128, 4, 2)
    b = moe.moe_workspace_size(32, 256, 128, 4, 2)
    assert b > a
    # xq + hq + scales + combine buffer at least
    T, H, I, E, k = 64, 7168, 2048, 256, 8
    assert moe.moe_workspace_size(T, H, I, E, k) >= T * k * (H + I) + 4 * T * H
    assert moe.moe_workspace_size(-1, 256, 128, 4, 2) == 0
    assert moe.moe_route_workspace_size(16, 2, 4) > 0


FAKE = 1 << 20  # an aligned address never dereferenced: validation fails first


def _fused(T=16, H=256, I=128, E=4, k=2, ws_bytes=1 << 30, x=FAKE, ws=FAKE):
    return moe.moe_fp8_fused(x, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws, ws_bytes,
                             dims=(T, H, I, E, k), stream=0, check=False)


def test_fused_rejects_bad_arguments(L):
    assert _fused(H=200) == moe.MOE_ERR_INVALID_ARG
    assert _fused(I=100) == moe.MOE_ERR_INVALID_ARG
    assert _fused(k=5, E=4) == moe.MOE_ERR_INVALID_ARG
    assert _fused(k=0) == moe.MOE_ERR_INVALID_ARG
    assert _fused(E=0) == moe.MOE_ERR_INVALID_ARG
    assert _fused(E=2000, k=2) == moe.MOE_ERR_UNSUPPORTED
    assert _fused(T=-1) == moe.MOE_ERR_INVALID_ARG
    assert _fused(ws_bytes=10) == moe.MOE_ERR_INVALID_ARG
    assert _fused(x=FAKE + 2) == moe.MOE_ERR_INVALID_ARG
    assert _fused(x=0) == moe.MOE_ERR_INVALID_ARG


def _gemm(R=64, N=256, K=256, E=4, mode=0, sg=(1, 128, 128), gated=0, tm=-1, tn=-1):
    return moe.fp8_groupwise_moe_gemm(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, mode, sg, gated, tm, tn,
                                      dims=(R, N, K, E), stream=0, check=False)


def test_gemm_rejects_bad_arguments(L):
    assert _gemm(sg=(1, 64, 128)) == moe.MOE_ERR_UNSUPPORTED
    assert _gemm(sg=(128, 128, 128)) == moe.MOE_ERR_UNSUPPORTED
    assert _gemm(tm=48) == moe.MOE_ERR_NO_TILE_CONFIG
    assert _gemm(tn=64) == moe.MOE_ERR_NO_TILE_CONFIG
    assert _gemm(gated=1, tn=256) == moe.MOE_ERR_NO_TILE_CONFIG
    assert _gemm(gated=1, N=384) == moe.MOE_ERR_INVALID_ARG      # N/2 not a multiple of 128
    assert _gemm(N=200) == moe.MOE_ERR_INVALID_ARG
    assert _gemm(K=100) == moe.MOE_ERR_INVALID_ARG
    assert _gemm(mode=2) == moe.MOE_ERR_INVALID_ARG
    assert _gemm(E=4096) == moe.MOE_ERR_UNSUPPORTED


def test_swiglu_and_route_reject_bad_arguments(L):
    assert moe.swiglu_mxfp8_quant(FAKE, FAKE, FAKE, dims=(4, 48), stream=0, check=False) == \
        moe.MOE_ERR_INVALID_ARG
    assert moe.swiglu_mxfp8_quant(FAKE, FAKE, FAKE, dims=(-1, 64), stream=0, check=False) == \
        moe.MOE_ERR_INVALID_ARG
    assert moe.moe_route_permute(FAKE, 2000, FAKE, FAKE, None, FAKE, 1 << 20, T=4, k=2, stream=0,
                                 check=False) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_route_permute(FAKE, 8, FAKE, FAKE, None, FAKE, 4, T=4, k=2, stream=0,
                                 check=False) == moe.MOE_ERR_INVALID_ARG


def test_mxfp8_entry_points_reject_bad_arguments(L):
    def mx(R=64, N=256, K=256, E=4, mode=0, gated=0, a_sf=FAKE, b_sf=FAKE):
        return moe.mxfp8_moe_gemm(FAKE, FAKE, a_sf, b_sf, FAKE, FAKE, gated, mode,
                                  dims=(R, N, K, E), stream=0, check=False)
    assert mx(K=96) == moe.MOE_ERR_INVALID_ARG          # K not a multiple of 128
    assert mx(N=200) == moe.MOE_ERR_INVALID_ARG
    assert mx(gated=1, N=384) == moe.MOE_ERR_INVALID_ARG
    assert mx(mode=2) == moe.MOE_ERR_INVALID_ARG
    assert mx(a_sf=FAKE + 2) == moe.MOE_ERR_INVALID_ARG  # activation scales 4-byte aligned
    assert mx(b_sf=FAKE + 4) == moe.MOE_ERR_INVALID_ARG  # tiled weight scales 16-byte aligned
    assert mx(E=4096) == moe.MOE_ERR_UNSUPPORTED
    assert moe.mxfp8_tile_scales(FAKE, FAKE, dims=(100, 256), stream=0, check=False) == \
        moe.MOE_ERR_INVALID_ARG                          # rows not a multiple of 128
    assert moe.mxfp8_tile_scales(FAKE, FAKE, dims=(128, 96), stream=0, check=False) == \
        moe.MOE_ERR_INVALID_ARG
    ws = moe.moe_workspace_size(8, 256, 128, 4, 2)
    assert moe.moe_mxfp8_fused(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws,
                               dims=(8, 200, 128, 4, 2), stream=0, check=False) == \
        moe.MOE_ERR_INVALID_ARG
    assert moe.moe_mxfp8_fused(FAKE, FAKE, FAKE, FAKE, FAKE + 4, FAKE, FAKE, FAKE, FAKE, ws,
                               dims=(8, 256, 128, 4, 2), stream=0, check=False) == \
        moe.MOE_ERR_INVALID_ARG                          # weight scales 16-byte aligned
    assert moe.moe_mxfp8_fused(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 10,
                               dims=(8, 256, 128, 4, 2), stream=0, check=False) == \
        moe.MOE_ERR_INVALID_ARG                          # workspace too small


def test_router_rejects_bad_arguments(L):
    def r(T=8, E=64, k=4):
        return moe.moe_router_topk(FAKE, FAKE, FAKE, dims=(T, E, k), stream=0, check=False)
    assert r(k=0) == moe.MOE_ERR_INVALID_ARG
    assert r(k=65) == moe.MOE_ERR_INVALID_ARG            # k > E
    assert r(E=128, k=33) == moe.MOE_ERR_INVALID_ARG     # k above the router's limit
    assert r(T=-1) == moe.MOE_ERR_INVALID_ARG
    assert r(E=2048, k=4) == moe.MOE_ERR_UNSUPPORTED


def test_product_path_does_not_touch_oracle():
    """The binding and the CUDA sources never import, link or name the oracle."""
    pkg = os.path.join(ROOT, "fp8_block_scaled_route_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                txt = open(os.path.join(dirpath, fn)).read()
                assert "oracle" not in txt.lower(), fn


def test_expert_parallel_entry_points_reject_bad_arguments(L):
    ws = 1 << 20
    assert moe.moe_ep_plan(FAKE, 10, 4, FAKE, FAKE, FAKE, FAKE, ws, T=8, k=2, stream=0,
                           check=False) == moe.MOE_ERR_INVALID_ARG      # E % G != 0
    assert moe.moe_ep_plan(FAKE, 8, 4, FAKE, FAKE, FAKE, FAKE, 16, T=8, k=2, stream=0,
                           check=False) == moe.MOE_ERR_INVALID_ARG      # workspace too small
    assert moe.moe_ep_pack(FAKE, FAKE, FAKE, 8, 4, 16, FAKE, FAKE, FAKE, dims=(8, 200, 2),
                           stream=0, check=False) == moe.MOE_ERR_INVALID_ARG  # H % 128
    assert moe.moe_fp8_expert_rows(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws,
                                   dims=(16, 256, 100, 4), stream=0, check=False) == \
        moe.MOE_ERR_INVALID_ARG                                          # I % 128
    assert moe.moe_fp8_expert_rows(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 64,
                                   dims=(16, 256, 128, 4), stream=0, check=False) == \
        moe.MOE_ERR_INVALID_ARG                                          # workspace too small
    assert moe.moe_combine(FAKE, FAKE, FAKE, FAKE, dims=(4, 2, 12), stream=0, check=False) == \
        moe.MOE_ERR_INVALID_ARG                                          # H % 8
    assert moe.moe_ep_workspace_size(16, 2, 4) > 0
    assert moe.moe_fp8_expert_rows_workspace_size(16, 256, 128, 4) > 0
