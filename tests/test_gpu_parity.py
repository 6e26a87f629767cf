"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on
the same seeded inputs.  Needs a B200; run with `-m gpu`."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_route_b200 as moe
import oracle as O
import synth
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


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


DEV = "cuda"


# ------------------------------------------------------------------ routing
def _route_gpu(ids_cpu: torch.Tensor, E: int):
    T, k = ids_cpu.shape
    R = T * k
    ids = ids_cpu.to(DEV)
    guards = {}
    m_indptr, guards["m_indptr"] = G.guarded_empty((E + 1,), torch.int32, DEV, fill=-7)
    perm, guards["perm"] = G.guarded_empty((max(R, 1),), torch.int32, DEV, fill=-7)
    inv, guards["inv_perm"] = G.guarded_empty((max(R, 1),), torch.int32, DEV, fill=-7)
    ws, guards["ws"] = G.guarded_empty((moe.moe_route_workspace_size(T, k, E),), torch.uint8, DEV)
    moe.moe_route_permute(ids, E, m_indptr, perm, inv, ws,
                          ws_bytes=moe.moe_route_workspace_size(T, k, E))
    st = moe.moe_get_device_status(ws)
    G.check_guards(guards, "routing")
    return G.i32(m_indptr), G.i32(perm)[:R], G.i32(inv)[:R], st


@pytest.mark.parametrize("T,k,E,routing", [
    (16, 2, 4, "normal"), (64, 8, 256, "normal"), (512, 8, 128, "normal"),
    (8192, 8, 256, "zipf"), (1000, 6, 1024, "normal"), (1, 1, 1, "normal"),
    (3, 4, 4, "normal"), (300, 1, 7, "zipf"),
])
def test_route_permute_bit_exact(T, k, E, routing):
    g = torch.Generator().manual_seed(T * 31 + E)
    ids, _ = synth.make_routing(T, E, k, routing, g, "cpu")
    m_g, p_g, i_g, st = _route_gpu(ids, E)
    m_o, p_o, i_o, bad = O.route_permute(ids.numpy(), E)
    assert st == moe.MOE_OK and bad == 0
    assert np.array_equal(m_g, m_o)
    assert np.array_equal(p_g, p_o)
    assert np.array_equal(i_g, i_o)


def test_route_permute_empty():
    ids = torch.zeros(0, 8, dtype=torch.int32)
    m_g, _, _, st = _route_gpu(ids, 16)
    assert st == moe.MOE_OK and np.all(m_g == 0)


def test_route_bad_ids_multi_chunk():
    """More than eight 1024-pair chunks: the three-launch path, with bad ids."""
    g = torch.Generator().manual_seed(77)
    ids, _ = synth.make_routing(2000, 64, 8, "normal", g, "cpu")
    ids[5, 3] = -2
    ids[1999, 0] = 64
    m_g, p_g, i_g, st = _route_gpu(ids, 64)
    m_o, p_o, i_o, bad = O.route_permute(ids.numpy(), 64)
    assert st == moe.MOE_ERR_BAD_EXPERT_ID and bad == 2
    assert np.array_equal(m_g, m_o)
    n = int(m_o[-1])
    assert np.array_equal(p_g[:n], p_o[:n])
    assert np.array_equal(i_g, i_o)


def test_route_bad_ids_dropped_and_reported():
    ids = torch.tensor([[0, 5], [1, -1], [2, 3], [9, 1]], dtype=torch.int32)
    m_g, p_g, i_g, st = _route_gpu(ids, 4)
    m_o, p_o, i_o, bad = O.route_permute(ids.numpy(), 4)
    assert st == moe.MOE_ERR_BAD_EXPERT_ID and bad == 3
    assert np.array_equal(m_g, m_o)
    n = int(m_o[-1])
    assert np.array_equal(p_g[:n], p_o[:n])
    assert np.array_equal(i_g, i_o)


# ------------------------------------------------------------------ SwiGLU + MXFP8
@pytest.mark.parametrize("M,K", synth.SWIGLU_SHAPES + ((1, 32), (7, 96), (300, 544)))
@pytest.mark.parametrize("variant", ["normal", "block_scaled"])
def test_swiglu_mxfp8(M, K, variant):
    x = synth.make_swiglu_input(M, K, variant, seed=M + K)
    xd = x.to(DEV)
    out = torch.empty(M, K, dtype=torch.uint8, device=DEV)
    sc = torch.empty(M, K // 32, dtype=torch.uint8, device=DEV)
    moe.swiglu_mxfp8_quant(xd, out, sc)
    assert moe.moe_get_device_status(None) == moe.MOE_OK
    q_o, s_o = O.swiglu_mxfp8(G.bf16_bits(x))
    q_g, s_g = G.u8(out), G.u8(sc)
    # a scale may differ only where the block max sits on a power-of-two
    # boundary (silu's exp differs by an ulp); those blocks are compared by value
    same_scale = s_g == s_o
    assert same_scale.mean() >= G.CODE_MATCH_MIN
    assert np.all(np.abs(s_g.astype(int) - s_o.astype(int)) <= 1)
    blk_ok = np.repeat(same_scale, 32, axis=1)
    G.compare_codes(q_g[blk_ok], q_o[blk_ok], f"mxfp8 {M}x{K} {variant}")
    if (~same_scale).any():
        dq_g = O.e4m3_decode(q_g) * np.repeat(np.exp2(s_g.astype(np.float64) - 127), 32, axis=1)
        dq_o = O.e4m3_decode(q_o) * np.repeat(np.exp2(s_o.astype(np.float64) - 127), 32, axis=1)
        bad = ~blk_ok
        assert np.allclose(dq_g[bad], dq_o[bad], rtol=2**-3, atol=0)


def test_swiglu_mxfp8_empty():
    x = torch.empty(0, 256, dtype=torch.bfloat16, device=DEV)
    out = torch.empty(0, 128, dtype=torch.uint8, device=DEV)
    sc = torch.empty(0, 4, dtype=torch.uint8, device=DEV)
    assert moe.swiglu_mxfp8_quant(x, out, sc, check=False) == moe.MOE_OK


# ------------------------------------------------------------------ grouped GEMM
def _small_int_case(sizes, N, K, seed):
    rng = np.random.default_rng(seed)
    E = len(sizes)
    m_indptr = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    R = int(m_indptr[-1])
    lut = np.array([0x00, 0x38, 0x40, 0x44, 0x48], np.uint8)   # 0,1,2,3,4
    def codes(shape):
        mag = rng.integers(0, 5, size=shape)
        sign = (rng.integers(0, 2, size=shape) * 0x80).astype(np.uint8)
        return (lut[mag] | np.where(mag == 0, 0, sign)).astype(np.uint8)
    a = codes((R, K))
    b = codes((E, N, K))
    # scales 2^-2..2^2 keep every partial and total sum inside fp32's 24 bits
    a_s = np.exp2(rng.integers(-2, 3, size=(R, K // 128))).astype(np.float32)
    b_s = np.exp2(rng.integers(-2, 3, size=(E, N // 128, K // 128))).astype(np.float32)
    return a, a_s, b, b_s, m_indptr


def _run_gemm(a, a_s, b, b_s, m_indptr, gated, tile_m, mode):
    R, K = a.shape
    E, N, _ = b.shape
    a_d = torch.from_numpy(a).to(DEV)
    b_d = torch.from_numpy(b).to(DEV)
    as_d = torch.from_numpy(a_s if mode == "K" else np.ascontiguousarray(a_s.T)).to(DEV)
    bs_d = torch.from_numpy(b_s).to(DEV)
    mi = torch.from_numpy(m_indptr).to(DEV)
    n_out = N // 2 if gated else N
    out, guard = G.guarded_empty((R, n_out), torch.bfloat16, DEV, fill=float("nan"))
    moe.fp8_groupwise_moe_gemm(a_d, b_d, as_d, bs_d, mi, out, mode, (1, 128, 128), gated,
                               tile_m, -1)
    assert moe.moe_get_device_status(None) == moe.MOE_OK
    G.check_guards({"out": guard}, f"grouped GEMM tile_m={tile_m}")
    return G.bf16_bits(out)


@pytest.mark.parametrize("tile_m", [16, 32, 64, 128])
@pytest.mark.parametrize("mode", ["K", "MN"])
def test_gemm_plain_exact_small_integers(tile_m, mode):
    # every sum is exact in fp32: the GPU must reproduce the oracle bit for bit
    a, a_s, b, b_s, mi = _small_int_case([37, 0, 130, 5, 200, 1], N=384, K=384, seed=tile_m)
    got = _run_gemm(a, a_s, b, b_s, mi, False, tile_m, mode)
    ref = O.groupwise_gemm_bf16(a, a_s, b, b_s, mi, False)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("tile_m", [16, 32, 64, 128])
@pytest.mark.parametrize("gated", [False, True])
def test_gemm_random(tile_m, gated):
    sizes = [0, 3, 150, 17, 64, 0, 129, 1]
    inp = synth.make_grouped_gemm_inputs(0, 512, 640, len(sizes), seed=7 + tile_m,
                                         group_sizes=sizes)
    a, a_s, b, b_s, mi = (G.u8(inp["a"]), G.f32(inp["a_scale"]), G.u8(inp["b"]),
                          G.f32(inp["b_scale"]), G.i32(inp["m_indptr"]))
    got = _run_gemm(a, a_s, b, b_s, mi, gated, tile_m, "K")
    ref = O.groupwise_gemm_bf16(a, a_s, b, b_s, mi, gated)
    G.compare_out(got, ref, f"gemm tile_m={tile_m} gated={gated}")
    # the result is within a few bf16 ulps element by element
    g64, r64 = G.bits_to_f64(got), G.bits_to_f64(ref)
    assert np.all(np.abs(g64 - r64) <= 2**-6 * np.abs(r64) + 1e-3 * np.sqrt(np.mean(r64**2)))


def test_gemm_auto_tile_and_large_k():
    inp = synth.make_grouped_gemm_inputs(0, 256, 7168, 3, seed=5, group_sizes=[5, 40, 2])
    a, a_s, b, b_s, mi = (G.u8(inp["a"]), G.f32(inp["a_scale"]), G.u8(inp["b"]),
                          G.f32(inp["b_scale"]), G.i32(inp["m_indptr"]))
    got = _run_gemm(a, a_s, b, b_s, mi, True, -1, "MN")
    ref = O.groupwise_gemm_bf16(a, a_s, b, b_s, mi, True)
    G.compare_out(got, ref, "gemm auto tile K=7168")


# ------------------------------------------------------------------ fused layer
def _check_fused_full(inp, what):
    res = G.run_fused(inp, debug=True)
    assert res["status"] == moe.MOE_OK
    ref = O.moe_fused(*G.oracle_args(inp))
    assert np.array_equal(res["m_indptr"], ref["m_indptr"]), what
    assert np.array_equal(res["perm"], ref["perm"]), what
    G.compare_codes(res["hq"], ref["hq"], what + " intermediate codes")
    G.compare_scales(res["hs"], ref["hs"], what + " intermediate scales")
    G.compare_layer(res, ref, inp, what + " output")


# "off": the two-launch path (GEMM1 then GEMM2); "auto": whatever the plan
# picks for the shape (the fused-expert launch for tiny layers).
@pytest.fixture(params=["off", "auto"])
def fusion(request):
    mode = {"off": moe.MOE_FUSION_OFF, "auto": moe.MOE_FUSION_AUTO}[request.param]
    moe.moe_set_expert_fusion(mode)
    yield request.param
    moe.moe_set_expert_fusion(moe.MOE_FUSION_AUTO)


def test_fused_tiny(fusion):
    inp = synth.make_moe_inputs(synth.CONFIGS["tiny"], seed=0, device=DEV)
    _check_fused_full(inp, f"tiny ({fusion})")


@pytest.mark.parametrize("T,H,I,E,k,routing", [
    (100, 512, 256, 16, 4, "normal"),     # ragged groups, several tiles
    (1, 256, 128, 4, 2, "normal"),        # single token
    (40, 384, 384, 1, 1, "normal"),       # one expert: a dense SwiGLU FFN
    (24, 256, 128, 6, 6, "normal"),       # every expert chosen by every token
    (200, 256, 256, 64, 2, "zipf"),       # many empty experts
    (1000, 256, 128, 8, 2, "zipf"),       # balanced 250 rows/expert: 128-row tiles
    (700, 512, 256, 4, 2, "normal"),      # ~350 rows/expert: 128-row tiles with a ragged tail
    (1500, 256, 256, 3, 1, "zipf"),       # ~500 rows/expert, skewed: several tiles each
])
def test_fused_small_shapes(fusion, T, H, I, E, k, routing):
    cfg = synth.MoEConfig("case", T, H, I, E, k, routing)
    inp = synth.make_moe_inputs(cfg, seed=T + E, device=DEV)
    _check_fused_full(inp, f"T={T} H={H} I={I} E={E} k={k} ({fusion})")


def test_fused_zero_tokens():
    cfg = synth.MoEConfig("empty", 0, 256, 128, 4, 2)
    inp = synth.make_moe_inputs(cfg, seed=1, device=DEV)
    res = G.run_fused(inp, debug=True)
    assert res["status"] == moe.MOE_OK and np.all(res["m_indptr"] == 0)


def test_fused_bad_expert_ids(fusion):
    cfg = synth.MoEConfig("bad", 32, 256, 128, 8, 2)
    inp = synth.make_moe_inputs(cfg, seed=4, device=DEV)
    inp["topk_ids"][3, 1] = -1
    inp["topk_ids"][10, 0] = 8
    res = G.run_fused(inp, debug=True)
    assert res["status"] == moe.MOE_ERR_BAD_EXPERT_ID
    ref = O.moe_fused(*G.oracle_args(inp))
    assert ref["n_bad"] == 2
    assert np.array_equal(res["m_indptr"], ref["m_indptr"])
    n = int(ref["m_indptr"][-1])
    assert np.array_equal(res["perm"][:n], ref["perm"])
    G.compare_layer(res, ref, inp, "bad ids")


def _check_sampled(inp, tokens, what):
    """Full-size check: routing tables exactly, intermediate and output rows
    of the sampled tokens through the per-token oracle."""
    res = G.run_fused(inp, debug=True)
    assert res["status"] == moe.MOE_OK
    E = inp["w13"].shape[0]
    m_o, p_o, i_o, _ = O.route_permute(G.i32(inp["topk_ids"]), E)
    assert np.array_equal(res["m_indptr"], m_o), what
    assert np.array_equal(res["perm"], p_o), what
    sub = synth.compact_experts(inp, tokens)
    out_o, hq_o, hs_o = O.moe_tokens(sub["x"], sub["topk_ids"], sub["topk_w"], sub["w13"],
                                     sub["w13_scale"], sub["w2"], sub["w2_scale"],
                                     np.arange(len(tokens), dtype=np.int32), want_h=True)
    k = inp["topk_ids"].shape[1]
    n = len(tokens)
    rows = np.array([[i_o[t * k + j] for j in range(k)] for t in tokens])
    G.compare_codes(res["hq"][rows.ravel()], hq_o.reshape(n * k, -1), what + " codes")
    G.compare_scales(res["hs"][rows.ravel()], hs_o.reshape(n * k, -1), what + " scales")
    ids = G.i32(inp["topk_ids"])[tokens]
    tw = G.f32(inp["topk_w"])[tokens]
    w2, w2s = G.u8(inp["w2"]), G.f32(inp["w2_scale"])

    def own_h(idx):
        return G.own_h_rows(rows[idx], res["hq"], res["hs"], w2, w2s, ids[idx], tw[idx])

    G.compare_layer_rows(res["out"][tokens], out_o, res["hq"][rows.ravel()].reshape(n, -1),
                         hq_o.reshape(n, -1), own_h, what + " output")


def test_fused_mid_sampled(fusion):
    inp = synth.make_moe_inputs(synth.CONFIGS["mid"], seed=0, device=DEV)
    tokens = list(range(0, 512, 16)) + [511]
    _check_sampled(inp, tokens, f"mid ({fusion})")


def test_fused_two_groups_per_expert_sampled(fusion):
    """~128 rows per expert: two 64-token work items per expert in the
    fused-expert launch (the plan fuses this shape), 128-row tiles otherwise."""
    cfg = synth.MoEConfig("mid2k", 2048, 2048, 768, 128, 8)
    inp = synth.make_moe_inputs(cfg, seed=5, device=DEV)
    _check_sampled(inp, [0, 1, 777, 1500, 2047], f"T=2048 mid shape ({fusion})")


def test_fused_decode_full_size_sampled():
    inp = synth.make_moe_inputs(synth.CONFIGS["decode"], seed=0, device=DEV)
    _check_sampled(inp, [0, 17, 42, 63], "decode")
    del inp
    torch.cuda.empty_cache()


def test_fused_prefill_full_size_sampled():
    inp = synth.make_moe_inputs(synth.CONFIGS["prefill"], seed=0, device=DEV)
    ids = inp["topk_ids"]
    counts = torch.bincount(ids.flatten().long(), minlength=256)
    assert int(counts.max()) > 2000 and int((counts == 0).sum()) >= 1   # skewed as specified
    # tokens routed to the largest and to the smallest non-empty groups
    big = int(torch.argmax(counts))
    nz = torch.nonzero(counts).flatten()
    small = int(nz[torch.argmin(counts[nz])])
    t_big = int(torch.nonzero((ids == big).any(1)).flatten()[0])
    t_small = int(torch.nonzero((ids == small).any(1)).flatten()[0])
    _check_sampled(inp, sorted({0, t_big, t_small, 8191}), "prefill")
    del inp
    torch.cuda.empty_cache()
