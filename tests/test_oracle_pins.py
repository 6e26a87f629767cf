"""Pins of the CPU oracle against facts that do not come from the oracle:
format tables, closed forms, brute force, library routines and the
invariants the method fixes.  CPU only.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _torch_e4m3_decode_all():
    codes = torch.arange(256, dtype=torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float32).numpy()


# ------------------------------------------------------------ FP8 E4M3 codec
def test_e4m3_spec_table(oracle):
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "e4m3_spec_values.txt"))
            if ln.strip() and not ln.startswith("#")]
    for code_hex, val in rows:
        c = int(code_hex, 16)
        got = float(oracle.e4m3_decode([c])[0])
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))
            assert int(oracle.e4m3_encode([float(val)])[0]) == c


def test_e4m3_decode_matches_torch_all_codes(oracle):
    ours = oracle.e4m3_decode(np.arange(256))
    ref = _torch_e4m3_decode_all()
    finite = ~np.isnan(ref)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    assert np.array_equal(ours[finite], ref[finite])


def test_e4m3_roundtrip_every_code(oracle):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = oracle.e4m3_decode(codes)
    assert np.array_equal(oracle.e4m3_encode(vals), codes)


def test_e4m3_midpoints_round_to_even(oracle):
    pos = np.arange(0, 0x7F)                     # 0 .. 0x7E: +0 .. 448
    v = oracle.e4m3_decode(pos).astype(np.float64)
    mids = (v[:-1] + v[1:]) / 2                  # exact in fp32 (few mantissa bits)
    got = oracle.e4m3_encode(mids.astype(np.float32)).astype(int)
    lo, hi = pos[:-1], pos[1:]
    want = np.where(lo % 2 == 0, lo, hi)
    assert np.array_equal(got, want)
    assert np.array_equal(oracle.e4m3_encode(-mids.astype(np.float32)).astype(int), want | 0x80)


def test_e4m3_encode_bruteforce_and_torch(oracle):
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(3000) * 40.0,
        rng.uniform(-0.03, 0.03, 2000),          # subnormal / small-normal range
        rng.uniform(-448, 448, 2000),
    ]).astype(np.float32)
    got = oracle.e4m3_encode(vals)
    table = oracle.e4m3_decode(np.arange(0x7F)).astype(np.float64)   # non-negative finite
    a = np.abs(vals.astype(np.float64))
    dist = np.abs(a[:, None] - table[None, :])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    # nearest code; on a tie the even code
    choice = np.where(cand.sum(1) > 1, np.argmax(cand & (np.arange(0x7F) % 2 == 0), axis=1),
                      np.argmax(cand, axis=1))
    want = choice | np.where(np.signbit(vals), 0x80, 0)
    assert np.array_equal(got.astype(int), want)
    t = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, t)


def test_e4m3_saturates(oracle):
    got = oracle.e4m3_encode(np.array([448.0, 449.0, 463.9, 470.0, 1e6, np.inf, -1e6], np.float32))
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


# ------------------------------------------------------------ E8M0
def test_e8m0_decode(oracle):
    for c in range(0, 255, 7):
        assert oracle.e8m0_decode(c) == math.ldexp(1.0, c - 127)
    assert oracle.e8m0_decode(127) == 1.0
    assert math.isnan(oracle.e8m0_decode(255))


def test_e8m0_scale_rule_bruteforce(oracle):
    rng = np.random.default_rng(2)
    amaxes = np.concatenate([np.exp(rng.uniform(-60, 60, 3000)),
                             448.0 * np.exp2(np.arange(-20, 20)),          # exact boundaries
                             448.0 * np.exp2(np.arange(-20, 20)) * (1 + 2**-20)]).astype(np.float32)
    for a in amaxes:
        c = oracle.e8m0_scale_code(float(a))
        s = c - 127
        assert float(a) <= 448.0 * 2.0 ** s
        assert float(a) > 448.0 * 2.0 ** (s - 1)
    assert oracle.e8m0_scale_code(0.0) == 0


# ------------------------------------------------------------ quantisers
def test_quant_roundtrip_representable(oracle):
    rng = np.random.default_rng(3)
    rows, cols = 6, 512
    codes = rng.integers(0, 0x7E, size=(rows, cols)).astype(np.uint8)
    codes |= (rng.integers(0, 2, size=(rows, cols)) * 0x80).astype(np.uint8)
    codes[:, ::128] = 0x7E                         # each block holds +-448
    exps = rng.integers(-10, 10, size=(rows, cols // 128))
    scale = np.exp2(exps).astype(np.float32)
    x = oracle.e4m3_decode(codes) * np.repeat(scale, 128, axis=1)
    q, s = oracle.quant_rows_128(x)
    assert np.array_equal(s, scale)
    assert np.array_equal(q, codes)


def test_quant_block_max_decodes_to_448(oracle):
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((8, 1024)) * 3).astype(np.float32)
    q, s = oracle.quant_rows_128(x)
    dq = np.abs(oracle.e4m3_decode(q)).reshape(8, 8, 128)
    assert np.all(dq.max(axis=2) == 448.0)
    # dequantised values sit within half a quantum (relative 2^-4) of the input
    rec = oracle.e4m3_decode(q) * np.repeat(s, 128, axis=1)
    assert np.all(np.abs(rec - x) <= np.abs(x) * 2**-4 + np.repeat(s, 128, axis=1) * 2**-10)


def test_quant_zero_block(oracle):
    x = np.zeros((2, 256), np.float32)
    x[1, 128:] = 1.0
    q, s = oracle.quant_rows_128(x)
    assert s[0, 0] == 1.0 and s[0, 1] == 1.0 and s[1, 0] == 1.0
    assert np.all(q[0] == 0) and np.all(q[1, :128] == 0)
    assert s[1, 1] == np.float32(1.0) / np.float32(448.0)


def test_quant_bf16_matches_fp32_path(oracle):
    t = torch.randn(5, 384, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    q1, s1 = oracle.quant_rows_128_bf16(_bf16_bits(t))
    q2, s2 = oracle.quant_rows_128(t.to(torch.float32).numpy())
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


# ------------------------------------------------------------ routing
@pytest.mark.parametrize("T,k,E,seed", [(16, 2, 4, 0), (64, 8, 256, 1), (33, 3, 5, 2),
                                        (1, 1, 1, 3), (0, 2, 4, 4), (40, 4, 1024, 5)])
def test_route_permute_bruteforce(oracle, T, k, E, seed):
    rng = np.random.default_rng(seed)
    ids = np.array([rng.permutation(E)[:k] for _ in range(T)], np.int32).reshape(T, k)
    m_indptr, perm, inv_perm, bad = oracle.route_permute(ids, E)
    R = T * k
    assert bad == 0
    assert m_indptr[0] == 0 and m_indptr[E] == R
    assert np.all(np.diff(m_indptr) >= 0)
    assert sorted(perm.tolist()) == list(range(R))            # bijection
    flat = ids.ravel()
    for e in range(E):
        grp = perm[m_indptr[e]:m_indptr[e + 1]]
        assert np.all(flat[grp] == e)
        assert np.all(np.diff(grp) > 0)                          # stable: ascending pair id
        assert len(grp) == int(np.sum(flat == e))
    for p in range(R):
        assert perm[inv_perm[p]] == p


def test_route_bad_ids_counted(oracle):
    ids = np.array([[0, 5], [1, -1], [2, 3]], np.int32)
    m_indptr, perm, inv_perm, bad = oracle.route_permute(ids, 4)
    assert bad == 2 and m_indptr[4] == 4
    assert inv_perm[1] == -1 and inv_perm[3] == -1


# ------------------------------------------------------------ grouped GEMM
def _small_int_codes(rng, shape):
    # E4M3 codes of the integers -4..4 (exact): 0, 1=0x38, 2=0x40, 3=0x44, 4=0x48
    lut = np.array([0x00, 0x38, 0x40, 0x44, 0x48], np.uint8)
    mag = rng.integers(0, 5, size=shape)
    sign = rng.integers(0, 2, size=shape).astype(np.uint8) * 0x80
    return (lut[mag] | np.where(mag == 0, 0, sign)).astype(np.uint8), \
        np.where(sign > 0, -mag, mag).astype(np.int64)


def test_grouped_gemm_exact_small_integers(oracle):
    rng = np.random.default_rng(6)
    E, N, K = 3, 256, 384
    sizes = [5, 0, 11]
    m_indptr = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    R = int(m_indptr[-1])
    a, ai = _small_int_codes(rng, (R, K))
    b, bi = _small_int_codes(rng, (E, N, K))
    a_s = np.exp2(rng.integers(-3, 4, size=(R, K // 128))).astype(np.float32)
    b_s = np.exp2(rng.integers(-3, 4, size=(E, N // 128, K // 128))).astype(np.float32)
    out = oracle.grouped_gemm(a, a_s, b, b_s, m_indptr)
    want = np.zeros((R, N))
    for e in range(E):
        for r in range(m_indptr[e], m_indptr[e + 1]):
            for kb in range(K // 128):
                blk = ai[r, kb * 128:(kb + 1) * 128] @ bi[e, :, kb * 128:(kb + 1) * 128].T
                want[r] += blk * a_s[r, kb] * np.repeat(b_s[e, :, kb], 128)
    assert np.array_equal(out.astype(np.float64), want)


def test_grouped_gemm_single_block_is_dot(oracle):
    rng = np.random.default_rng(7)
    R, N, K = 4, 128, 128
    a = rng.integers(0, 0x7E, size=(R, K)).astype(np.uint8)
    b = rng.integers(0, 0x7E, size=(1, N, K)).astype(np.uint8)
    a_s = np.ones((R, 1), np.float32)
    b_s = np.ones((1, 1, 1), np.float32)
    out = oracle.grouped_gemm(a, a_s, b, b_s, np.array([0, R], np.int32))
    ref = oracle.e4m3_decode(a).astype(np.float64) @ oracle.e4m3_decode(b[0]).astype(np.float64).T
    np.testing.assert_allclose(out, ref, rtol=1e-6, atol=1e-6 * np.abs(ref).max())


# ------------------------------------------------------------ whole layer
def _fp64_layer_torch(inp):
    """Dense fp64 restatement with torch ops (matmul on dequantised operands,
    torch's float8 cast for the requantisation).  Only for E=1, top-1, w=1."""
    x = inp["x"].to(torch.float64)
    T, H = x.shape
    blocks = x.view(T, H // 128, 128)
    amax = blocks.abs().amax(2).to(torch.float32)
    s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    xq = (blocks.to(torch.float32) / s[:, :, None]).to(torch.float8_e4m3fn)
    xd = (xq.to(torch.float64) * s[:, :, None].to(torch.float64)).view(T, H)
    w13 = inp["w13"][0].to(torch.float64)
    N2 = w13.shape[0]
    w13d = (w13.view(N2 // 128, 128, H // 128, 128) *
            inp["w13_scale"][0].to(torch.float64)[:, None, :, None]).view(N2, H)
    g = xd @ w13d.T
    I = N2 // 2
    h = (g[:, :I] / (1 + torch.exp(-g[:, :I]))) * g[:, I:]
    hb = h.view(T, I // 128, 128)
    hamax = hb.abs().amax(2).to(torch.float32)
    hs = torch.where(hamax > 0, hamax / 448.0, torch.ones_like(hamax))
    hq = (hb.to(torch.float32) / hs[:, :, None]).to(torch.float8_e4m3fn)
    hd = (hq.to(torch.float64) * hs[:, :, None].to(torch.float64)).view(T, I)
    w2 = inp["w2"][0].to(torch.float64)
    w2d = (w2.view(H // 128, 128, I // 128, 128) *
           inp["w2_scale"][0].to(torch.float64)[:, None, :, None]).view(H, I)
    return hd @ w2d.T, hq.view(T, I)


def test_layer_reduces_to_dense_ffn(oracle):
    cfg = synth.MoEConfig("dense", 24, 256, 256, 1, 1)
    inp = synth.make_moe_inputs(cfg, seed=11)
    inp["topk_w"] = torch.ones_like(inp["topk_w"])
    res = oracle.moe_fused(_bf16_bits(inp["x"]), inp["topk_ids"].numpy(), inp["topk_w"].numpy(),
                           inp["w13"].view(torch.uint8).numpy(), inp["w13_scale"].numpy(),
                           inp["w2"].view(torch.uint8).numpy(), inp["w2_scale"].numpy())
    ref, hq_ref = _fp64_layer_torch(inp)
    got = torch.from_numpy(res["out"].view(np.int16)).view(torch.bfloat16).to(torch.float64)
    err = (got - ref).norm() / ref.norm()
    assert err < 4e-3, err                     # bf16 output rounding + requant flips
    same = (torch.from_numpy(res["hq"]) == hq_ref.view(torch.uint8)).float().mean()
    assert same > 0.99


def test_pertoken_equals_grouped(oracle):
    cfg = synth.CONFIGS["tiny"]
    inp = synth.make_moe_inputs(cfg, seed=0)
    args = (_bf16_bits(inp["x"]), inp["topk_ids"].numpy(), inp["topk_w"].numpy(),
            inp["w13"].view(torch.uint8).numpy(), inp["w13_scale"].numpy(),
            inp["w2"].view(torch.uint8).numpy(), inp["w2_scale"].numpy())
    res = oracle.moe_fused(*args)
    toks = np.arange(cfg.T, dtype=np.int32)
    out, hq, hs = oracle.moe_tokens(*args, toks, want_h=True)
    assert np.array_equal(out, res["out"])
    inv = np.empty(cfg.R, np.int64)
    inv[res["perm"]] = np.arange(cfg.R)
    assert np.array_equal(hq.reshape(cfg.R, -1), res["hq"][inv])
    assert np.array_equal(hs.reshape(cfg.R, -1), res["hs"][inv])


def test_layer_linear_in_router_weight(oracle):
    """Scaling every router weight by 2 doubles the output exactly."""
    cfg = synth.CONFIGS["tiny"]
    inp = synth.make_moe_inputs(cfg, seed=3)
    base = (_bf16_bits(inp["x"]), inp["topk_ids"].numpy())
    rest = (inp["w13"].view(torch.uint8).numpy(), inp["w13_scale"].numpy(),
            inp["w2"].view(torch.uint8).numpy(), inp["w2_scale"].numpy())
    toks = np.arange(cfg.T, dtype=np.int32)
    o1 = oracle.moe_tokens(*base, inp["topk_w"].numpy(), *rest, toks)
    o2 = oracle.moe_tokens(*base, inp["topk_w"].numpy() * 2, *rest, toks)
    f1 = torch.from_numpy(o1.view(np.int16)).view(torch.bfloat16).float()
    f2 = torch.from_numpy(o2.view(np.int16)).view(torch.bfloat16).float()
    assert torch.equal(f2, 2 * f1)


def test_gated_gemm_matches_swiglu_of_plain(oracle):
    inp = synth.make_grouped_gemm_inputs(40, 512, 256, 3, seed=8)
    a = inp["a"].view(torch.uint8).numpy(); b = inp["b"].view(torch.uint8).numpy()
    plain = oracle.grouped_gemm(a, inp["a_scale"].numpy(), b, inp["b_scale"].numpy(),
                                inp["m_indptr"].numpy())
    gated = oracle.groupwise_gemm_bf16(a, inp["a_scale"].numpy(), b, inp["b_scale"].numpy(),
                                       inp["m_indptr"].numpy(), True)
    g = torch.from_numpy(plain).double()
    h = g[:, :256] / (1 + torch.exp(-g[:, :256])) * g[:, 256:]
    got = torch.from_numpy(gated.view(np.int16)).view(torch.bfloat16).double()
    assert torch.allclose(got, h, rtol=2**-8, atol=1e-6)


# ------------------------------------------------------------ SwiGLU + MXFP8
def test_swiglu_mxfp8_scale_rule_and_accuracy(oracle):
    x = synth.make_swiglu_input(16, 256, "block_scaled", seed=9)
    q, sc = oracle.swiglu_mxfp8(_bf16_bits(x))
    xf = x.to(torch.float64)
    v = (xf[:, :256] / (1 + torch.exp(-xf[:, :256])) * xf[:, 256:]).numpy()
    X = np.exp2(sc.astype(np.float64) - 127)
    dq = oracle.e4m3_decode(q).astype(np.float64) * np.repeat(X, 32, axis=1)
    vb = np.abs(v).reshape(16, 8, 32).max(2)
    # scale rule: block max fits under 448*X and not under 224*X
    assert np.all(vb <= 448 * X * (1 + 1e-6)) and np.all(vb > 224 * X * (1 - 1e-6))
    # each value within half an E4M3 quantum of silu(g)*u (plus fp32 rounding)
    quantum = np.maximum(np.exp2(np.floor(np.log2(np.maximum(np.abs(v), 1e-300))) - 3),
                         np.repeat(X, 32, axis=1) * 2**-9)
    assert np.all(np.abs(dq - v) <= 0.5 * quantum + 1e-6 * np.abs(v))
    mx = np.abs(oracle.e4m3_decode(q)).reshape(16, 8, 32).max(2)
    # block max lies in (224, 448] before rounding, so its code decodes to [224, 448]
    assert np.all((mx >= 224) & (mx <= 448))


def test_swiglu_mxfp8_block_permutation(oracle):
    x = synth.make_swiglu_input(4, 128, "normal", seed=10)
    bits = _bf16_bits(x)
    q, sc = oracle.swiglu_mxfp8(bits)
    order = np.array([2, 0, 3, 1])
    g = bits[:, :128].reshape(4, 4, 32)[:, order].reshape(4, 128)
    u = bits[:, 128:].reshape(4, 4, 32)[:, order].reshape(4, 128)
    q2, sc2 = oracle.swiglu_mxfp8(np.concatenate([g, u], axis=1))
    assert np.array_equal(q2, q.reshape(4, 4, 32)[:, order].reshape(4, 128))
    assert np.array_equal(sc2, sc[:, order])


# ------------------------------------------------------------ tile selection
def test_tile_select_page_cases(oracle):
    d = json.load(open(os.path.join(GOLDEN, "tile_select_page_cases.json")))
    for c in d["cases"]:
        tm, _ = oracle.select_tile_m(c["total_rows"], c["n"], c["k"], c["E"], 148,
                                     bool(c["is_gated"]))
        assert tm == c["tile_m"], c["why"]


def test_balanced_tile_count_bruteforce(oracle):
    rng = np.random.default_rng(12)
    for _ in range(200):
        E = int(rng.integers(1, 300)); R = int(rng.integers(0, 20000))
        tm = int(rng.choice([16, 32, 64, 128])); n = int(rng.choice([128, 256, 1024, 7168]))
        sizes = [R // E + (1 if e < R % E else 0) for e in range(E)]
        want = sum(-(-s // tm) for s in sizes) * (-(-n // 128))
        assert oracle.balanced_tile_count(R, n, E, tm, 128) == want
        assert oracle.balanced_max_rows(R, E) == max(sizes)


# ------------------------------------------------------------ router (top-k + softmax)
@pytest.mark.parametrize("T,E,k,seed", [(64, 256, 8, 0), (17, 5, 5, 1), (40, 1024, 3, 2), (9, 4, 1, 3)])
def test_router_topk_bruteforce(oracle, T, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    logits = torch.randn(T, E, generator=g)
    # a few exact ties inside the selected set and at its edge
    logits[0, 1] = logits[0, 0]
    logits[1, E - 1] = logits[1, 0]
    ids, w = oracle.router_topk(logits.numpy(), k)
    for t in range(T):
        # descending logit, ties to the lower index: a stable sort on -logit
        order = np.argsort(-logits[t].numpy().astype(np.float64), kind="stable")[:k]
        np.testing.assert_array_equal(ids[t], order)
        sel = logits[t].numpy().astype(np.float64)[order]
        ref = np.exp(sel - sel.max())
        ref /= ref.sum()
        np.testing.assert_allclose(w[t], ref, rtol=2e-6, atol=1e-9)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-6)


def test_router_matches_generator_for_normal_logits(oracle):
    # the input generator draws routing with torch.topk + softmax; with
    # continuous logits (no ties) the oracle's router gives the same ids
    g = torch.Generator().manual_seed(5)
    logits = torch.randn(32, 64, generator=g)
    top_v, top_i = torch.topk(logits, 4, dim=1, largest=True, sorted=True)
    ids, w = oracle.router_topk(logits.numpy(), 4)
    np.testing.assert_array_equal(ids, top_i.numpy())
    np.testing.assert_allclose(w, torch.softmax(top_v, dim=1).numpy(), rtol=2e-6)
