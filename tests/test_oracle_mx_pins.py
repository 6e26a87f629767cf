"""Pins of the oracle's MXFP8 variant (E8M0 scale per 32 K elements on both
operands; Wave page, section "들어가며", and the Cake-act page's scale rule)
against facts that do not come from the oracle: exact power-of-two scaling,
the format's rounding bound, a float64 library matmul of the decoded
operands, and exact small-integer products.  CPU only.
"""
import numpy as np
import pytest
import torch


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _e4m3_table():
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _dequant(q, sf):
    """Decoded value of every element: E4M3 code (torch's table) x 2^(sf-127)."""
    vals = _e4m3_table()[q.astype(np.int64)]
    return vals * np.exp2(np.repeat(sf.astype(np.float64) - 127.0, 32, axis=-1))


def test_mx_quant_scale_rule(oracle):
    # amax exactly 448 * 2^s -> code s + 127; just above -> s + 128
    for s in (-6, -1, 0, 3):
        x = torch.zeros(1, 32, dtype=torch.float32)
        x[0, 5] = 448.0 * 2.0 ** s
        q, sf = oracle.quant_rows_mx_bf16(_bf16_bits(x.to(torch.bfloat16)))
        assert sf[0, 0] == s + 127
        assert q[0, 5] == 0x7E  # 448 = largest finite E4M3
        x[0, 5] = 450.0 * 2.0 ** s  # next bf16 value above 448 * 2^s
        q, sf = oracle.quant_rows_mx_bf16(_bf16_bits(x.to(torch.bfloat16)))
        assert sf[0, 0] == s + 128


def test_mx_quant_zero_block(oracle):
    x = torch.zeros(3, 64, dtype=torch.bfloat16)
    q, sf = oracle.quant_rows_mx_bf16(_bf16_bits(x))
    assert not q.any() and not sf.any()


def test_mx_quant_powers_of_two_exact(oracle):
    # signed powers of two within 2^8 of the block maximum are E4M3 values
    # after an exact power-of-two scaling: they round-trip exactly
    rng = np.random.default_rng(0)
    e = rng.integers(-8, 1, size=(4, 96))
    sign = rng.choice([-1.0, 1.0], size=e.shape)
    x = torch.tensor(sign * np.exp2(e + 3.0), dtype=torch.float32)
    q, sf = oracle.quant_rows_mx_bf16(_bf16_bits(x.to(torch.bfloat16)))
    np.testing.assert_array_equal(_dequant(q, sf), x.numpy().astype(np.float64))


def test_mx_quant_rounding_bound(oracle):
    # E4M3 keeps 3 fraction bits: normal values are within half an ulp
    # (2^-4 relative); values below the normal range of the scaled block are
    # within half the subnormal step 2^-9 * X
    g = torch.Generator().manual_seed(1)
    x = torch.randn(16, 256, generator=g) * torch.exp2(torch.randint(-6, 6, (16, 8), generator=g)
                                                       .float().repeat_interleave(32, dim=1))
    xb = x.to(torch.bfloat16)
    q, sf = oracle.quant_rows_mx_bf16(_bf16_bits(xb))
    deq = _dequant(q, sf)
    ref = xb.to(torch.float64).numpy()
    X = np.exp2(np.repeat(sf.astype(np.float64) - 127.0, 32, axis=1))
    bound = np.maximum(np.abs(ref) * 2.0 ** -4, X * 2.0 ** -10)
    assert np.all(np.abs(deq - ref) <= bound * (1 + 1e-12))
    # the block maximum never saturates: its scaled magnitude lies in (224, 448]
    amax = np.abs(ref).reshape(16, 8, 32).max(axis=2)
    scaled = amax / np.exp2(sf.astype(np.float64) - 127.0)
    assert np.all((scaled > 224.0) & (scaled <= 448.0))


def _mx_operands(seed, R, N, K, E):
    g = torch.Generator().manual_seed(seed)
    q_a = torch.randint(0, 256, (R, K), generator=g, dtype=torch.int32).numpy().astype(np.uint8)
    q_b = torch.randint(0, 256, (E, N, K), generator=g, dtype=torch.int32).numpy().astype(np.uint8)
    # drop NaN codes (S.1111.111)
    q_a[(q_a & 0x7F) == 0x7F] = 0
    q_b[(q_b & 0x7F) == 0x7F] = 0
    sf_a = torch.randint(120, 134, (R, K // 32), generator=g).numpy().astype(np.uint8)
    sf_b = torch.randint(120, 134, (E, N, K // 32), generator=g).numpy().astype(np.uint8)
    return q_a, sf_a, q_b, sf_b


def test_mx_gemm_matches_float64_matmul(oracle):
    R, N, K, E = 40, 48, 160, 3
    q_a, sf_a, q_b, sf_b = _mx_operands(2, R, N, K, E)
    m_indptr = np.array([0, 7, 7, 33], np.int32)  # expert 1 empty, rows 33..39 in no group
    got = oracle.mx_grouped_gemm(q_a, sf_a, q_b, sf_b, m_indptr)
    A = _dequant(q_a, sf_a)
    B = _dequant(q_b, sf_b)
    for e in range(E):
        r0, r1 = m_indptr[e], m_indptr[e + 1]
        if r1 == r0:
            continue
        ref = A[r0:r1] @ B[e].T
        np.testing.assert_allclose(got[r0:r1], ref.astype(np.float32), rtol=1e-6,
                                   atol=1e-30 + 1e-7 * np.abs(ref).max())
    assert not got[33:].any()


def test_mx_gemm_exact_small_integers(oracle):
    # integer codes with unit scales (code 127): every partial sum is an
    # integer below 2^24, so the fp32 result is exact
    rng = np.random.default_rng(3)
    R, N, K, E = 8, 16, 64, 2
    table = _e4m3_table()
    ints = {int(v): c for c, v in enumerate(table) if np.isfinite(v) and v == int(v) and abs(v) <= 8}
    vals_a = rng.integers(-8, 9, size=(R, K))
    vals_b = rng.integers(-8, 9, size=(E, N, K))
    q_a = np.vectorize(ints.get)(vals_a).astype(np.uint8)
    q_b = np.vectorize(ints.get)(vals_b).astype(np.uint8)
    sf_a = np.full((R, K // 32), 127, np.uint8)
    sf_b = np.full((E, N, K // 32), 127, np.uint8)
    m_indptr = np.array([0, 3, 8], np.int32)
    got = oracle.mx_grouped_gemm(q_a, sf_a, q_b, sf_b, m_indptr)
    ref = np.concatenate([vals_a[0:3] @ vals_b[0].T, vals_a[3:8] @ vals_b[1].T])
    np.testing.assert_array_equal(got, ref.astype(np.float32))
    # a scale on one 32-block of one row multiplies exactly that block's share
    sf_a2 = sf_a.copy()
    sf_a2[1, 1] = 130
    got2 = oracle.mx_grouped_gemm(q_a, sf_a2, q_b, sf_b, m_indptr)
    part = vals_a[1, 32:] @ vals_b[0][:, 32:].T
    np.testing.assert_array_equal(got2[1], (ref[1] + 7 * part).astype(np.float32))


def test_mx_gemm_bf16_gated_is_swiglu_of_plain(oracle):
    R, N, K, E = 24, 64, 96, 2
    q_a, sf_a, q_b, sf_b = _mx_operands(4, R, N, K, E)
    sf_a[:] = 124
    sf_b[:] = 118  # keep the products in a range where silu is not saturated
    m_indptr = np.array([0, 10, 24], np.int32)
    g = oracle.mx_grouped_gemm(q_a, sf_a, q_b, sf_b, m_indptr)
    gated = oracle.mx_gemm_bf16(q_a, sf_a, q_b, sf_b, m_indptr, True)
    plain = oracle.mx_gemm_bf16(q_a, sf_a, q_b, sf_b, m_indptr, False)
    gt = torch.from_numpy(g.astype(np.float64))
    h = (gt[:, :N // 2] * torch.sigmoid(gt[:, :N // 2]) * gt[:, N // 2:]).to(torch.bfloat16)
    got_h = torch.from_numpy(gated.view(np.int16)).view(torch.bfloat16)
    diff = (got_h.to(torch.float64) - h.to(torch.float64)).abs()
    ulp = h.to(torch.float64).abs() * 2.0 ** -7 + 1e-30
    assert torch.all(diff <= ulp)
    np.testing.assert_array_equal(plain.view(np.int16),
                                  torch.from_numpy(g).to(torch.bfloat16).view(torch.int16).numpy())


# ------------------------------------------------------------ fused MXFP8 layer
def _mx_layer_inputs(seed=0):
    import synth
    cfg = synth.MoEConfig("mx_pin", 12, 256, 128, 4, 2)
    return cfg, synth.make_mx_moe_inputs(cfg, seed=seed)


def _mx_layer(oracle, inp, topk_w=None, perm_tokens=None):
    x = inp["x"]
    ids = inp["topk_ids"]
    w = inp["topk_w"] if topk_w is None else topk_w
    if perm_tokens is not None:
        x, ids, w = x[perm_tokens], ids[perm_tokens], w[perm_tokens]
    bits = oracle.moe_mx_fused(_bf16_bits(x), ids.numpy(), w.numpy(),
                               inp["w13"].view(torch.uint8).numpy(), inp["w13_sf"].numpy(),
                               inp["w2"].view(torch.uint8).numpy(), inp["w2_sf"].numpy())
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


def test_mx_layer_close_to_float64_ffn(oracle):
    # the decoded weights in float64 with unquantised activations: the layer
    # differs from it only by the MXFP8 rounding of x and of the intermediate
    cfg, inp = _mx_layer_inputs(1)
    got = _mx_layer(oracle, inp).to(torch.float64)
    w13 = torch.from_numpy(_dequant(inp["w13"].view(torch.uint8).numpy(), inp["w13_sf"].numpy()))
    w2 = torch.from_numpy(_dequant(inp["w2"].view(torch.uint8).numpy(), inp["w2_sf"].numpy()))
    x = inp["x"].to(torch.float64)
    ref = torch.zeros(cfg.T, cfg.H, dtype=torch.float64)
    for t in range(cfg.T):
        for j in range(cfg.k):
            e = int(inp["topk_ids"][t, j])
            gu = w13[e] @ x[t]
            h = torch.nn.functional.silu(gu[:cfg.I]) * gu[cfg.I:]
            ref[t] += float(inp["topk_w"][t, j]) * (w2[e] @ h)
    rel = ((got - ref).norm() / ref.norm()).item()
    assert rel < 0.06, rel
    # and clearly farther from a layer with a wrong expert choice
    wrong = torch.zeros_like(ref)
    for t in range(cfg.T):
        for j in range(cfg.k):
            e = (int(inp["topk_ids"][t, j]) + 1) % cfg.E
            gu = w13[e] @ x[t]
            wrong[t] += float(inp["topk_w"][t, j]) * (w2[e] @ (torch.nn.functional.silu(gu[:cfg.I]) * gu[cfg.I:]))
    assert ((got - wrong).norm() / ref.norm()).item() > 5 * rel


def test_mx_layer_linear_in_router_weight(oracle):
    # doubling every router weight doubles every fp32 sum exactly, so the
    # bf16 outputs double exactly
    _, inp = _mx_layer_inputs(2)
    base = _mx_layer(oracle, inp).to(torch.float32)
    dbl = _mx_layer(oracle, inp, topk_w=inp["topk_w"] * 2).to(torch.float32)
    assert torch.equal(dbl, 2 * base)


def test_mx_layer_token_order(oracle):
    # each token's result depends only on its own row: permuting the tokens
    # permutes the outputs bit for bit
    cfg, inp = _mx_layer_inputs(3)
    base = _mx_layer(oracle, inp)
    p = torch.randperm(cfg.T, generator=torch.Generator().manual_seed(0))
    got = _mx_layer(oracle, inp, perm_tokens=p)
    assert torch.equal(got.view(torch.int16), base[p].view(torch.int16))


def test_mx_layer_per_token_form_equals_grouped(oracle):
    # the per-token form (used for sampled checks at full size) computes every
    # row with the same arithmetic as the grouped layer: identical bits
    cfg, inp = _mx_layer_inputs(4)
    args = (_bf16_bits(inp["x"]), inp["topk_ids"].numpy(), inp["topk_w"].numpy(),
            inp["w13"].view(torch.uint8).numpy(), inp["w13_sf"].numpy(),
            inp["w2"].view(torch.uint8).numpy(), inp["w2_sf"].numpy())
    full, m_indptr, perm, hq, hsf = oracle.moe_mx_fused(*args, want_dump=True)
    tokens = np.array([0, 5, cfg.T - 1], np.int32)
    out, hq_t, hsf_t = oracle.moe_mx_tokens(*args, tokens, want_h=True)
    np.testing.assert_array_equal(out, full[tokens])
    inv = np.empty(len(perm), np.int64)
    inv[perm] = np.arange(len(perm))
    for i, t in enumerate(tokens):
        for j in range(cfg.k):
            r = inv[t * cfg.k + j]
            np.testing.assert_array_equal(hq_t[i, j], hq[r])
            np.testing.assert_array_equal(hsf_t[i, j], hsf[r])
