"""Pins of the oracle's NVFP4 variant (E2M1 values, an E4M3 scale per 16
elements, an fp32 global scale; the cuTile page's NVFP4 W4A4 quantisation)
against facts that do not come from the oracle: the E2M1 bit-field
definition, round-to-nearest-even on brute-force midpoints, the rounding
bound, a float64 matmul of the decoded operands and exact small products.
CPU only."""
import numpy as np
import torch


def _e2m1_from_bits(c):
    """Value of an E2M1 code from its fields: sign, 2-bit exponent (bias 1),
    1-bit mantissa; exponent 0 is subnormal (m * 0.5)."""
    s = -1.0 if c & 8 else 1.0
    e, m = (c >> 1) & 3, c & 1
    return s * (m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1.0 + m / 2.0))


def test_e2m1_decode_matches_bit_fields(oracle):
    got = oracle.e2m1_decode(np.arange(16))
    np.testing.assert_array_equal(got, np.array([_e2m1_from_bits(c) for c in range(16)], np.float32))


def test_e2m1_encode_bruteforce(oracle):
    vals = np.array([_e2m1_from_bits(c) for c in range(8)])
    xs = np.linspace(-7.5, 7.5, 3001)
    got = oracle.e2m1_encode(xs)
    for x, c in zip(xs, got):
        a = min(abs(x), 6.0)
        d = np.abs(vals - a)
        best = np.flatnonzero(d == d.min())
        want = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]  # ties: even code
        assert (c & 7) == want, (x, c)
        if x < 0 and want != 0:
            assert c & 8
    # every code survives a round trip
    np.testing.assert_array_equal(oracle.e2m1_encode(oracle.e2m1_decode(np.arange(16))),
                                  np.array([c if c != 8 else 8 for c in range(16)], np.uint8))


def _dequant(oracle, q, sf, g):
    e4 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    vals = oracle.e2m1_decode(np.arange(16)).astype(np.float64)[q.astype(np.int64)]
    return vals * np.repeat(e4[sf.astype(np.int64)], 16, axis=-1) / g


def test_nvfp4_quant_rounding_bound(oracle):
    g_ = torch.Generator().manual_seed(0)
    x = (torch.randn(8, 256, generator=g_) * 3).numpy()
    g = 448.0 * 6.0 / float(np.abs(x).max())
    q, sf = oracle.quant_rows_nvfp4(x, g)
    deq = _dequant(oracle, q, sf, g)
    e4 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    s = np.repeat(e4[sf.astype(np.int64)], 16, axis=1)
    scaled = np.abs(x) * g / s
    # half the gap of the E2M1 grid around the scaled value (0.25 below 2, 0.5 below 4, 1 above),
    # plus the saturation at 6 (the block scale's E4M3 rounding can put the maximum above 6)
    half_gap = np.where(scaled < 2, 0.25, np.where(scaled < 4, 0.5, 1.0))
    bound = (half_gap + np.maximum(scaled - 6.0, 0.0)) * s / g
    assert np.all(np.abs(deq - x) <= bound * (1 + 1e-9) + 1e-12)


def test_nvfp4_gemm_matches_float64_matmul(oracle):
    rng = np.random.default_rng(1)
    R, N, K, E = 24, 32, 64, 2
    q_a = rng.integers(0, 16, (R, K)).astype(np.uint8)
    q_b = rng.integers(0, 16, (E, N, K)).astype(np.uint8)
    sf_a = rng.integers(0x30, 0x48, (R, K // 16)).astype(np.uint8)    # E4M3 codes 0.5 .. 4
    sf_b = rng.integers(0x30, 0x48, (E, N, K // 16)).astype(np.uint8)
    ga, gb = 3.0, np.array([2.0, 0.75], np.float32)
    m_indptr = np.array([0, 9, 24], np.int32)
    got = oracle.nvfp4_grouped_gemm(q_a, sf_a, ga, q_b, sf_b, gb, m_indptr)
    A = _dequant(oracle, q_a, sf_a, ga)
    for e in range(E):
        r0, r1 = m_indptr[e], m_indptr[e + 1]
        ref = A[r0:r1] @ _dequant(oracle, q_b[e], sf_b[e], float(gb[e])).T
        np.testing.assert_allclose(got[r0:r1], ref.astype(np.float32), rtol=1e-6,
                                   atol=1e-7 * np.abs(ref).max())


def test_nvfp4_gemm_exact_small_values(oracle):
    # unit block scales (E4M3 1.0 = 0x38), unit global scales: sums of
    # products of E2M1 values are exact multiples of 0.25
    rng = np.random.default_rng(2)
    R, N, K, E = 8, 8, 32, 1
    q_a = rng.integers(0, 16, (R, K)).astype(np.uint8)
    q_b = rng.integers(0, 16, (E, N, K)).astype(np.uint8)
    dec = np.array([_e2m1_from_bits(c) for c in range(16)])
    got = oracle.nvfp4_grouped_gemm(q_a, np.full((R, 2), 0x38, np.uint8), 1.0, q_b,
                                    np.full((E, N, 2), 0x38, np.uint8), np.ones(1, np.float32),
                                    np.array([0, R], np.int32))
    np.testing.assert_array_equal(got, (dec[q_a] @ dec[q_b[0]].T).astype(np.float32))


def _e4m3_code_of(v):
    table = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    hits = np.flatnonzero(table == v)
    assert len(hits), v
    return int(hits[0])


def test_nvfp4_bf16_reduces_to_mxfp8_bf16(oracle):
    """Every E2M1 value is an E4M3 value and a power-of-two E4M3 block scale is
    an E8M0 scale: with unit global scales and the same scale on both 16-wide
    halves of every 32-wide block, the NVFP4 GEMM is an MXFP8 GEMM, so the
    bf16 outputs (plain and gated) are bit-identical to the pinned MXFP8 ones."""
    rng = np.random.default_rng(3)
    R, N, K, E = 40, 64, 128, 3
    m_indptr = np.array([0, 11, 11, 40], np.int32)
    q_a = rng.integers(0, 16, (R, K)).astype(np.uint8)
    q_b = rng.integers(0, 16, (E, N, K)).astype(np.uint8)
    exp_a = rng.integers(-3, 4, (R, K // 32))
    exp_b = rng.integers(-3, 4, (E, N, K // 32))
    to_e4 = np.vectorize(lambda e: _e4m3_code_of(2.0 ** e))
    sf_a = np.repeat(to_e4(exp_a), 2, axis=-1).astype(np.uint8)
    sf_b = np.repeat(to_e4(exp_b), 2, axis=-1).astype(np.uint8)
    e2m1_to_e4m3 = np.array([_e4m3_code_of(v) if v != 0 else (0x80 if c & 8 else 0)
                             for c, v in enumerate(_e2m1_from_bits(c) for c in range(16))], np.uint8)
    mx_a, mx_b = e2m1_to_e4m3[q_a], e2m1_to_e4m3[q_b]
    for gated in (False, True):
        got = oracle.nvfp4_gemm_bf16(q_a, sf_a, 1.0, q_b, sf_b, np.ones(E, np.float32), m_indptr, gated)
        want = oracle.mx_gemm_bf16(mx_a, (exp_a + 127).astype(np.uint8), mx_b,
                                   (exp_b + 127).astype(np.uint8), m_indptr, gated)
        np.testing.assert_array_equal(got[:40], want[:40])


def test_nvfp4_bf16_global_scales(oracle):
    """Global scales divide the output: halving ga doubles every output (exact
    in bf16, a power of two)."""
    rng = np.random.default_rng(4)
    R, N, K, E = 16, 32, 64, 2
    q_a = rng.integers(0, 16, (R, K)).astype(np.uint8)
    q_b = rng.integers(0, 16, (E, N, K)).astype(np.uint8)
    sf_a = rng.integers(0x30, 0x48, (R, K // 16)).astype(np.uint8)
    sf_b = rng.integers(0x30, 0x48, (E, N, K // 16)).astype(np.uint8)
    gb = np.array([3.0, 0.5], np.float32)
    m = np.array([0, 7, 16], np.int32)
    one = oracle.nvfp4_gemm_bf16(q_a, sf_a, 4.0, q_b, sf_b, gb, m, False).view(np.int16)
    two = oracle.nvfp4_gemm_bf16(q_a, sf_a, 2.0, q_b, sf_b, gb, m, False).view(np.int16)
    f = lambda b: torch.from_numpy(b.copy()).view(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(f(two), 2.0 * f(one))
