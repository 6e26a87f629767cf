"""Pins of the oracle's standalone combine (the AlphaMoE page's stage 5,
"문제점: MoE Expert 계산의 병목": the router-weighted sum of each token's expert
outputs, then bf16) against facts that do not come from the oracle itself:
torch's bf16 rounding, exact dyadic arithmetic, dropped pairs, and the fused
layer's own last stage.  CPU only."""
import numpy as np
import torch

import synth


def _bf16_bits(x64: np.ndarray) -> np.ndarray:
    """torch's round-to-nearest-even bf16 cast of exactly representable fp32 values."""
    return torch.from_numpy(np.asarray(x64, np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def test_single_slot_unit_weight_is_bf16_cast(oracle):
    rng = np.random.default_rng(0)
    T, H = 37, 384
    y = rng.standard_normal((T + 5, H)).astype(np.float32) * 3.0
    inv = rng.permutation(T + 5)[:T].astype(np.int32)
    got = oracle.combine(y, inv, np.ones((T, 1), np.float32))
    assert np.array_equal(got, _bf16_bits(y[inv]))


def test_dyadic_values_sum_exactly(oracle):
    """Small integers times 2^-4 and weights that are sums of a few powers of
    two: every product and partial sum is exact in fp32, so the result is the
    exact weighted sum (int64 / float64) rounded to bf16 once."""
    rng = np.random.default_rng(1)
    T, k, H = 50, 8, 256
    R = T * k
    y_int = rng.integers(-2000, 2001, size=(R, H))
    y = (y_int * 2.0 ** -4).astype(np.float32)
    w_int = rng.integers(0, 64, size=(T, k))        # weights = w_int / 64
    w = (w_int / 64.0).astype(np.float32)
    inv = rng.permutation(R).astype(np.int32)
    got = oracle.combine(y, inv, w)
    exact = np.einsum("tj,tjh->th", w_int.astype(np.float64),
                      y_int[inv.reshape(T, k)].astype(np.float64)) * (2.0 ** -4 / 64.0)
    assert np.array_equal(got, _bf16_bits(exact))


def test_dropped_pairs_contribute_nothing(oracle):
    rng = np.random.default_rng(2)
    T, k, H = 20, 4, 256
    y = rng.standard_normal((T * k, H)).astype(np.float32)
    w = rng.random((T, k)).astype(np.float32)
    inv = rng.permutation(T * k).astype(np.int32)
    drop = rng.random(T * k) < 0.3
    inv_d = np.where(drop, -1, inv).astype(np.int32)
    w_z = np.where(drop.reshape(T, k), 0.0, w).astype(np.float32)
    assert np.array_equal(oracle.combine(y, inv_d, w), oracle.combine(y, inv, w_z))


def test_equals_fused_layers_last_stage(oracle):
    """GEMM2 on the fused layer's dumped intermediate, then the standalone
    combine, reproduces the fused layer's output bit for bit."""
    cfg = synth.MoEConfig("c", 24, 256, 256, 6, 3)
    inp = synth.make_moe_inputs(cfg, seed=3)
    x = inp["x"].view(torch.int16).numpy().view(np.uint16)
    ids = inp["topk_ids"].numpy()
    w = inp["topk_w"].numpy()
    w13 = inp["w13"].view(torch.uint8).numpy()
    w2 = inp["w2"].view(torch.uint8).numpy()
    ref = oracle.moe_fused(x, ids, w, w13, inp["w13_scale"].numpy(), w2, inp["w2_scale"].numpy())
    y = oracle.grouped_gemm(ref["hq"], ref["hs"], w2, inp["w2_scale"].numpy(), ref["m_indptr"])
    _, _, inv, _ = oracle.route_permute(ids, cfg.E)
    assert np.array_equal(oracle.combine(y, inv, w), ref["out"])
