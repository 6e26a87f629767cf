"""Pins of the oracle's NVFP4 layer (x and the intermediate quantised to
NVFP4 with calibrated global scales, NVFP4 weights; the AlphaMoE page's
five-stage pipeline in the cuTile page's NVFP4 format) against facts that do
not come from the layer code: a float64 MoE layer on the dequantised weights
(the only differences are the two activation roundings, bounded by the E2M1
grid), the per-token form, and exact scaling by the top-k weights.  CPU only."""
import numpy as np
import torch

import synth


def _np(inp, name):
    v = inp[name]
    return v.numpy() if torch.is_tensor(v) else v


def _bits(x):
    return x.view(torch.int16).numpy().view(np.uint16)


def _run(oracle, inp, want_dump=False, topk_w=None):
    return oracle.moe_nvfp4_fused(_bits(inp["x"]), _np(inp, "topk_ids"),
                                  _np(inp, "topk_w") if topk_w is None else topk_w,
                                  _np(inp, "w13"), _np(inp, "w13_sf"), _np(inp, "w13_g"),
                                  _np(inp, "w2"), _np(inp, "w2_sf"), _np(inp, "w2_g"),
                                  inp["a1_g"], inp["a2_g"], want_dump=want_dump)


def _to_f64(bits):
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()


def _dequant_weights(inp, name):
    e2m1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6])
    e4m3 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    q, sf, g = _np(inp, name), _np(inp, name + "_sf"), _np(inp, name + "_g")
    return e2m1[q] * np.repeat(e4m3[sf], 16, axis=-1) / g.astype(np.float64)[:, None, None]


CASES = [synth.CONFIGS["tiny"], synth.MoEConfig("nv_case", 33, 256, 256, 5, 3, "normal"),
         synth.MoEConfig("nv_skew", 40, 512, 128, 8, 2, "zipf")]


def test_nvfp4_layer_close_to_float64_layer(oracle):
    """Against the float64 layer on the same (dequantised) weights and the
    unquantised x: relative RMS error below 0.22.  NVFP4 rounding of Gaussian
    data has a relative RMS error eps ~ 0.095 (checked below); x's error
    enters gate and up, the intermediate's once more, so the layer's error is
    ~ sqrt(3) eps = 0.165.  A dropped term, a wrong global scale (a factor of
    2) or a wrong expert is far outside the bound."""
    for cfg in CASES:
        inp = synth.make_nvfp4_moe_inputs(cfg, seed=cfg.T)
        got = _to_f64(_run(oracle, inp))
        w13, w2 = _dequant_weights(inp, "w13"), _dequant_weights(inp, "w2")
        x = inp["x"].double().numpy()
        ids, w = _np(inp, "topk_ids"), _np(inp, "topk_w").astype(np.float64)
        I = cfg.I
        ref = np.zeros_like(x)
        for t in range(cfg.T):
            for j in range(cfg.k):
                e = ids[t, j]
                g = w13[e] @ x[t]
                h = g[:I] / (1 + np.exp(-g[:I])) * g[I:]
                ref[t] += w[t, j] * (w2[e] @ h)
        rel = np.sqrt(((got - ref) ** 2).sum() / (ref ** 2).sum())
        assert rel < 0.22, (cfg.name, rel)


def test_nvfp4_rounding_error_of_gaussian_data(oracle):
    """The eps the bound above rests on: 0.08 < eps < 0.11 for N(0,1) rows."""
    x = torch.randn(64, 1024, generator=torch.Generator().manual_seed(3)).numpy()
    g = synth.NVFP4_A1_GSCALE
    q, sf = oracle.quant_rows_nvfp4(x, g)
    e2m1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6])
    e4m3 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    d = e2m1[q] * np.repeat(e4m3[sf], 16, axis=-1) / g
    eps = np.sqrt(((d - x) ** 2).sum() / (x ** 2).sum())
    assert 0.08 < eps < 0.11, eps


def test_nvfp4_layer_tokens_match_fused(oracle):
    """The per-token form (no grouping, one dot product at a time) gives the
    same bits as the grouped layer, intermediate included."""
    for cfg in CASES:
        inp = synth.make_nvfp4_moe_inputs(cfg, seed=cfg.T + 1)
        out, m, perm, hq, hsf = _run(oracle, inp, want_dump=True)
        toks = np.arange(cfg.T, dtype=np.int32)
        o2, hq2, hsf2 = oracle.moe_nvfp4_tokens(
            _bits(inp["x"]), _np(inp, "topk_ids"), _np(inp, "topk_w"), _np(inp, "w13"),
            _np(inp, "w13_sf"), _np(inp, "w13_g"), _np(inp, "w2"), _np(inp, "w2_sf"),
            _np(inp, "w2_g"), inp["a1_g"], inp["a2_g"], toks, want_h=True)
        np.testing.assert_array_equal(out, o2)
        # grouped row r holds pair perm[r] = t * k + j
        np.testing.assert_array_equal(hq, hq2.reshape(-1, cfg.I)[perm])
        np.testing.assert_array_equal(hsf, hsf2.reshape(-1, cfg.I // 16)[perm])


def test_nvfp4_layer_topk_weight_scaling(oracle):
    """The combine is linear in the top-k weights: doubling them doubles every
    output exactly (a power of two in fp32 and bf16)."""
    inp = synth.make_nvfp4_moe_inputs(CASES[1], seed=5)
    one = _to_f64(_run(oracle, inp))
    two = _to_f64(_run(oracle, inp, topk_w=2.0 * _np(inp, "topk_w")))
    np.testing.assert_array_equal(two, 2.0 * one)
