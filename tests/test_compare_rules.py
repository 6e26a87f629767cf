"""The layer comparison rule of the GPU parity tests, exercised on the CPU
with the oracle standing in for the GPU: an allowed adjacent code in the
intermediate is accepted when the output follows from it, and an output
error in any row is caught."""
import numpy as np
import pytest

import oracle as O
import synth
from tests import gpu_helpers as G


@pytest.fixture(scope="module")
def case(oracle):
    cfg = synth.MoEConfig("rule", 24, 256, 256, 6, 2)
    inp = synth.make_moe_inputs(cfg, seed=11, device="cpu")
    ref = O.moe_fused(*G.oracle_args(inp))
    return inp, ref


def _fake_gpu(inp, ref, hq):
    """A 'GPU' result: the oracle's routing, the given intermediate, and the
    output the oracle's down GEMM + combine give for it."""
    ids = G.i32(inp["topk_ids"])
    T, k = ids.shape
    inv = np.full(T * k, -1, np.int32)
    inv[ref["perm"]] = np.arange(len(ref["perm"]))
    y = O.grouped_gemm(hq, ref["hs"], G.u8(inp["w2"]), G.f32(inp["w2_scale"]), ref["m_indptr"])
    out = O.combine(y, inv, G.f32(inp["topk_w"]))
    return dict(out=out, hq=hq, hs=ref["hs"], m_indptr=ref["m_indptr"], perm=ref["perm"])


def _largest_code(ref):
    """Grouped row and column of an intermediate code at its block's maximum."""
    mags = np.abs(O.e4m3_decode(ref["hq"]))
    return np.unravel_index(int(np.argmax(mags)), mags.shape)


def test_identical_result_passes(case):
    inp, ref = case
    G.compare_layer(_fake_gpu(inp, ref, ref["hq"].copy()), ref, inp, "identical")


def test_adjacent_code_with_consistent_output_passes(case):
    inp, ref = case
    hq = ref["hq"].copy()
    r, c = _largest_code(ref)
    hq[r, c] = hq[r, c] - 1 if hq[r, c] & 0x7F else hq[r, c] + 1   # one step toward zero
    G.compare_layer(_fake_gpu(inp, ref, hq), ref, inp, "one adjacent code")


def test_output_error_in_unaffected_row_fails(case):
    inp, ref = case
    res = _fake_gpu(inp, ref, ref["hq"].copy())
    f = G.bits_to_f64(res["out"])
    rms = float(np.sqrt(np.mean(G.bits_to_f64(ref["out"]) ** 2)))
    bad = f.copy()
    bad[3, 7] += 0.05 * rms
    res["out"] = O.f32_to_bf16_bits(bad.astype(np.float32))
    with pytest.raises(AssertionError):
        G.compare_layer(res, ref, inp, "planted error")


def test_output_error_in_row_with_code_difference_fails(case):
    inp, ref = case
    hq = ref["hq"].copy()
    r, c = _largest_code(ref)
    hq[r, c] = hq[r, c] - 1 if hq[r, c] & 0x7F else hq[r, c] + 1
    res = _fake_gpu(inp, ref, hq)
    t = int(ref["perm"][r]) // G.i32(inp["topk_ids"]).shape[1]
    f = G.bits_to_f64(res["out"])
    rms = float(np.sqrt(np.mean(G.bits_to_f64(ref["out"]) ** 2)))
    f[t, 0] += 0.05 * rms
    res["out"] = O.f32_to_bf16_bits(f.astype(np.float32))
    with pytest.raises(AssertionError):
        G.compare_layer(res, ref, inp, "planted error beside a code difference")
