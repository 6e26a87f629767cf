"""The expert-parallel steps (moe_ep_plan, moe_ep_pack, moe_fp8_expert_rows,
moe_combine) on one GPU, through the C ABI, for G = 2 and 4 expert ranks
whose exchanges a single process performs by moving rows between the
ranks' buffers (no collective: nothing waits on another rank).  Checks:

  * the plan's index maps bit-exact against the oracle's routing of the
    owner ranks (stable, ascending pair id);
  * the packed rows: FP8 codes and scales bit-exact against the oracle's
    per-token quantisation, local expert ids exact;
  * every rank's output against the oracle's whole layer on that rank's
    tokens with all E experts (the layer's tolerances), and against
    moe_fp8_fused on the same GPU (the same kernels row by row: at most a
    few bf16 ulps apart).
B200 only."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_route_b200 as moe
from fp8_block_scaled_route_b200 import ep
import oracle as O
import synth
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from fp8_block_scaled_route_b200 import build
    build.build()
    O.build()
    torch.cuda.set_device(0)
    yield


def _loopback_layer(ranks, inputs):
    """Runs the ranks' steps and moves the rows between them as the two
    all-to-all exchanges would."""
    W = len(ranks)
    ds = [r.dispatch(inp["x"], inp["topk_ids"]) for r, inp in zip(ranks, inputs)]
    starts = [np.concatenate([[0], np.cumsum(d.send_counts)]) for d in ds]

    def seg(t, s, d):  # rows rank s sends to rank d
        return t[int(starts[s][d]):int(starts[s][d + 1])]

    ys = []
    for d in range(W):
        xq = torch.cat([seg(ds[s].xq, s, d) for s in range(W)])
        xs = torch.cat([seg(ds[s].xs, s, d) for s in range(W)])
        eid = torch.cat([seg(ds[s].eid, s, d) for s in range(W)])
        ys.append(ranks[d].experts(xq, xs, eid))
    recv_starts = [np.concatenate([[0], np.cumsum([ds[s].send_counts[d] for s in range(W)])])
                   for d in range(W)]
    outs = []
    for s in range(W):
        y_back = torch.cat([ys[d][int(recv_starts[d][s]):int(recv_starts[d][s + 1])]
                            for d in range(W)])
        outs.append(ranks[s].finish(y_back, ds[s], inputs[s]["topk_w"]))
    return ds, outs


@pytest.mark.parametrize("world,E,H,I,k,T0", [
    (2, 8, 512, 256, 4, 40),       # small groups: swapped GEMM tiles reading rows in place
    (4, 16, 256, 384, 6, 40),
    (2, 4, 512, 1024, 2, 330),     # ~330 rows per local expert: 128-token GEMM1 tiles on grouped copies
])
def test_expert_parallel_loopback(world, E, H, I, k, T0):
    wts = synth.make_moe_inputs(synth.MoEConfig("w", 1, H, I, E, k), seed=11, device="cuda")
    inputs = []
    for r in range(world):
        cfg = synth.MoEConfig("ep", T0 + 37 * r, H, I, E, k, "zipf" if r % 2 else "normal")
        inputs.append(synth.make_moe_inputs(cfg, seed=200 + r, device="cuda", weights=False))
    inputs[0]["topk_ids"][3, 0] = -1          # dropped pair
    epr = E // world
    ranks = []
    for r in range(world):
        sl = slice(r * epr, (r + 1) * epr)
        ranks.append(ep.ExpertParallelMoE(E, wts["w13"][sl], wts["w13_scale"][sl].contiguous(),
                                          wts["w2"][sl], wts["w2_scale"][sl].contiguous(),
                                          world=(world, r)))
    ds, outs = _loopback_layer(ranks, inputs)
    w13, w13s = G.u8(wts["w13"]), G.f32(wts["w13_scale"])
    w2, w2s = G.u8(wts["w2"]), G.f32(wts["w2_scale"])
    for r in range(world):
        inp = inputs[r]
        ids = G.i32(inp["topk_ids"])
        T = ids.shape[0]
        # plan: bit-exact against the oracle's stable grouping by owner rank
        owner = np.where((ids >= 0) & (ids < E), ids // epr, -1).astype(np.int32)
        m_o, _, inv_o, bad = O.route_permute(owner, world)
        assert np.array_equal(np.concatenate([[0], np.cumsum(ds[r].send_counts)]), m_o)
        assert np.array_equal(G.i32(ds[r].slot_of_pair), inv_o)
        assert ranks[r].ops.last_plan_status == (moe.MOE_ERR_BAD_EXPERT_ID if bad else moe.MOE_OK)
        # pack: the oracle's per-token quantisation, placed at each pair's slot
        xq_t, xs_t = O.quant_rows_128_bf16(G.bf16_bits(inp["x"]))
        xq, xs, eid = G.u8(ds[r].xq), G.f32(ds[r].xs), G.i32(ds[r].eid)
        for p, s in enumerate(inv_o):
            if s >= 0:
                assert np.array_equal(xq[s], xq_t[p // k]), (r, p)
                assert np.array_equal(xs[s], xs_t[p // k]), (r, p)
                assert eid[s] == ids.ravel()[p] % epr
        # the layer: oracle (tolerances), single-GPU fused layer (same kernels)
        ref = O.moe_fused(G.bf16_bits(inp["x"]), ids, G.f32(inp["topk_w"]), w13, w13s, w2, w2s)
        G.compare_out(G.bf16_bits(outs[r]), ref["out"], f"ep rank {r}/{world} vs oracle")
        fused = G.run_fused(dict(inp, w13=wts["w13"], w13_scale=wts["w13_scale"], w2=wts["w2"],
                                 w2_scale=wts["w2_scale"]), debug=False)
        g = G.bits_to_f64(G.bf16_bits(outs[r]))
        f = G.bits_to_f64(fused["out"])
        assert np.all(np.abs(g - f) <= 2 ** -6 * np.abs(f) + 1e-6), f"ep rank {r} vs fused layer"


def test_expert_parallel_nccl_single_rank():
    """The layer called through its NCCL exchanges (a process group of one
    rank: every exchange is the rank's own rows) equals moe_fp8_fused."""
    import os
    import socket
    import torch.distributed as dist
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        E, H, I, k = 8, 512, 256, 4
        wts = synth.make_moe_inputs(synth.MoEConfig("w", 1, H, I, E, k), seed=21, device="cuda")
        inp = synth.make_moe_inputs(synth.MoEConfig("ep1", 150, H, I, E, k), seed=22,
                                    device="cuda", weights=False)
        layer = ep.ExpertParallelMoE(E, wts["w13"], wts["w13_scale"], wts["w2"], wts["w2_scale"])
        out = layer(inp["x"], inp["topk_ids"], inp["topk_w"])
        torch.cuda.synchronize()
        fused = G.run_fused(dict(inp, w13=wts["w13"], w13_scale=wts["w13_scale"], w2=wts["w2"],
                                 w2_scale=wts["w2_scale"]), debug=False)
        assert fused["status"] == moe.MOE_OK
        g = G.bits_to_f64(G.bf16_bits(out))
        f = G.bits_to_f64(fused["out"])
        assert np.all(np.abs(g - f) <= 2 ** -6 * np.abs(f) + 1e-6)
    finally:
        dist.destroy_process_group()
