"""Expert parallelism (fp8_block_scaled_route_b200.ep) across gloo ranks on
CPU: the orchestration (dispatch plan, exchanges with their splits, the
expert step on received rows, the return exchange and the combine) with the
four local steps computed by the oracle on the host.  Checks, on every rank:

  * the index maps: every row a rank receives belongs to an expert it owns,
    carries that expert's local id, and arrives in ascending pair order per
    source rank; every pair of every rank is received exactly once;
  * the output of the whole expert-parallel layer equals, bit for bit, the
    oracle's single-process layer on that rank's tokens with all E experts
    (every step of the layer is row-wise and the combine order is fixed, so
    splitting the experts changes nothing).

No GPU: the CUDA steps are checked by the GPU tests (single process)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

E, H, I, K = 12, 256, 256, 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


class OracleEpOps:
    """The four local steps of the expert-parallel layer on the host, from
    the oracle's functions (test infrastructure only)."""

    def __init__(self, oracle):
        self.O = oracle

    def plan(self, topk_ids, E_, G):
        ids = topk_ids.numpy()
        epr = E_ // G
        owner = np.where((ids >= 0) & (ids < E_), ids // epr, -1).astype(np.int32)
        m, _, inv, _ = self.O.route_permute(owner, G)
        return torch.from_numpy(m.copy()), torch.from_numpy(inv.copy())

    def pack(self, x, topk_ids, slot_of_pair, E_, G, S):
        xq_t, xs_t = self.O.quant_rows_128_bf16(_bits(x))
        ids = topk_ids.numpy().ravel()
        k = topk_ids.shape[1]
        xq = np.zeros((S, x.shape[1]), np.uint8)
        xs = np.zeros((S, x.shape[1] // 128), np.float32)
        eid = np.zeros(S, np.int32)
        for p, s in enumerate(slot_of_pair.numpy()):
            if s >= 0:
                xq[s], xs[s], eid[s] = xq_t[p // k], xs_t[p // k], ids[p] % (E_ // G)
        return torch.from_numpy(xq), torch.from_numpy(xs), torch.from_numpy(eid)

    def expert_rows(self, xq, xs, eid, w13, w13_scale, w2, w2_scale):
        n = xq.shape[0]
        El = w13.shape[0]
        e = eid.numpy()
        order = np.argsort(e, kind="stable")
        m = np.concatenate([[0], np.cumsum(np.bincount(e, minlength=El))]).astype(np.int32)
        a, a_s = xq.numpy()[order], xs.numpy()[order]
        g = self.O.grouped_gemm(a, a_s, w13.numpy(), w13_scale.numpy(), m)
        h = self.O.swiglu(g)
        hq, hs = self.O.quant_rows_128(h)
        y_g = self.O.grouped_gemm(hq, hs, w2.numpy(), w2_scale.numpy(), m)
        y = np.zeros((n, w2.shape[1]), np.float32)
        y[order] = y_g
        return torch.from_numpy(y)

    def combine(self, y, slot_of_pair, topk_w, H_):
        out = self.O.combine(y.numpy() if y.numel() else np.zeros((1, H_), np.float32),
                             slot_of_pair.numpy(), topk_w.numpy())
        return torch.from_numpy(out.view(np.int16)).view(torch.bfloat16)


def _rank_inputs(rank):
    import synth
    T = 17 + 9 * rank
    cfg = synth.MoEConfig("ep", T, H, I, E, K, "zipf" if rank % 2 else "normal")
    return synth.make_moe_inputs(cfg, seed=100 + rank, weights=False)


def _weights():
    import synth
    return synth.make_moe_inputs(synth.MoEConfig("w", 1, H, I, E, K), seed=7)


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import oracle
    from fp8_block_scaled_route_b200 import ep
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        oracle.build()
        inp = _rank_inputs(rank)
        if rank == 0:
            inp["topk_ids"][2, 1] = E       # an id outside [0, E): dropped
        wts = _weights()
        epr = E // world
        sl = slice(rank * epr, (rank + 1) * epr)
        w13 = wts["w13"][sl].view(torch.uint8)
        w2 = wts["w2"][sl].view(torch.uint8)
        moe = ep.ExpertParallelMoE(E, w13, wts["w13_scale"][sl].contiguous(), w2,
                                   wts["w2_scale"][sl].contiguous(), ops=OracleEpOps(oracle))
        # index maps: send (source rank, pair) beside the rows
        d = moe.dispatch(inp["x"], inp["topk_ids"])
        recv_counts = ep._exchange_counts(d.send_counts, None, torch.device("cpu"))
        S = sum(d.send_counts)
        desc = torch.zeros(S, 2, dtype=torch.int32)
        for p, s in enumerate(d.slot_of_pair.tolist()):
            if s >= 0:
                desc[s, 0], desc[s, 1] = rank, p
        got_desc = ep._all_to_all(desc, d.send_counts, recv_counts, None)
        got_eid = ep._all_to_all(d.eid, d.send_counts, recv_counts, None)
        all_ids = [_rank_inputs(r)["topk_ids"] for r in range(world)]
        all_ids[0][2, 1] = E
        for (src, p), e_local in zip(got_desc.tolist(), got_eid.tolist()):
            e = int(all_ids[src].view(-1)[p])
            assert e // epr == rank and e % epr == e_local, (src, p, e, e_local)
        for src in range(world):
            ps = [p for s_, p in got_desc.tolist() if s_ == src]
            assert ps == sorted(ps)
        n_recv = torch.tensor([got_desc.shape[0]], dtype=torch.int64)
        dist.all_reduce(n_recv)
        valid = sum(int(((a >= 0) & (a < E)).sum()) for a in all_ids)
        # the whole layer against the oracle's single-process layer
        out = moe(inp["x"], inp["topk_ids"], inp["topk_w"])
        ref = oracle.moe_fused(_bits(inp["x"]), inp["topk_ids"].numpy(), inp["topk_w"].numpy(),
                               wts["w13"].view(torch.uint8).numpy(), wts["w13_scale"].numpy(),
                               wts["w2"].view(torch.uint8).numpy(), wts["w2_scale"].numpy())
        same = bool(np.array_equal(_bits(out), ref["out"]))
        dist.barrier()
        results[rank] = (same, int(n_recv), valid)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_layer_gloo(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for r in range(world):
        same, n_recv, valid = results[r]
        assert same, f"rank {r}: expert-parallel output differs from the oracle's layer"
        assert n_recv == valid


def test_ep_rejects_uneven_split():
    from fp8_block_scaled_route_b200 import ep

    # E must be a multiple of the group size: checked before any exchange
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        w = torch.zeros(3, 2 * I, H, dtype=torch.uint8)
        with pytest.raises(ValueError):
            ep.ExpertParallelMoE(E, w, w, w, w)   # 3 local experts, E/G = 12
    finally:
        dist.destroy_process_group()
