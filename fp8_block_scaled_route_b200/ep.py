"""Expert parallelism: the fused FP8 MoE layer with its experts split over
G GPUs, one process per GPU, torch.distributed (NCCL over NVLink on GPUs)
for the exchanges.

Rank g owns experts [g*E/G, (g+1)*E/G) (their FP8 weights and scales only)
and keeps its own tokens.  One layer call, on every rank:

  1. plan     moe_ep_plan: each (token, slot) pair gets a send slot, the
              slots grouped by the rank that owns the pair's expert;
  2. pack     moe_ep_pack: x quantised per token per 128 columns, each
              pair's FP8 row, its scales and its expert's local id written
              into its send slot;
  3. exchange counts, then rows, scales and ids (all-to-all);
  4. experts  moe_fp8_expert_rows: the expert FFN (GEMM1 + SwiGLU + FP8
              requant, GEMM2) on the rows this rank received;
  5. exchange the fp32 rows back (all-to-all, the reverse splits);
  6. combine  moe_combine: each token's k rows weighted and summed in
              ascending slot order, bf16 out.

The layer is the one of the page "FlashInfer: Blackwell W8A8 AlphaMoE Expert
계산 커널 퓨전으로 성능 비약적 향상" (section "문제점: MoE Expert 계산의 병목");
the pages do not describe expert parallelism, so the split is the plainest
one the layer allows (a pair's rows only meet its own expert's weights).
As the AG-matmul page binds a process group and its buffers once ("2. API
개선": prepare_all_gather_matmul), ExpertParallelMoE holds the group, the
local weights and grown-on-demand buffers across calls.

Every per-row computation is the same kernel as in moe_fp8_fused and the
combine order is the same, so the output equals the single-GPU layer's up to
the GEMMs' accumulation order (the token tile a row lands in).

The exchanges use torch.distributed.all_to_all_single, so the same code runs
on NCCL (GPU tensors) and on gloo (CPU tensors, with `ops` computing the
steps on the host: the multi-process tests do that).  Unmeasured on
multi-GPU hardware.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import (moe_combine, moe_ep_pack, moe_ep_plan, moe_ep_workspace_size,
               moe_fp8_expert_rows, moe_fp8_expert_rows_workspace_size, moe_get_device_status,
               MOE_ERR_BAD_EXPERT_ID, MOE_OK, MoEError)


class CudaEpOps:
    """The four steps on the GPU, through the C ABI.  Buffers are torch
    tensors on the rank's device; workspaces grow on demand and are reused."""

    def __init__(self, device):
        self.device = torch.device(device)
        self._ws = {}
        self.last_plan_status = MOE_OK

    def _workspace(self, name: str, nbytes: int):
        ws = self._ws.get(name)
        if ws is None or ws.numel() < nbytes:
            ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
            self._ws[name] = ws
        return ws

    def plan(self, topk_ids, E: int, G: int):
        T, k = topk_ids.shape
        R = T * k
        send_indptr = torch.empty(G + 1, dtype=torch.int32, device=self.device)
        send_pair = torch.empty(max(R, 1), dtype=torch.int32, device=self.device)
        slot_of_pair = torch.empty(max(R, 1), dtype=torch.int32, device=self.device)
        ws = self._workspace("plan", moe_ep_workspace_size(T, k, G))
        moe_ep_plan(topk_ids, E, G, send_indptr, send_pair, slot_of_pair, ws)
        # ids outside [0, E) are dropped (as moe_fp8_fused drops them) and reported here
        self.last_plan_status = moe_get_device_status(ws)
        if self.last_plan_status not in (MOE_OK, MOE_ERR_BAD_EXPERT_ID):
            raise MoEError(self.last_plan_status, "moe_ep_plan (device)")
        return send_indptr.cpu(), slot_of_pair[:R]

    def pack(self, x, topk_ids, slot_of_pair, E: int, G: int, S: int):
        H = x.shape[1]
        xq = torch.empty(max(S, 1), H, dtype=torch.uint8, device=self.device)
        xs = torch.empty(max(S, 1), H // 128, dtype=torch.float32, device=self.device)
        eid = torch.empty(max(S, 1), dtype=torch.int32, device=self.device)
        moe_ep_pack(x, topk_ids, slot_of_pair, E, G, S, xq, xs, eid)
        return xq[:S], xs[:S], eid[:S]

    def expert_rows(self, xq, xs, eid, w13, w13_scale, w2, w2_scale):
        n, H = xq.shape
        E, I2, _ = w13.shape
        I = I2 // 2
        y = torch.empty(max(n, 1), H, dtype=torch.float32, device=self.device)
        if n == 0:
            return y[:0]
        ws = self._workspace("experts", moe_fp8_expert_rows_workspace_size(n, H, I, E))
        moe_fp8_expert_rows(xq, xs, eid, w13, w13_scale, w2, w2_scale, y, ws, dims=(n, H, I, E))
        st = moe_get_device_status(ws)
        if st != MOE_OK:
            raise MoEError(st, "moe_fp8_expert_rows (device)")
        return y[:n]

    def combine(self, y, slot_of_pair, topk_w, H: int):
        T, k = topk_w.shape
        out = torch.empty(T, H, dtype=torch.bfloat16, device=self.device)
        if T:
            src = y if y.numel() else torch.empty(1, H, dtype=torch.float32, device=self.device)
            moe_combine(src, slot_of_pair, topk_w, out, dims=(T, k, H))
        return out


@dataclass
class Dispatch:
    """What one rank sends: counts per destination rank and the send-ordered
    rows, plus the map the combine needs."""
    send_counts: list
    slot_of_pair: torch.Tensor
    xq: torch.Tensor
    xs: torch.Tensor
    eid: torch.Tensor


class ExpertParallelMoE:
    """The layer over `group` (default: the world), this rank's experts
    w13 [E/G, 2I, H], w13_scale [E/G, 2I/128, H/128], w2 [E/G, H, I],
    w2_scale [E/G, H/128, I/128] (FP8 codes / fp32, as moe_fp8_fused takes
    them), E = the total expert count.  `ops` computes the four local steps
    (default CudaEpOps on the weights' device).  `world` = (G, rank) sets
    the split without a process group, for a driver that runs the ranks'
    steps itself (dispatch / experts / finish) and moves the rows between
    them; calling the object then is not possible."""

    def __init__(self, E: int, w13, w13_scale, w2, w2_scale, group=None, ops=None, world=None):
        self.group = group
        if world is not None:
            self.G, self.rank = int(world[0]), int(world[1])
        else:
            self.G = dist.get_world_size(group)
            self.rank = dist.get_rank(group)
        self._grouped = world is None
        if E % self.G:
            raise ValueError(f"E={E} is not a multiple of the group size {self.G}")
        if w13.shape[0] != E // self.G:
            raise ValueError(f"{w13.shape[0]} local experts, expected E/G = {E // self.G}")
        self.E = E
        self.w13, self.w13_scale, self.w2, self.w2_scale = w13, w13_scale, w2, w2_scale
        self.H = w2.shape[1]
        self.ops = ops if ops is not None else CudaEpOps(w13.device)

    # -- the steps, usable on their own (a driver may run ranks stage by stage)
    def dispatch(self, x, topk_ids) -> Dispatch:
        send_indptr, slot_of_pair = self.ops.plan(topk_ids, self.E, self.G)
        ind = [int(v) for v in send_indptr.tolist()]
        S = ind[self.G]
        xq, xs, eid = self.ops.pack(x, topk_ids, slot_of_pair, self.E, self.G, S)
        counts = [ind[g + 1] - ind[g] for g in range(self.G)]
        return Dispatch(counts, slot_of_pair, xq, xs, eid)

    def experts(self, xq, xs, eid):
        return self.ops.expert_rows(xq, xs, eid, self.w13, self.w13_scale, self.w2, self.w2_scale)

    def finish(self, y_back, d: Dispatch, topk_w):
        return self.ops.combine(y_back, d.slot_of_pair, topk_w, self.H)

    # -- one layer call with the exchanges over the group
    def __call__(self, x, topk_ids, topk_w):
        if not self._grouped:
            raise RuntimeError("built with an explicit world: run dispatch / experts / finish")
        d = self.dispatch(x, topk_ids)
        recv_counts = _exchange_counts(d.send_counts, self.group, x.device)
        xq = _all_to_all(d.xq, d.send_counts, recv_counts, self.group)
        xs = _all_to_all(d.xs, d.send_counts, recv_counts, self.group)
        eid = _all_to_all(d.eid, d.send_counts, recv_counts, self.group)
        y = self.experts(xq, xs, eid)
        y_back = _all_to_all(y, recv_counts, d.send_counts, self.group)
        return self.finish(y_back, d, topk_w)


def _exchange_counts(send_counts, group, device):
    G = len(send_counts)
    dev = device if device.type == "cuda" else torch.device("cpu")
    send = torch.tensor(send_counts, dtype=torch.int64, device=dev)
    recv = torch.empty(G, dtype=torch.int64, device=dev)
    dist.all_to_all_single(recv, send, group=group)
    return [int(v) for v in recv.tolist()]


def _all_to_all(t, send_counts, recv_counts, group):
    """Rows [sum(send_counts), ...] out, rows [sum(recv_counts), ...] back."""
    out = torch.empty((sum(recv_counts),) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    dist.all_to_all_single(out, t.contiguous(), output_split_sizes=list(recv_counts),
                           input_split_sizes=list(send_counts), group=group)
    return out
