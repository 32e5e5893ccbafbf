"""Expert parallelism for the MXFP4 expert layer.

The experts are split into contiguous ranges over the ranks of a process group;
rank r owns experts ranges[r] = [lo_r, hi_r) and holds only their banks.  Every rank
routes its own tokens, then (transformers PR #49431, "Restore GPT-OSS's router-masked
expert-parallel plan": each rank's MXFP4 experts consume the routing data restricted
to the experts it owns):

  1. permute    its (token, slot) pairs grouped by expert.  Experts are numbered in
                rank order, so expert order is also destination order: rows
                offsets[lo_r] .. offsets[hi_r] go to rank r.
  2. gather     those rows as a self-contained batch: x row, expert id, routing weight.
  3. exchange   counts, then the rows, with one all_to_all_single each.
  4. experts    the received rows through the rank's own experts (ids relative to
                lo_rank), one fp32 row per (token, slot): w * (y + b), or y with the
                router weight on the input.
  5. return     each row goes back to the rank it came from, in the order it came.
  6. combine    each token's k rows summed in slot order, rounded once to bf16.

With one rank the result is moe_mxfp4_forward_ex's output bit for bit.  The device
steps run in the library's kernels (moe_permute, moe_gather_pairs,
moe_mxfp4_expert_rows, moe_combine_pairs); the exchanges are torch.distributed
collectives (NCCL between GPUs).  The rows cross the interconnect in the exchange
and land in this GPU's own memory before any kernel reads them.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple


def expert_ranges(num_experts: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous expert ranges, one per rank, sizes differing by at most one."""
    if world < 1 or num_experts < world:
        raise ValueError(f"cannot split {num_experts} experts over {world} ranks")
    return [(r * num_experts // world, (r + 1) * num_experts // world) for r in range(world)]


def rows_per_rank(offsets: Sequence[int], ranges: Sequence[Tuple[int, int]]) -> List[int]:
    """Rows of an expert-ordered batch that go to each rank (offsets: the exclusive
    scan of the per-expert row counts, E + 1 entries)."""
    return [int(offsets[hi]) - int(offsets[lo]) for lo, hi in ranges]


class CudaLayerOps:
    """The device steps on the library's kernels (tensors on the current CUDA device)."""

    def __init__(self):
        import mxfp4_expert_ffn_moe_b200 as moe
        self.moe = moe

    def permute(self, ids, num_experts: int):
        perm = self.moe.moe_permute(ids, num_experts, tile_rows=1, want_pair_rows=True)
        return perm, perm["offsets"].cpu().tolist()

    def gather(self, x, ids, weights, perm, num_experts: int):
        return self.moe.moe_gather_pairs(x, ids, weights, perm, num_experts)

    def expert_rows(self, x_rows, row_ids, row_weights, expert_base: int, banks, alpha, limit, flags):
        return self.moe.moe_mxfp4_expert_rows(
            x_rows, row_ids, row_weights, expert_base, banks["gate_up_blocks"], banks["gate_up_scales"],
            banks.get("gate_up_bias"), banks["down_blocks"], banks["down_scales"], banks.get("down_bias"),
            alpha=alpha, limit=limit, flags=flags)

    def combine(self, y_rows, perm, T: int, k: int):
        return self.moe.moe_combine_pairs(y_rows, perm["pair_rows"], T, k)


class ExpertParallelMoE:
    """One rank's share of an expert-parallel MoE layer.

    num_experts  experts of the whole layer (E)
    banks        this rank's experts only, experts expert_ranges(E, world)[rank]:
                 gate_up_blocks [E_r, 2I, H/2], gate_up_scales [E_r, 2I, H/32],
                 gate_up_bias [E_r, 2I] or None, down_blocks [E_r, H, I/2],
                 down_scales [E_r, H, I/32], down_bias [E_r, H] or None
    group        torch.distributed process group (None: the default group)
    ops          the device steps (CudaLayerOps by default)
    """

    def __init__(self, num_experts: int, banks: dict, group=None, ops=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.E = int(num_experts)
        self.ranges = expert_ranges(self.E, self.world)
        lo, hi = self.ranges[self.rank]
        n_local = banks["gate_up_blocks"].shape[0]
        if n_local != hi - lo:
            raise ValueError(f"rank {self.rank} owns experts [{lo}, {hi}) but was given {n_local} banks")
        self.banks = banks
        self.ops = ops if ops is not None else CudaLayerOps()
        self.last_plan: Optional[dict] = None

    def _exchange(self, send, send_rows: List[int], recv_rows: List[int]):
        import torch
        out = torch.empty((sum(recv_rows),) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
        self.dist.all_to_all_single(out, send.contiguous(), recv_rows, send_rows, group=self.group)
        return out

    def forward(self, x, ids, weights, alpha: float = 1.702, limit: float = 7.0, flags: int = 0):
        """This rank's tokens x [T, H] with routing ids / weights [T, k] (global expert
        ids) -> the layer output for those tokens, [T, H]."""
        import torch
        T, k = ids.shape
        perm, offsets = self.ops.permute(ids, self.E)
        send_rows = rows_per_rank(offsets, self.ranges)
        rows = int(offsets[self.E])
        counts = torch.tensor(send_rows, dtype=torch.int64, device=x.device)
        got = torch.empty_like(counts)
        self.dist.all_to_all_single(got, counts, group=self.group)
        recv_rows = [int(v) for v in got.cpu().tolist()]
        x_rows, row_ids, row_w = self.ops.gather(x, ids, weights, perm, self.E)
        # bf16 rows travel as their bit patterns, two per 32-bit word (H is even)
        rx = self._exchange(x_rows[:rows].view(torch.int32), send_rows, recv_rows).view(x_rows.dtype)
        rids = self._exchange(row_ids[:rows], send_rows, recv_rows)
        rw = self._exchange(row_w[:rows], send_rows, recv_rows)
        lo, _ = self.ranges[self.rank]
        if rx.shape[0] > 0:
            y_local = self.ops.expert_rows(rx, rids, rw, lo, self.banks, alpha, limit, flags)
        else:
            y_local = self._empty_rows(x)
        y_back = self._exchange(y_local, recv_rows, send_rows)
        self.last_plan = {"send_rows": send_rows, "recv_rows": recv_rows, "recv_ids": rids}
        return self.ops.combine(y_back, perm, T, k)

    def _empty_rows(self, x):
        import torch
        dtype = getattr(self.ops, "row_dtype", torch.float32)
        return torch.empty((0, x.shape[1]), dtype=dtype, device=x.device)
