"""Expert parallelism on CPU: gloo ranks run mxfp4_expert_ffn_moe_b200.expert_parallel
(partition of the experts, dispatch counts, the row exchange, the return and the
slot-ordered combine) with the device steps stood in by CPU code: numpy bookkeeping
for the permutation, the gather and the combine, and the CPU oracle for each rank's
own experts.  Every rank's output must equal the single-process oracle over the whole
layer bit for bit (double precision), because each exchanged row is exactly one
oracle slot w * (y + b) and the combine adds them in the oracle's order.  No GPU.
"""
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """Device steps on the CPU: the permutation, gather and combine restated in numpy,
    the experts by the oracle (test infrastructure)."""
    row_dtype = None

    def __init__(self, oracle):
        import torch
        self.oracle = oracle
        OracleOps.row_dtype = torch.float64

    def permute(self, ids, num_experts):
        import torch
        flat = ids.reshape(-1).numpy().astype(np.int64)
        valid = (flat >= 0) & (flat < num_experts)
        p = np.nonzero(valid)[0]
        order = p[np.argsort(flat[p], kind="stable")]
        counts = np.bincount(flat[valid], minlength=num_experts)
        offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
        pair_rows = np.full(flat.size, -1, np.int64)
        pair_rows[order] = np.arange(order.size)
        perm = {"sorted_pairs": torch.from_numpy(order), "pair_rows": torch.from_numpy(pair_rows)}
        return perm, offsets.tolist()

    def gather(self, x, ids, weights, perm, num_experts):
        import torch
        sp = perm["sorted_pairs"].numpy()
        k = ids.shape[1]
        x_rows = torch.from_numpy(x.numpy()[sp // k].copy())
        return (x_rows, torch.from_numpy(ids.reshape(-1).numpy()[sp].astype(np.int32)),
                torch.from_numpy(weights.reshape(-1).numpy()[sp].astype(np.float32)))

    def expert_rows(self, x_rows, row_ids, row_weights, expert_base, banks, alpha, limit, flags):
        import torch
        ids = (row_ids.numpy().astype(np.int64) - expert_base).astype(np.int32)[:, None]
        out = self.oracle.forward_tokens(x_rows.numpy().view(np.uint16), ids, row_weights.numpy()[:, None],
                                         banks["gate_up_blocks"], banks["gate_up_scales"], banks.get("gate_up_bias"),
                                         banks["down_blocks"], banks["down_scales"], banks.get("down_bias"),
                                         alpha=alpha, limit=limit, weight_on_input=bool(flags & 1))
        return torch.from_numpy(out)

    def combine(self, y_rows, perm, T, k):
        import torch
        y = y_rows.numpy()
        pr = perm["pair_rows"].numpy().reshape(T, k)
        out = np.zeros((T, y.shape[1]), np.float64)
        for j in range(k):                       # slot order, as the oracle sums
            m = pr[:, j] >= 0
            out[m] = out[m] + y[pr[m, j]]
        return torch.from_numpy(out)


def _layer(seed, woi):
    from mxfp4_expert_ffn_moe_b200.workloads import make_layer
    return make_layer(7, 64, 64, 5, 2, seed=seed, biases=not woi, weight_on_input=woi, bias_std=0.5)


def _rank(rank, world, port, woi, q):
    import datetime

    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    sys.path.insert(0, ROOT)
    import oracle
    from mxfp4_expert_ffn_moe_b200.expert_parallel import ExpertParallelMoE, expert_ranges
    bank_layer = _layer(100, woi)                 # the layer's weights, known to every rank
    E = bank_layer.E
    lo, hi = expert_ranges(E, world)[rank]
    banks = {"gate_up_blocks": bank_layer.gate_up.blocks[lo:hi], "gate_up_scales": bank_layer.gate_up.scales[lo:hi],
             "down_blocks": bank_layer.down.blocks[lo:hi], "down_scales": bank_layer.down.scales[lo:hi]}
    if not woi:
        banks["gate_up_bias"] = bank_layer.gate_up_bias[lo:hi]
        banks["down_bias"] = bank_layer.down_bias[lo:hi]
    tok = _layer(200 + rank, woi)                 # this rank's own tokens and routing
    ids, w = oracle.route(tok.logits, tok.k)
    if rank == 1:
        ids[3, 1] = E + 2                         # an out-of-range id: the slot is dropped
    layer = ExpertParallelMoE(E, banks, ops=OracleOps(oracle))
    out = layer.forward(torch.from_numpy(tok.x_bits.view(np.int16)), torch.from_numpy(ids), torch.from_numpy(w),
                        flags=1 if woi else 0).numpy()
    ids_ref, w_ref = ids.copy(), w.copy()
    if rank == 1:
        ids_ref[3, 1], w_ref[3, 1] = 0, 0.0       # a zero-weight slot adds exactly zero
    want = oracle.forward_tokens(tok.x_bits, ids_ref, w_ref, bank_layer.gate_up.blocks, bank_layer.gate_up.scales,
                                 None if woi else bank_layer.gate_up_bias, bank_layer.down.blocks,
                                 bank_layer.down.scales, None if woi else bank_layer.down_bias,
                                 weight_on_input=woi)
    plan = layer.last_plan
    recv_ids = plan["recv_ids"].numpy()
    # bookkeeping: rows sent per owner = the pairs routed to its experts; rows received
    # all belong to this rank's experts
    flat = ids.reshape(-1)
    owners = [np.sum((flat >= a) & (flat < b)) for a, b in expert_ranges(E, world)]
    q.put((rank, bool(np.array_equal(out, want)), float(np.max(np.abs(out - want))),
           list(plan["send_rows"]) == [int(v) for v in owners],
           bool(np.all((recv_ids >= lo) & (recv_ids < hi))), int(sum(plan["recv_rows"]))))
    dist.barrier()
    dist.destroy_process_group()


def _run_world(world, woi):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, woi, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(200)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, equal, maxdiff, sends_ok, recv_ok, nrecv in res:
        assert equal, (rank, maxdiff)
        assert sends_ok and recv_ok, rank
    # every valid pair of every rank was computed exactly once (7 tokens x 2 slots per
    # rank, one dropped on rank 1)
    assert sum(r[5] for r in res) == world * 7 * 2 - 1


@pytest.mark.timeout(240)
@pytest.mark.parametrize("woi", [False, True], ids=["weight_on_output", "weight_on_input"])
def test_two_rank_expert_parallel_equals_single_rank_oracle(woi):
    _run_world(2, woi)


@pytest.mark.timeout(240)
def test_three_rank_expert_parallel_with_uneven_ranges():
    # 5 experts over 3 ranks: ranges of 1, 2 and 2 experts
    _run_world(3, False)


def test_expert_ranges_and_rows_per_rank():
    sys.path.insert(0, ROOT)
    from mxfp4_expert_ffn_moe_b200.expert_parallel import expert_ranges, rows_per_rank
    assert expert_ranges(32, 4) == [(0, 8), (8, 16), (16, 24), (24, 32)]
    assert expert_ranges(5, 2) == [(0, 2), (2, 5)]
    r = expert_ranges(128, 3)
    assert r[0][0] == 0 and r[-1][1] == 128 and all(b - a in (42, 43) for a, b in r)
    assert all(r[i][1] == r[i + 1][0] for i in range(2))
    assert rows_per_rank([0, 3, 3, 7, 9, 12], [(0, 2), (2, 5)]) == [3, 9]
    with pytest.raises(ValueError):
        expert_ranges(2, 3)
