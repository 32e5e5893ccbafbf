"""The expert-parallel device steps on one GPU.

moe_permute + moe_gather_pairs + moe_mxfp4_expert_rows + moe_combine_pairs must give
moe_mxfp4_forward_ex's output bit for bit when one rank owns every expert, both
directly and through ExpertParallelMoE over a one-rank NCCL group.  Splitting the
experts over several ranks is emulated on the one GPU by running each rank's slice
of the rows against its slice of the banks (expert_base = its first expert), with the
exchange reduced to placing the rows: the result must meet the layer tolerance
against the oracle.  The multi-rank exchange itself is tested with gloo ranks on the
CPU (tests/test_expert_parallel_gloo.py).
"""
import socket

import numpy as np
import pytest

from mxfp4_expert_ffn_moe_b200.workloads import workload
from tests._metrics import MAX_ABS_OVER_RMS_TOL, REL_L2_TOL, max_abs_over_rms, rel_l2
from tests.gpu_util import bf16_tensor_to_f64, layer_to_device, oracle_forward, stratified_tokens

pytestmark = pytest.mark.gpu


def _banks(dev, lo=None, hi=None):
    sl = slice(lo, hi)
    b = {"gate_up_blocks": dev["gu_blocks"][sl], "gate_up_scales": dev["gu_scales"][sl],
         "down_blocks": dev["d_blocks"][sl], "down_scales": dev["d_scales"][sl]}
    if dev["gu_bias"] is not None:
        b["gate_up_bias"] = dev["gu_bias"][sl]
        b["down_bias"] = dev["d_bias"][sl]
    return b


def _split_run(moe, layer, dev, ids, w, world):
    """The expert-parallel steps with `world` expert ranges, all on this GPU."""
    import torch
    from mxfp4_expert_ffn_moe_b200.expert_parallel import expert_ranges
    flags = moe.MOE_FLAG_WEIGHT_ON_INPUT if layer.weight_on_input else 0
    perm = moe.moe_permute(ids, layer.E, tile_rows=1)
    offsets = perm["offsets"].cpu().tolist()
    x_rows, row_ids, row_w = moe.moe_gather_pairs(dev["x"], ids, w, perm, layer.E)
    y = torch.empty((layer.T * layer.k, layer.H), dtype=torch.float32, device="cuda")
    for lo, hi in expert_ranges(layer.E, world):
        a, b = offsets[lo], offsets[hi]
        if b > a:
            bk = _banks(dev, lo, hi)
            moe.moe_mxfp4_expert_rows(x_rows[a:b], row_ids[a:b], row_w[a:b], lo, bk["gate_up_blocks"],
                                      bk["gate_up_scales"], bk.get("gate_up_bias"), bk["down_blocks"],
                                      bk["down_scales"], bk.get("down_bias"), alpha=layer.alpha, limit=layer.limit,
                                      flags=flags, y_rows=y[a:b])
    out = moe.moe_combine_pairs(y, perm["pair_rows"], layer.T, layer.k)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("name", ["tiny_woo", "tiny_woi", "20b_decode_T64", "20b_prefill_T4096"])
def test_one_rank_steps_equal_the_forward(moe_gpu, name):
    import torch
    layer = workload(name)
    dev = layer_to_device(layer)
    ids, w = moe_gpu.moe_route(dev["logits"], layer.k)
    flags = moe_gpu.MOE_FLAG_WEIGHT_ON_INPUT if layer.weight_on_input else 0
    ref = moe_gpu.moe_mxfp4_forward_ex(dev["x"], ids, w, dev["gu_blocks"], dev["gu_scales"], dev["gu_bias"],
                                       dev["d_blocks"], dev["d_scales"], dev["d_bias"], alpha=layer.alpha,
                                       limit=layer.limit, flags=flags)
    out = _split_run(moe_gpu, layer, dev, ids, w, 1)
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert moe_gpu.moe_get_device_error() == 0


@pytest.mark.parametrize("name,world", [("tiny_woo", 3), ("tiny_woi", 2), ("20b_decode_T64", 4),
                                        ("120b_zipf_T256", 8)])
def test_expert_slices_meet_the_layer_tolerance(moe_gpu, oracle_mod, name, world):
    layer = workload(name)
    dev = layer_to_device(layer)
    ids_np, w_np = oracle_mod.route(layer.logits, layer.k)
    import torch
    ids = torch.from_numpy(ids_np).cuda()
    w = torch.from_numpy(w_np).cuda()
    got = bf16_tensor_to_f64(_split_run(moe_gpu, layer, dev, ids, w, world))
    tokens = np.arange(layer.T) if layer.T <= 64 else stratified_tokens(ids_np, layer.E, 32)
    want = oracle_forward(oracle_mod, layer, ids_np, w_np, tokens)
    r, m = rel_l2(got[tokens], want), max_abs_over_rms(got[tokens], want)
    assert r <= REL_L2_TOL and m <= MAX_ABS_OVER_RMS_TOL, (r, m)
    assert moe_gpu.moe_get_device_error() == 0


def test_expert_parallel_layer_on_a_one_rank_nccl_group(moe_gpu):
    import datetime

    import torch
    import torch.distributed as dist
    from mxfp4_expert_ffn_moe_b200.expert_parallel import ExpertParallelMoE
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        layer = workload("20b_decode_T8")
        dev = layer_to_device(layer)
        ids, w = moe_gpu.moe_route(dev["logits"], layer.k)
        ep = ExpertParallelMoE(layer.E, _banks(dev))
        out = ep.forward(dev["x"], ids, w, alpha=layer.alpha, limit=layer.limit)
        ref = moe_gpu.moe_mxfp4_forward_ex(dev["x"], ids, w, dev["gu_blocks"], dev["gu_scales"], dev["gu_bias"],
                                           dev["d_blocks"], dev["d_scales"], dev["d_bias"], alpha=layer.alpha,
                                           limit=layer.limit)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
        assert ep.last_plan["send_rows"] == [layer.T * layer.k]
    finally:
        dist.destroy_process_group()
    assert moe_gpu.moe_get_device_error() == 0
