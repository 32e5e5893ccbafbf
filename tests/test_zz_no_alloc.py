"""The allocation-free entry point against the allocating one, on the GPU.

moe_mxfp4_forward_noalloc serves callers that cannot allocate device memory (a
plugin given only its buffers, a serving loop that must not allocate after
start-up); it places the layer's scratch in the library's static device array.
Both calls run the same deterministic kernels on the same inputs, so their outputs
must agree bit for bit; one case is also compared with the oracle at the layer
tolerance.  This file is collected last so that a run stopping at the first
failure has run every other test before it.
"""
import ctypes

import numpy as np
import pytest

from mxfp4_expert_ffn_moe_b200.workloads import make_layer, workload
from tests._metrics import MAX_ABS_OVER_RMS_TOL, REL_L2_TOL, max_abs_over_rms, rel_l2
from tests.gpu_util import bf16_tensor_to_f64, layer_to_device

pytestmark = pytest.mark.gpu


def _inputs(moe, layer):
    dev = layer_to_device(layer)
    ids, w = moe.moe_route(dev["logits"], layer.k)
    args = (dev["x"], ids, w, dev["gu_blocks"], dev["gu_scales"], dev["gu_bias"],
            dev["d_blocks"], dev["d_scales"], dev["d_bias"])
    flags = moe.MOE_FLAG_WEIGHT_ON_INPUT if layer.weight_on_input else 0
    return layer, args, flags


def test_noalloc_matches_allocating_entry_on_two_calls_in_a_row(moe_gpu, oracle_mod):
    import torch
    moe = moe_gpu
    # decode tiles (block-scaled kernel), weight on the output with heavy biases,
    # weight on the input, and the prefill-tile path at the gpt-oss-20b shape (1,280
    # pairs > 32 E) whose workspace still fits the static array
    prefill = make_layer(320, 2880, 2880, 32, 4, seed=5, name="20b_T320")
    assert moe.moe_token_tile_rows(320, 2880, 2880, 32, 4) > 32
    assert moe.moe_mxfp4_workspace_size(320, 2880, 2880, 32, 4) <= moe.MOE_NOALLOC_SCRATCH_BYTES
    cases = [_inputs(moe, L) for L in (workload("20b_decode_T64"), workload("tiny_bias_heavy"),
                                        workload("tiny_woi"), prefill)]
    refs = [moe.moe_mxfp4_forward_ex(*args, alpha=L.alpha, limit=L.limit, flags=f) for L, args, f in cases]
    # two rounds in a row: each call finds the previous call's data in the scratch
    for _ in range(2):
        outs = [moe.moe_mxfp4_forward_noalloc(*args, alpha=L.alpha, limit=L.limit, flags=f)
                for L, args, f in cases]
        torch.cuda.synchronize()
        for (L, _, _), ref, out in zip(cases, refs, outs):
            assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), L.name
    assert moe.moe_get_device_error() == 0
    # and the result itself against the oracle
    L = cases[1][0]
    ids, w = oracle_mod.route(L.logits, L.k)
    want = oracle_mod.forward_tokens(L.x_bits, ids, w, L.gate_up.blocks, L.gate_up.scales, L.gate_up_bias,
                                     L.down.blocks, L.down.scales, L.down_bias, alpha=L.alpha, limit=L.limit)
    got = bf16_tensor_to_f64(outs[1])
    assert rel_l2(got, want) <= REL_L2_TOL and max_abs_over_rms(got, want) <= MAX_ABS_OVER_RMS_TOL


def test_noalloc_refuses_sizes_beyond_its_scratch(moe_gpu):
    moe = moe_gpu
    lib = moe.load_library()
    T, H, I, E, k = 4096, 2880, 2880, 32, 4
    assert moe.moe_mxfp4_workspace_size(T, H, I, E, k) > moe.MOE_NOALLOC_SCRATCH_BYTES
    p = ctypes.c_void_p(0x100000)   # refused before any pointer is used
    rc = lib.moe_mxfp4_forward_noalloc(p, T, H, I, E, k, p, p, p, p, None, p, p, None,
                                       ctypes.c_float(1.702), ctypes.c_float(7.0), p,
                                       ctypes.c_uint32(0), None)
    assert rc == -4
    assert moe.moe_status_string(rc).startswith("out of memory")
