"""The allocation-free entry point against the allocating one, on the GPU.

moe_mxfp4_forward_noalloc serves callers that cannot allocate device memory (a
plugin given only its buffers, a serving loop that must not allocate after
start-up); it places the layer's scratch in the library's static device array.
This file is collected last so that a run stopping at the first failure has run
every other test before it.
"""
import ctypes

import numpy as np
import pytest

from mxfp4_expert_ffn_moe_b200.workloads import workload
from tests._metrics import MAX_ABS_OVER_RMS_TOL, REL_L2_TOL, max_abs_over_rms, rel_l2
from tests.gpu_util import bf16_tensor_to_f64, layer_to_device

pytestmark = pytest.mark.gpu


def _inputs(moe, name):
    layer = workload(name)
    dev = layer_to_device(layer)
    ids, w = moe.moe_route(dev["logits"], layer.k)
    args = (dev["x"], ids, w, dev["gu_blocks"], dev["gu_scales"], dev["gu_bias"],
            dev["d_blocks"], dev["d_scales"], dev["d_bias"])
    return layer, args


def test_noalloc_matches_allocating_entry_on_two_calls_in_a_row(moe_gpu):
    import torch
    moe = moe_gpu
    cases = [_inputs(moe, "20b_decode_T64"), _inputs(moe, "tiny_bias_heavy")]
    refs = [moe.moe_mxfp4_forward(*args, alpha=L.alpha, limit=L.limit) for L, args in cases]
    # two calls in a row: the second finds the first call's data in the scratch
    outs = [moe.moe_mxfp4_forward_noalloc(*args, alpha=L.alpha, limit=L.limit) for L, args in cases]
    torch.cuda.synchronize()
    for (L, _), ref, out in zip(cases, refs, outs):
        want, got = bf16_tensor_to_f64(ref), bf16_tensor_to_f64(out)
        assert rel_l2(got, want) <= REL_L2_TOL, L.name
        assert max_abs_over_rms(got, want) <= MAX_ABS_OVER_RMS_TOL, L.name
    assert moe.moe_get_device_error() == 0


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
