"""The bounds-checked build of the library (MOE_CHECKED=1) on the GPU.

Every data-dependent global index of the gather, split, grouped-GEMM epilogues and
combine kernels is tested against its buffer there; an index outside its buffer
raises MOE_DEVERR_OUT_OF_BOUNDS and the access is skipped.  Running the ragged edge
shapes, both tile configurations and the permutation through that build with the
error word clear shows that the schedule the kernels derive (token tiles, weight
tiles, expert-ordered rows, ragged N and K tails) stays inside every buffer; the
results must also match the normal build bit for bit.
"""
import numpy as np
import pytest

from mxfp4_expert_ffn_moe_b200.workloads import make_layer, workload
from tests.gpu_util import layer_to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def checked(moe_gpu):
    from mxfp4_expert_ffn_moe_b200 import build as moe_build
    moe_build.build(checked=True)
    yield moe_gpu
    moe_gpu.use_checked_library(False)


def _forward(moe, layer, dev, ids, w):
    flags = moe.MOE_FLAG_WEIGHT_ON_INPUT if layer.weight_on_input else 0
    return moe.moe_mxfp4_forward_ex(dev["x"], ids, w, dev["gu_blocks"], dev["gu_scales"], dev["gu_bias"],
                                    dev["d_blocks"], dev["d_scales"], dev["d_bias"], alpha=layer.alpha,
                                    limit=layer.limit, flags=flags)


LAYERS = [
    ("edge", (37, 192, 320, 5, 3, False)),     # ragged token tiles, N tails of 64 rows
    ("edge", (130, 128, 64, 3, 2, True)),      # weight on the input, three tiles per expert
    ("edge", (3, 8192, 64, 4, 2, False)),      # decode tiles through the converter kernel
    ("edge", (300, 64, 128, 2, 2, False)),     # prefill tiles, K of one step
    ("named", "20b_decode_T8"),                # block-scaled decode tiles
    ("named", "120b_zipf_T256"),               # skewed: one expert with eight token tiles
    ("named", "20b_prefill_T4096"),            # 256-row tiles
]


@pytest.mark.parametrize("kind,spec", LAYERS, ids=[str(s) for _, s in LAYERS])
def test_checked_build_stays_in_bounds_and_matches(checked, kind, spec):
    import torch
    moe = checked
    if kind == "edge":
        T, H, I, E, k, woi = spec
        layer = make_layer(T, H, I, E, k, seed=T + H, biases=not woi, weight_on_input=woi, bias_std=1.0)
    else:
        layer = workload(spec)
    dev = layer_to_device(layer)
    moe.use_checked_library(False)
    ids, w = moe.moe_route(dev["logits"], layer.k)
    ref = _forward(moe, layer, dev, ids, w)
    torch.cuda.synchronize()
    moe.use_checked_library(True)
    moe.moe_get_device_error()
    out = _forward(moe, layer, dev, ids, w)
    perm = moe.moe_permute(ids, layer.E, 32)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error() == 0
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert int(perm["offsets"][-1].item()) == layer.T * layer.k
    moe.use_checked_library(False)


def test_checked_build_flags_and_skips_a_bad_row_index(checked):
    # moe_combine_pairs with one inverse-map entry one past the pairs: the checked build
    # skips that row and flags it.  y_rows is allocated with spare rows, so the access
    # stays inside the allocation whatever happens.
    import torch
    moe = checked
    T, k, H = 6, 2, 64
    y = torch.randn((T * k + 64, H), dtype=torch.float32, device="cuda")
    pair_rows = torch.arange(T * k, dtype=torch.int32, device="cuda")
    pair_rows[5] = T * k
    moe.use_checked_library(True)
    moe.moe_get_device_error()
    out = moe.moe_combine_pairs(y, pair_rows, T, k)
    err = moe.moe_get_device_error()
    moe.use_checked_library(False)
    assert err & moe.MOE_DEVERR_OUT_OF_BOUNDS
    want = y[:T * k].view(T, k, H).clone()
    want[2, 1] = 0.0                                 # pair 5 = token 2, slot 1 was skipped
    want = want.sum(dim=1).to(torch.bfloat16)
    assert torch.equal(out.view(torch.int16), want.view(torch.int16))
