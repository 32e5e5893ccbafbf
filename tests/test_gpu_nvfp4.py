"""The NVFP4 expert variant on the GPU against the CPU oracle.

nvfp4_dequantize is compared bit for bit (one rounding of the exact product);
moe_nvfp4_forward_ex with the layer tolerance of the MXFP4 layer (relative L2 error
<= 1e-2, max |error| <= 2e-2 * RMS of the oracle output; the edge shapes with the
rounding envelope of the MXFP4 edge tests).  Full-size workloads are compared on
sampled tokens.
"""
import os

import numpy as np
import pytest

from mxfp4_expert_ffn_moe_b200.workloads import make_layer, make_nvfp4_dequant_bank, workload
from tests._metrics import (MAX_ABS_OVER_RMS_TOL, REL_L2_TOL, envelope_excess_over_rms,
                            max_abs_over_rms, rel_l2)
from tests.gpu_util import (bf16_tensor_to_f64, bits_of, nvfp4_layer_to_device, oracle_nvfp4_forward,
                            run_nvfp4_forward, sample_tokens, stratified_tokens, to_dev)

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _gpu_dequant(moe, blocks, scales, scale2):
    import torch
    out = moe.nvfp4_dequantize(to_dev(blocks), to_dev(scales), to_dev(scale2))
    torch.cuda.synchronize()
    return bits_of(out)


# --------------------------------------------------------------------------- dequant

def test_dequant_worked_examples(moe_gpu, oracle_mod):
    rows = []
    with open(os.path.join(GOLDEN, "nvfp4_dequant_worked_examples.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    E = len(rows)
    blocks = np.zeros((E, 1, 8), np.uint8)
    scales = np.zeros((E, 1, 1), np.uint8)
    s2 = np.zeros(E, np.float32)
    for e, (b, s, f, _, _) in enumerate(rows):
        blocks[e, 0, :] = int(b, 16)
        scales[e, 0, 0] = int(s, 16)
        s2[e] = np.uint32(int(f, 16)).view(np.float32)
    got = _gpu_dequant(moe_gpu, blocks, scales, s2)
    for e, row in enumerate(rows):
        assert np.all(got[e, 0, 0::2] == int(row[3], 16)), (row, hex(got[e, 0, 0]))
        assert np.all(got[e, 0, 1::2] == int(row[4], 16)), (row, hex(got[e, 0, 1]))
    # one row holds the NaN scale byte 0x7f
    assert moe_gpu.moe_get_device_error() & moe_gpu.MOE_DEVERR_BAD_SCALE


def test_dequant_every_scale_byte(moe_gpu, oracle_mod):
    # row n uses E4M3 byte n in every block: zeros, subnormals, 448, both NaNs, negatives
    E, N, K = 2, 256, 64
    rng = np.random.default_rng(5)
    blocks = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    scales = np.repeat(np.arange(256, dtype=np.uint8)[None, :, None], K // 16, axis=2)
    scales = np.repeat(scales, E, axis=0)
    s2 = np.float32([1.0, 0.7310585])
    got = _gpu_dequant(moe_gpu, blocks, scales, s2)
    np.testing.assert_array_equal(got, oracle_mod.nvfp4_dequantize(blocks, scales, s2, E, N, K))
    assert moe_gpu.moe_get_device_error() & moe_gpu.MOE_DEVERR_BAD_SCALE


@pytest.mark.parametrize("E,N,K,with_s2", [(1, 1, 16, True), (3, 5, 96, True), (2, 7, 2880, False),
                                           (4, 129, 160, True), (70, 3, 48, True)])
def test_dequant_ragged_shapes(moe_gpu, oracle_mod, E, N, K, with_s2):
    rng = np.random.default_rng(E * 100 + N)
    blocks = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    scales = rng.integers(0, 0x7F, size=(E, N, K // 16), dtype=np.uint8)
    scales |= (rng.integers(0, 2, size=scales.shape, dtype=np.uint8) << 7)      # both signs, no NaN
    s2 = (rng.uniform(-2.0, 2.0, size=E) * 2.0 ** rng.integers(-20, 20, size=E)).astype(np.float32) \
        if with_s2 else None
    got = _gpu_dequant(moe_gpu, blocks, scales, s2)
    np.testing.assert_array_equal(got, oracle_mod.nvfp4_dequantize(blocks, scales, s2, E, N, K))
    assert moe_gpu.moe_get_device_error() == 0


def test_dequant_tiny_and_huge_products_round_once(moe_gpu, oracle_mod):
    # weight_scale_2 values that push the products into the bf16 subnormals, below
    # 2^-118 (the double-precision branch) and past the largest finite bf16
    E, N, K = 6, 16, 64
    rng = np.random.default_rng(9)
    blocks = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    scales = rng.integers(0, 0x7F, size=(E, N, K // 16), dtype=np.uint8)
    s2 = np.float32([2.0 ** -120 * 1.3, 2.0 ** -130 * 1.7, 2.0 ** -140, 3.0e38, 2.0 ** 120 * 1.9,
                     np.float32(1.0) + np.float32(2.0 ** -23)])
    got = _gpu_dequant(moe_gpu, blocks, scales, s2)
    np.testing.assert_array_equal(got, oracle_mod.nvfp4_dequantize(blocks, scales, s2, E, N, K))
    assert moe_gpu.moe_get_device_error() == 0


def test_dequant_full_20b_bank_bit_exact(moe_gpu, oracle_mod):
    # the NVFP4 twin of the gpt-oss-20b bank, every element of both projections
    import torch
    gu, dn = make_nvfp4_dequant_bank(seed=0)
    for bank in (gu, dn):
        E, N, K = bank.shape
        out = moe_gpu.nvfp4_dequantize(to_dev(bank.blocks), to_dev(bank.scales), to_dev(bank.scale2))
        torch.cuda.synchronize()
        got = bits_of(out)
        del out
        want = oracle_mod.nvfp4_dequantize(bank.blocks, bank.scales, bank.scale2, E, N, K)
        assert np.array_equal(got, want), f"{int(np.count_nonzero(got != want))} elements differ"
        del got, want
    assert moe_gpu.moe_get_device_error() == 0


# --------------------------------------------------------------------------- layer

def _assert_close(got, want, what=""):
    r, m = rel_l2(got, want), max_abs_over_rms(got, want)
    assert r <= REL_L2_TOL and m <= MAX_ABS_OVER_RMS_TOL, f"{what}: rel_l2={r:.3g} max/rms={m:.3g}"


def _assert_close_envelope(got, want, env, what=""):
    """The edge-shape bound (tests/_metrics.py): bf16 output rounding plus one bf16
    rounding of each activation operand, scaled by the magnitude envelope."""
    r, m = rel_l2(got, want), envelope_excess_over_rms(got, want, env)
    assert r <= REL_L2_TOL and m <= MAX_ABS_OVER_RMS_TOL, f"{what}: rel_l2={r:.3g} excess/rms={m:.3g}"


def _check_layer(moe, oracle, layer, n_sample=None, seed=0, envelope=False, stratified=False):
    dev = nvfp4_layer_to_device(layer)
    ids, w = oracle.route(layer.logits, layer.k)
    out = run_nvfp4_forward(moe, dev, ids, w, layer)
    got = bf16_tensor_to_f64(out)
    if stratified:
        tile = moe.moe_token_tile_rows(layer.T, layer.H, layer.I, layer.E, layer.k, nvfp4=True)
        tokens = stratified_tokens(ids, layer.E, tile, extra=8, seed=seed)
    else:
        tokens = sample_tokens(layer.T, n_sample or layer.T, seed)
    if envelope:
        want, env = oracle_nvfp4_forward(oracle, layer, ids, w, tokens, envelope=True)
        _assert_close_envelope(got[tokens], want, env, layer.name)
    else:
        _assert_close(got[tokens], oracle_nvfp4_forward(oracle, layer, ids, w, tokens), layer.name)
    assert moe.moe_get_device_error() == 0
    return out


@pytest.mark.parametrize("name", ["nvfp4_tiny_woo", "nvfp4_tiny_woi", "nvfp4_tiny_bias_heavy"])
def test_tiny_layers_full_compare(moe_gpu, oracle_mod, name):
    _check_layer(moe_gpu, oracle_mod, workload(name))


@pytest.mark.parametrize("T,H,I,E,k,woi", [
    (1, 64, 64, 1, 1, False),        # dense MLP, single token
    (37, 192, 320, 5, 3, False),     # ragged token tiles, several weight tiles
    (130, 128, 64, 3, 2, True),      # weight on input, more than two token tiles per expert
    (3, 256, 128, 16, 4, False),     # most experts empty
    (300, 64, 128, 2, 2, False),     # prefill tiles (pairs > 32 E), two experts
])
def test_edge_shapes(moe_gpu, oracle_mod, T, H, I, E, k, woi):
    layer = make_layer(T, H, I, E, k, seed=T + H + 1, biases=not woi, weight_on_input=woi,
                       bias_std=1.0, name=f"nvfp4_edge_{T}_{H}_{I}_{E}_{k}", fmt="nvfp4")
    _check_layer(moe_gpu, oracle_mod, layer, envelope=True)


def test_full_size_decode_every_token(moe_gpu, oracle_mod):
    _check_layer(moe_gpu, oracle_mod, workload("nvfp4_20b_decode_T8"))


def test_full_size_prefill_every_tile(moe_gpu, oracle_mod):
    # every touched expert, the first and last row of each of its token tiles
    _check_layer(moe_gpu, oracle_mod, workload("nvfp4_20b_prefill_T4096"), stratified=True)


def test_missing_scale2_means_one(moe_gpu, oracle_mod):
    import torch
    layer = workload("nvfp4_tiny_bias_heavy")
    dev = nvfp4_layer_to_device(layer)
    ids, w = oracle_mod.route(layer.logits, layer.k)
    dev_none = dict(dev, gu_scale2=None, d_scale2=None)
    dev_ones = dict(dev, gu_scale2=to_dev(np.ones((layer.E, 2), np.float32)),
                    d_scale2=to_dev(np.ones(layer.E, np.float32)))
    a = run_nvfp4_forward(moe_gpu, dev_none, ids, w, layer)
    b = run_nvfp4_forward(moe_gpu, dev_ones, ids, w, layer)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    want = oracle_mod.nvfp4_forward_tokens(layer.x_bits, ids, w, layer.gate_up.blocks, layer.gate_up.scales,
                                           None, layer.gate_up_bias, layer.down.blocks, layer.down.scales,
                                           None, layer.down_bias)
    _assert_close(bf16_tensor_to_f64(a), want)


def test_repeat_runs_are_bit_identical(moe_gpu, oracle_mod):
    import torch
    layer = workload("nvfp4_20b_decode_T8")
    dev = nvfp4_layer_to_device(layer)
    ids, w = oracle_mod.route(layer.logits, layer.k)
    first = run_nvfp4_forward(moe_gpu, dev, ids, w, layer).view(torch.int16).clone()
    for _ in range(4):
        assert torch.equal(first, run_nvfp4_forward(moe_gpu, dev, ids, w, layer).view(torch.int16))
    assert moe_gpu.moe_get_device_error() == 0


def test_nan_scale_gives_nan_and_flag(moe_gpu, oracle_mod):
    import torch
    layer = workload("nvfp4_tiny_woo")
    ids, w = oracle_mod.route(layer.logits, layer.k)
    e = int(ids[0, 0])
    dev = nvfp4_layer_to_device(layer)
    scales = layer.down.scales.copy()
    scales[e, 0, 0] = 0x7F
    dev["d_scales"] = to_dev(scales)
    out = run_nvfp4_forward(moe_gpu, dev, ids, w, layer)
    assert moe_gpu.moe_get_device_error() & moe_gpu.MOE_DEVERR_BAD_SCALE
    assert torch.isnan(out.float()[0, 0]).item()


def test_weight_on_input_with_bias_is_refused(moe_gpu):
    layer = workload("nvfp4_tiny_woo")
    dev = nvfp4_layer_to_device(layer)
    ids = np.zeros((layer.T, layer.k), np.int32)
    w = np.ones((layer.T, layer.k), np.float32)
    with pytest.raises(moe_gpu.MoEError) as ei:
        run_nvfp4_forward(moe_gpu, dev, ids, w, layer, flags=moe_gpu.MOE_FLAG_WEIGHT_ON_INPUT)
    assert ei.value.status == -1
