"""Pins for the NVFP4 expert variant of the CPU oracle.

NVFP4 experts: E2M1 codes with one E4M3 scale per 16 elements and a per-expert fp32
weight_scale_2 that multiplies each projection's matrix product before its bias
(FreeToken PR #838, review item "NVFP4 down scale vs. down bias": sum w*(s*y + b)).
Each check ties the oracle to something other than itself: torch's float8_e4m3fn
conversion, hand-derived worked examples, the already pinned MXFP4 path (scales
that are powers of two make the two formats carry the same weights), numpy matrix
products on the dense special case, linearity, and planted mistakes.  No GPU needed.
"""
import os

import numpy as np
import pytest

from mxfp4_expert_ffn_moe_b200.workloads import bf16_bits_to_f32, make_layer, workload
from tests._metrics import MAX_ABS_OVER_RMS_TOL, REL_L2_TOL, max_abs_over_rms, rel_l2

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


def _torch_e4m3(bytes_u8):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bytes_u8, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


# --------------------------------------------------------------------------- formats

def test_e4m3_matches_torch_float8_e4m3fn(oracle_mod):
    every = np.arange(256, dtype=np.uint8)
    want = _torch_e4m3(every)
    got = np.array([oracle_mod.e4m3_value(int(b)) for b in every])
    nan = np.isnan(want)
    assert list(np.flatnonzero(nan)) == [0x7F, 0xFF]
    assert np.all(np.isnan(got[nan]))
    np.testing.assert_array_equal(got[~nan], want[~nan])
    assert np.all(np.signbit(got[~nan]) == np.signbit(want[~nan]))


def test_e4m3_hand_values(oracle_mod):
    assert oracle_mod.e4m3_value(0x38) == 1.0
    assert oracle_mod.e4m3_value(0x7E) == 448.0            # largest finite
    assert oracle_mod.e4m3_value(0x08) == 2.0 ** -6        # smallest normal
    assert oracle_mod.e4m3_value(0x01) == 2.0 ** -9        # smallest subnormal
    assert oracle_mod.e4m3_value(0x07) == 7 / 8 * 2.0 ** -6
    assert oracle_mod.e4m3_value(0xB8) == -1.0
    assert oracle_mod.e4m3_value(0x3C) == 1.5


def test_nvfp4_dequant_worked_examples(oracle_mod):
    rows = _read_rows("nvfp4_dequant_worked_examples.txt")
    E = len(rows)
    blocks = np.zeros((E, 1, 8), np.uint8)
    scales = np.zeros((E, 1, 1), np.uint8)
    s2 = np.zeros(E, np.float32)
    for e, (b, s, f, _, _) in enumerate(rows):
        blocks[e, 0, :] = int(b, 16)
        scales[e, 0, 0] = int(s, 16)
        s2[e] = np.uint32(int(f, 16)).view(np.float32)
    out = oracle_mod.nvfp4_dequantize(blocks, scales, s2, E, 1, 16)
    for e, row in enumerate(rows):
        assert np.all(out[e, 0, 0::2] == int(row[3], 16)), (row, hex(out[e, 0, 0]))
        assert np.all(out[e, 0, 1::2] == int(row[4], 16)), (row, hex(out[e, 0, 1]))


def test_nvfp4_dequant_matches_library_decode(oracle_mod):
    # Codes through the golden E2M1 table, scales through torch's float8_e4m3fn, the
    # 16-element blocks laid out with numpy reshapes; without weight_scale_2 every
    # product is a bf16 value, so the comparison is exact.
    E, N, K = 3, 5, 96
    rng = np.random.default_rng(3)
    blocks = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    scales = rng.integers(0, 256, size=(E, N, K // 16), dtype=np.uint8)
    scales[(scales & 0x7F) == 0x7F] = 0x38        # NaN scales are pinned elsewhere
    table = np.array([float(v) for _, v in _read_rows("e2m1_table.txt")])
    codes = np.stack([blocks & 0xF, blocks >> 4], axis=-1).reshape(E, N, K)
    vals = table[codes] * np.repeat(_torch_e4m3(scales), 16, axis=-1)
    want = bf16_bits_to_f32(oracle_mod.nvfp4_dequantize(blocks, scales, None, E, N, K))
    np.testing.assert_array_equal(want.astype(np.float64), vals)
    # with weight_scale_2: within half a bf16 ulp of the exact product
    s2 = rng.uniform(0.5, 1.0, size=E).astype(np.float32)
    got = bf16_bits_to_f32(oracle_mod.nvfp4_dequantize(blocks, scales, s2, E, N, K)).astype(np.float64)
    exact = vals * s2.astype(np.float64)[:, None, None]
    nz = exact != 0
    ulp = 2.0 ** (np.floor(np.log2(np.abs(exact[nz]))) - 7)
    assert np.all(np.abs(got[nz] - exact[nz]) <= ulp / 2)
    assert np.all(got[~nz] == 0)


def test_nvfp4_dequant_planted_block32_fails(oracle_mod):
    E, N, K = 1, 4, 64
    rng = np.random.default_rng(4)
    blocks = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    scales = rng.integers(0x08, 0x38, size=(E, N, K // 16), dtype=np.uint8)
    good = oracle_mod.nvfp4_dequantize(blocks, scales, None, E, N, K)
    bad = oracle_mod.nvfp4_dequantize(blocks, scales, None, E, N, K,
                                      defect=oracle_mod.DEFECT_NVFP4_BLOCK32)
    assert np.any(good != bad)


# --------------------------------------------------------------------------- layer

def _nv_args(layer, ids, w, gu_s2="layer", d_s2="layer"):
    return (layer.x_bits, ids, w, layer.gate_up.blocks, layer.gate_up.scales,
            layer.gate_up.scale2 if isinstance(gu_s2, str) else gu_s2, layer.gate_up_bias,
            layer.down.blocks, layer.down.scales,
            layer.down.scale2 if isinstance(d_s2, str) else d_s2, layer.down_bias)


def _e8m0_to_e4m3(b):
    # 2^(b - 127) as an E4M3 byte: normal for exponents -6..8, subnormal m/8 * 2^-6 below
    ex = b.astype(np.int64) - 127
    assert np.all((ex >= -9) & (ex <= 8))
    normal = ((ex + 7) << 3).astype(np.int64)
    sub = (1 << np.clip(ex + 9, 0, 2)).astype(np.int64)
    return np.where(ex >= -6, normal, sub).astype(np.uint8)


def test_e8m0_to_e4m3_helper_is_exact(oracle_mod):
    b = np.arange(118, 136, dtype=np.uint8)
    got = np.array([oracle_mod.e4m3_value(int(v)) for v in _e8m0_to_e4m3(b)])
    np.testing.assert_array_equal(got, 2.0 ** (b.astype(np.float64) - 127))


@pytest.mark.parametrize("name", ["tiny_woo", "tiny_woi", "tiny_bias_heavy"])
def test_nvfp4_with_power_of_two_scales_equals_mxfp4(oracle_mod, name):
    # An MXFP4 bank re-expressed as NVFP4 (each E8M0 scale written as the E4M3 byte of
    # the same power of two, for both 16-element halves of its 32-element block, and
    # weight_scale_2 = 1) carries exactly the same weights: the NVFP4 path must give
    # the pinned MXFP4 result bit for bit.
    layer = workload(name)
    ids, w = oracle_mod.route(layer.logits, layer.k)
    want = oracle_mod.forward_tokens(layer.x_bits, ids, w, layer.gate_up.blocks, layer.gate_up.scales,
                                     layer.gate_up_bias, layer.down.blocks, layer.down.scales,
                                     layer.down_bias, weight_on_input=layer.weight_on_input)
    gu_sc = np.repeat(_e8m0_to_e4m3(layer.gate_up.scales), 2, axis=-1)
    d_sc = np.repeat(_e8m0_to_e4m3(layer.down.scales), 2, axis=-1)
    for gu_s2, d_s2 in ((None, None), (np.ones((layer.E, 2), np.float32), np.ones(layer.E, np.float32))):
        got = oracle_mod.nvfp4_forward_tokens(layer.x_bits, ids, w, layer.gate_up.blocks, gu_sc, gu_s2,
                                              layer.gate_up_bias, layer.down.blocks, d_sc, d_s2,
                                              layer.down_bias, weight_on_input=layer.weight_on_input)
        np.testing.assert_array_equal(got, want)
    E, N, K = layer.gate_up.shape
    np.testing.assert_array_equal(
        oracle_mod.nvfp4_dequantize(layer.gate_up.blocks, gu_sc, None, E, N, K),
        oracle_mod.dequantize(layer.gate_up.blocks, layer.gate_up.scales, E, N, K))


def test_nvfp4_dense_special_case_matches_numpy(oracle_mod):
    # E = k = 1, w = 1: a dense gated MLP.  Weights from the pinned dequantiser (no
    # weight_scale_2, so exact), the two per-projection scales applied to the numpy
    # matrix products before the biases.
    layer = make_layer(T=5, H=64, I=96, E=1, k=1, seed=31, fmt="nvfp4", bias_std=1.0)
    ids = np.zeros((5, 1), np.int32)
    w = np.ones((5, 1), np.float32)
    got = oracle_mod.nvfp4_forward_tokens(*_nv_args(layer, ids, w))
    H, I = layer.H, layer.I
    Wgu = bf16_bits_to_f32(oracle_mod.nvfp4_dequantize(layer.gate_up.blocks, layer.gate_up.scales,
                                                       None, 1, 2 * I, H))[0].astype(np.float64)
    Wd = bf16_bits_to_f32(oracle_mod.nvfp4_dequantize(layer.down.blocks, layer.down.scales,
                                                      None, 1, H, I))[0].astype(np.float64)
    x = bf16_bits_to_f32(layer.x_bits).astype(np.float64)
    sg, su = layer.gate_up.scale2[0].astype(np.float64)
    sd = float(layer.down.scale2[0])
    acc = x @ Wgu.T
    gb = layer.gate_up_bias[0].astype(np.float64)
    gate = sg * acc[:, 0::2] + gb[0::2]
    up = su * acc[:, 1::2] + gb[1::2]
    act = np.vectorize(oracle_mod.swiglu)(gate, up)
    want = sd * (act @ Wd.T) + layer.down_bias[0].astype(np.float64)
    assert rel_l2(got, want) < 1e-12


def test_nvfp4_down_scale_before_bias(oracle_mod):
    # y = s*acc + b: doubling the down weight_scale_2 adds exactly the bias-free output,
    # out(2s) - out(s) = sum_j w_j s acc_j = out(s) without the down bias.
    layer = workload("nvfp4_tiny_bias_heavy")
    ids, w = oracle_mod.route(layer.logits, layer.k)
    old = oracle_mod.nvfp4_forward_tokens(*_nv_args(layer, ids, w))
    new = oracle_mod.nvfp4_forward_tokens(*_nv_args(layer, ids, w, d_s2=2 * layer.down.scale2))
    args = list(_nv_args(layer, ids, w))
    args[10] = None
    nobias = oracle_mod.nvfp4_forward_tokens(*args)
    np.testing.assert_allclose(new - old, nobias, rtol=1e-9, atol=1e-9 * np.abs(old).max())
    # the ordering the review item rejects, sum w*s*(y + b), fails the same identity
    bad_old = oracle_mod.nvfp4_forward_tokens(*_nv_args(layer, ids, w),
                                              defect=oracle_mod.DEFECT_NVFP4_SCALE_AFTER_BIAS)
    bad_new = oracle_mod.nvfp4_forward_tokens(*_nv_args(layer, ids, w, d_s2=2 * layer.down.scale2),
                                              defect=oracle_mod.DEFECT_NVFP4_SCALE_AFTER_BIAS)
    assert np.max(np.abs((bad_new - bad_old) - nobias)) > 1e-3 * np.abs(old).max()


def test_nvfp4_gate_and_up_scales_apply_to_their_rows(oracle_mod):
    # Halving every gate row's E4M3 block scale (one exponent step: bytes >= 0x18 stay
    # normal) and doubling the gate weight_scale_2 leaves the layer unchanged, bit for
    # bit; doing the same to the up rows with the gate scale does not.
    layer = make_layer(T=6, H=128, I=64, E=3, k=2, seed=41, fmt="nvfp4", bias_std=1.0)
    gu_sc = layer.gate_up.scales.copy()
    gu_sc = np.maximum(gu_sc, 0x18).astype(np.uint8)
    ids, w = oracle_mod.route(layer.logits, layer.k)

    def run(scales, s2, defect=0):
        return oracle_mod.nvfp4_forward_tokens(layer.x_bits, ids, w, layer.gate_up.blocks, scales, s2,
                                               layer.gate_up_bias, layer.down.blocks, layer.down.scales,
                                               layer.down.scale2, layer.down_bias, defect=defect)

    base = run(gu_sc, layer.gate_up.scale2)
    halved = gu_sc.copy()
    halved[:, 0::2, :] -= 8                       # gate rows (even): exponent - 1
    s2 = layer.gate_up.scale2.copy()
    s2[:, 0] *= 2
    np.testing.assert_array_equal(run(halved, s2), base)
    swapped = run(halved, s2, defect=oracle_mod.DEFECT_NVFP4_GU_SCALE_SWAP)
    assert rel_l2(swapped, base) > REL_L2_TOL
    up_halved = gu_sc.copy()
    up_halved[:, 1::2, :] -= 8
    assert rel_l2(run(up_halved, s2), base) > REL_L2_TOL


def test_nvfp4_clamp_is_exercised_on_tiny_config(oracle_mod):
    layer = workload("nvfp4_tiny_woo")
    ids, _ = oracle_mod.route(layer.logits, layer.k)
    H, I, E = layer.H, layer.I, layer.E
    Wgu = bf16_bits_to_f32(oracle_mod.nvfp4_dequantize(layer.gate_up.blocks, layer.gate_up.scales, None,
                                                       E, 2 * I, H)).astype(np.float64)
    x = bf16_bits_to_f32(layer.x_bits).astype(np.float64)
    gates = []
    for t in range(layer.T):
        for e in ids[t]:
            h = layer.gate_up.scale2[e, 0] * (Wgu[e][0::2] @ x[t]) + layer.gate_up_bias[e][0::2]
            gates.append(h)
    frac = np.mean(np.concatenate(gates) > layer.limit)
    assert 0.02 < frac < 0.98


@pytest.mark.parametrize("defect,layer_name", [
    ("DEFECT_NVFP4_SCALE_AFTER_BIAS", "nvfp4_tiny_bias_heavy"),
    ("DEFECT_NVFP4_BLOCK32", "nvfp4_tiny_woo"),
    ("DEFECT_NVFP4_GU_SCALE_SWAP", "nvfp4_tiny_woo"),
    ("DEFECT_NIBBLE_SWAP", "nvfp4_tiny_woo"),
    ("DEFECT_NO_CLAMP", "nvfp4_tiny_woo"),
    ("DEFECT_NVFP4_BLOCK32", "nvfp4_tiny_woi"),
])
def test_nvfp4_planted_mistakes_exceed_layer_tolerance(oracle_mod, defect, layer_name):
    layer = workload(layer_name)
    ids, w = oracle_mod.route(layer.logits, layer.k)
    good = oracle_mod.nvfp4_forward_tokens(*_nv_args(layer, ids, w), weight_on_input=layer.weight_on_input)
    bad = oracle_mod.nvfp4_forward_tokens(*_nv_args(layer, ids, w), weight_on_input=layer.weight_on_input,
                                          defect=getattr(oracle_mod, defect))
    assert rel_l2(bad, good) > REL_L2_TOL or max_abs_over_rms(bad, good) > MAX_ABS_OVER_RMS_TOL
