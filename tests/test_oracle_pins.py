"""Pins for the CPU oracle: each check ties it to something other than itself.

Hand-written values from the element-format definitions (golden files), closed
forms, invariants of the layer, special cases that reduce to numpy routines, brute
force on tiny inputs, and planted mistakes that the parity tolerance must catch.
No GPU needed.
"""
import itertools
import math
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


# --------------------------------------------------------------------------- formats

def test_e2m1_table_matches_golden(oracle_mod):
    rows = _read_rows("e2m1_table.txt")
    assert len(rows) == 16
    for code, val in rows:
        got = oracle_mod.e2m1_value(int(code))
        want = float(val)
        assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want), (code, got, want)


def test_e8m0_values(oracle_mod):
    assert oracle_mod.e8m0_value(127) == 1.0
    assert oracle_mod.e8m0_value(128) == 2.0
    assert oracle_mod.e8m0_value(126) == 0.5
    assert oracle_mod.e8m0_value(0) == 2.0 ** -127
    assert oracle_mod.e8m0_value(254) == 2.0 ** 127
    assert math.isnan(oracle_mod.e8m0_value(255))


def test_bf16_rounding_against_numpy_float32_path(oracle_mod):
    # For values already representable in float32, bf16 RNE equals the classic
    # float32 bit trick (round the upper 16 bits, ties to even).  Independent
    # implementation: numpy integer arithmetic on the float32 bit pattern.
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(2000).astype(np.float32),
        (rng.standard_normal(500) * 1e-38).astype(np.float32),   # subnormal region
        np.float32([0.0, -0.0, 1.0, 3.0e38, -3.0e38, 1.00390625, 1.01171875]),
    ])
    u = vals.view(np.uint32).astype(np.uint64)
    want = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    got = np.array([oracle_mod.double_to_bf16(float(v)) for v in vals], dtype=np.uint16)
    np.testing.assert_array_equal(got, want)
    assert oracle_mod.double_to_bf16(float("inf")) == 0x7F80
    assert oracle_mod.double_to_bf16(float("-inf")) == 0xFF80
    assert oracle_mod.double_to_bf16(float("nan")) == 0x7FC0
    # ties: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 -> even (1.0)
    assert oracle_mod.double_to_bf16(1.0 + 2.0 ** -8) == 0x3F80
    assert oracle_mod.double_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82


def test_dequant_worked_examples(oracle_mod):
    rows = _read_rows("dequant_worked_examples.txt")
    # One row of K = 32 elements per example: the byte repeated 16 times.
    E, N, K = 1, len(rows), 32
    blocks = np.zeros((E, N, K // 2), np.uint8)
    scales = np.zeros((E, N, K // 32), np.uint8)
    for n, (b, s, _, _) in enumerate(rows):
        blocks[0, n, :] = int(b, 16)
        scales[0, n, 0] = int(s)
    out = oracle_mod.dequantize(blocks, scales, E, N, K)
    for n, (_, _, even, odd) in enumerate(rows):
        assert np.all(out[0, n, 0::2] == int(even, 16)), (rows[n], hex(out[0, n, 0]))
        assert np.all(out[0, n, 1::2] == int(odd, 16)), (rows[n], hex(out[0, n, 1]))


def test_dequant_block_and_row_indexing(oracle_mod):
    # Each scale byte covers exactly 32 consecutive elements of one row: give every
    # block a distinct scale and every element code 2 (= 1.0); then element kk of
    # row n must equal 2^(s[n, kk // 32] - 127).  A shifted block index fails this.
    E, N, K = 2, 3, 128
    blocks = np.full((E, N, K // 2), 0x22, np.uint8)
    scales = (100 + np.arange(E * N * K // 32) % 50).astype(np.uint8).reshape(E, N, K // 32)
    out = oracle_mod.dequantize(blocks, scales, E, N, K)
    vals = bf16_bits_to_f32(out).astype(np.float64)
    for e in range(E):
        for n in range(N):
            for kk in range(K):
                assert vals[e, n, kk] == 2.0 ** (int(scales[e, n, kk // 32]) - 127)


def test_dequant_planted_mistakes_fail_golden(oracle_mod):
    rows = _read_rows("dequant_worked_examples.txt")[:6]
    E, N, K = 1, len(rows), 32
    blocks = np.zeros((E, N, K // 2), np.uint8)
    scales = np.zeros((E, N, K // 32), np.uint8)
    for n, (b, s, _, _) in enumerate(rows):
        blocks[0, n, :] = int(b, 16)
        scales[0, n, 0] = int(s)
    want = np.array([[int(r[2], 16), int(r[3], 16)] for r in rows])
    for defect in (oracle_mod.DEFECT_NIBBLE_SWAP, oracle_mod.DEFECT_E8M0_BIAS_126):
        out = oracle_mod.dequantize(blocks, scales, E, N, K, defect=defect)
        got = out[0, :, :2].astype(np.int64)
        assert not np.array_equal(got, want)


# --------------------------------------------------------------------------- routing

def _brute_force_topk(l, k):
    """The unique k-subset whose every member beats every non-member under
    (value desc, index asc), ordered by the same rule."""
    E = len(l)

    def beats(i, j):
        return l[i] > l[j] or (l[i] == l[j] and i < j)

    for sub in itertools.combinations(range(E), k):
        rest = [j for j in range(E) if j not in sub]
        if all(beats(i, j) for i in sub for j in rest):
            return sorted(sub, key=lambda i: (-l[i], i))
    raise AssertionError("no top-k subset")


def test_route_brute_force_tiny(oracle_mod):
    rng = np.random.default_rng(3)
    for E, k in [(4, 2), (5, 3), (6, 1), (6, 6), (7, 4)]:
        logits = rng.standard_normal((20, E)).astype(np.float32)
        logits[0, :] = 1.0                              # all tied
        logits[1, : E // 2] = logits[1, E - 1]          # partial ties
        ids, w = oracle_mod.route(logits, k)
        for t in range(logits.shape[0]):
            assert list(ids[t]) == _brute_force_topk(list(logits[t]), k)
            assert abs(float(np.sum(w[t], dtype=np.float64)) - 1.0) < 1e-6
            assert np.all(np.diff(w[t]) <= 0)


def test_route_matches_numpy_stable_argsort(oracle_mod):
    layer = workload("120b_zipf_T256")
    ids, w = oracle_mod.route(layer.logits, 4)
    order = np.argsort(-layer.logits, axis=1, kind="stable")[:, :4]
    np.testing.assert_array_equal(ids, order)


def test_route_worked_examples(oracle_mod):
    ids, w = oracle_mod.route(np.array([[1.0, 3.0, 2.0, 3.0]], np.float32), 2)
    assert list(ids[0]) == [1, 3]          # tie at 3.0 goes to the lower expert id
    assert w[0, 0] == np.float32(0.5) and w[0, 1] == np.float32(0.5)
    ids, w = oracle_mod.route(np.array([[0.0, math.log(3.0)]], np.float32), 2)
    assert list(ids[0]) == [1, 0]
    assert abs(w[0, 0] - 0.75) < 1e-7 and abs(w[0, 1] - 0.25) < 1e-7
    ids, w = oracle_mod.route(np.array([[0.3, -2.0, 9.0]], np.float32), 1)
    assert list(ids[0]) == [2] and w[0, 0] == 1.0


def test_route_softmax_ratio_closed_form(oracle_mod):
    rng = np.random.default_rng(4)
    logits = rng.standard_normal((50, 16)).astype(np.float32)
    ids, w = oracle_mod.route(logits, 4)
    for t in range(50):
        l_sel = logits[t, ids[t]].astype(np.float64)
        for j in range(1, 4):
            assert abs(w[t, j] / w[t, 0] - math.exp(l_sel[j] - l_sel[0])) < 1e-6


# --------------------------------------------------------------------------- SwiGLU

def test_swiglu_closed_forms(oracle_mod):
    sw = oracle_mod.swiglu
    for up in (-9.0, -3.0, 0.0, 2.5, 11.0):
        assert sw(0.0, up) == 0.0                       # gate 0 -> 0
    for gate in (-12.0, -1.0, 0.5, 3.0, 7.0, 40.0):
        assert sw(gate, -1.0) == 0.0                    # up = -1 -> (u + 1) = 0
    for up in (-2.0, 0.0, 5.0):
        assert sw(9.5, up) == sw(7.0, up)               # one-sided gate clamp at limit
        assert sw(1e6, up) == sw(7.0, up)
    for gate in (-4.0, 0.7, 8.0):
        assert sw(gate, 8.0) == sw(gate, 7.0)           # up clamp, upper side
        assert sw(gate, -30.0) == sw(gate, -7.0)        # up clamp, lower side
    # negative gates are not clamped: g*sigmoid(a g) - (-g)*sigmoid(-a g) = g
    for g in (0.25, 1.0, 3.0, 6.5):
        for up in (0.0, 1.5, -0.5):
            lhs = sw(g, up) - sw(-g, up)
            assert abs(lhs - (up + 1.0) * g) < 1e-12 * max(1.0, abs(lhs))
    assert sw(-50.0, 0.0) < 0.0 and sw(-50.0, 0.0) > -1e-30


def test_swiglu_hand_values(oracle_mod):
    # sigmoid(1.702) = 1 / (1 + e^-1.702); e^-1.702 = 0.18232..., by hand 0.845795
    assert abs(oracle_mod.swiglu(1.0, 0.0) - 0.845795) < 2e-6
    # gate clamped at 7: 7 * sigmoid(11.914) * (1 + 1); sigmoid(11.914) = 1 - 6.69e-6
    assert abs(oracle_mod.swiglu(50.0, 1.0) - 14.0 * (1.0 - 6.69e-6)) < 1e-6


# --------------------------------------------------------------------------- layer

def _args(layer, ids, w):
    return (layer.x_bits, ids, w, layer.gate_up.blocks, layer.gate_up.scales, layer.gate_up_bias,
            layer.down.blocks, layer.down.scales, layer.down_bias)


@pytest.fixture(scope="module")
def tiny_woo():
    return workload("tiny_woo")


@pytest.fixture(scope="module")
def tiny_woi():
    return workload("tiny_woi")


def test_two_formulations_agree(oracle_mod, tiny_woo, tiny_woi):
    for layer in (tiny_woo, tiny_woi):
        ids, w = oracle_mod.route(layer.logits, layer.k)
        a = oracle_mod.forward_tokens(*_args(layer, ids, w), weight_on_input=layer.weight_on_input)
        b = oracle_mod.forward_grouped(*_args(layer, ids, w), weight_on_input=layer.weight_on_input)
        assert rel_l2(a, b) < 1e-12
        assert np.max(np.abs(a - b)) <= 1e-9 * np.max(np.abs(a))


def test_dense_special_case_matches_numpy(oracle_mod):
    # E = k = 1 with weight 1 is a dense gated MLP; build it from the pinned
    # dequantiser and activation with numpy float64 matrix products.
    layer = make_layer(T=5, H=64, I=96, E=1, k=1, seed=11)
    ids = np.zeros((5, 1), np.int32)
    w = np.ones((5, 1), np.float32)
    got = oracle_mod.forward_tokens(*_args(layer, ids, w))
    H, I = layer.H, layer.I
    Wgu = bf16_bits_to_f32(oracle_mod.dequantize(layer.gate_up.blocks, layer.gate_up.scales, 1, 2 * I, H))[0]
    Wd = bf16_bits_to_f32(oracle_mod.dequantize(layer.down.blocks, layer.down.scales, 1, H, I))[0]
    x = bf16_bits_to_f32(layer.x_bits).astype(np.float64)
    h = x @ Wgu.astype(np.float64).T + layer.gate_up_bias[0].astype(np.float64)
    act = np.vectorize(oracle_mod.swiglu)(h[:, 0::2], h[:, 1::2])
    want = act @ Wd.astype(np.float64).T + layer.down_bias[0].astype(np.float64)
    assert rel_l2(got, want) < 1e-12


def test_token_permutation_equivariance(oracle_mod, tiny_woo):
    layer = tiny_woo
    ids, w = oracle_mod.route(layer.logits, layer.k)
    base = oracle_mod.forward_tokens(*_args(layer, ids, w))
    perm = np.random.default_rng(5).permutation(layer.T)
    args = list(_args(layer, ids, w))
    args[0], args[1], args[2] = layer.x_bits[perm], ids[perm], w[perm]
    got = oracle_mod.forward_tokens(*args)
    np.testing.assert_allclose(got, base[perm], rtol=0, atol=0)


def test_expert_relabelling_invariance(oracle_mod, tiny_woo):
    layer = tiny_woo
    ids, w = oracle_mod.route(layer.logits, layer.k)
    base = oracle_mod.forward_tokens(*_args(layer, ids, w))
    pi = np.array([2, 0, 3, 1])          # new expert index of old expert e is pi[e]
    inv = np.argsort(pi)
    args = list(_args(layer, ids, w))
    args[1] = pi[ids].astype(np.int32)
    for pos in (3, 4, 5, 6, 7, 8):
        args[pos] = args[pos][inv]
    got = oracle_mod.forward_tokens(*args)
    np.testing.assert_array_equal(got, base)


def test_down_bias_is_weighted_linearly(oracle_mod, tiny_woo):
    # out(b + d) - out(b) = sum_j w_j d[e_j]   (the bias sits inside the routing weight)
    layer = tiny_woo
    ids, w = oracle_mod.route(layer.logits, layer.k)
    base = oracle_mod.forward_tokens(*_args(layer, ids, w))
    d = np.random.default_rng(6).standard_normal(layer.down_bias.shape).astype(np.float32)
    args = list(_args(layer, ids, w))
    args[8] = layer.down_bias + d
    got = oracle_mod.forward_tokens(*args)
    delta_b = (layer.down_bias + d).astype(np.float64) - layer.down_bias.astype(np.float64)
    want = np.einsum("tj,tjh->th", w.astype(np.float64), delta_b[ids])
    np.testing.assert_allclose(got - base, want, rtol=1e-9, atol=1e-9 * np.abs(base).max())


def test_bias_after_block_scale(oracle_mod, tiny_woo):
    # Raising every down-projection scale byte by one doubles each expert's matrix
    # product but not its bias: out_new - out_old = out_old computed without the
    # down bias (the sum w*(s*y + b) ordering of the FreeToken review).
    layer = tiny_woo
    ids, w = oracle_mod.route(layer.logits, layer.k)
    old = oracle_mod.forward_tokens(*_args(layer, ids, w))
    args = list(_args(layer, ids, w))
    args[7] = (layer.down.scales + 1).astype(np.uint8)
    new = oracle_mod.forward_tokens(*args)
    args = list(_args(layer, ids, w))
    args[8] = None
    nobias = oracle_mod.forward_tokens(*args)
    np.testing.assert_allclose(new - old, nobias, rtol=1e-9, atol=1e-9 * np.abs(old).max())


def test_weight_on_input_reduces_to_output_mode_when_weights_are_one(oracle_mod, tiny_woi):
    layer = tiny_woi
    ids, _ = oracle_mod.route(layer.logits, layer.k)
    ones = np.ones_like(ids, dtype=np.float32)
    a = oracle_mod.forward_tokens(*_args(layer, ids, ones), weight_on_input=True)
    b = oracle_mod.forward_tokens(*_args(layer, ids, ones), weight_on_input=False)
    np.testing.assert_array_equal(a, b)


def test_weight_on_input_scales_the_input(oracle_mod, tiny_woi):
    # k = 1, E = 1: weight on input means the expert sees w*x.
    layer = make_layer(T=3, H=64, I=64, E=1, k=1, seed=12, biases=False)
    ids = np.zeros((3, 1), np.int32)
    w = np.full((3, 1), 0.375, np.float32)
    got = oracle_mod.forward_tokens(*_args(layer, ids, w), weight_on_input=True)
    H, I = layer.H, layer.I
    Wgu = bf16_bits_to_f32(oracle_mod.dequantize(layer.gate_up.blocks, layer.gate_up.scales, 1, 2 * I, H))[0]
    Wd = bf16_bits_to_f32(oracle_mod.dequantize(layer.down.blocks, layer.down.scales, 1, H, I))[0]
    x = 0.375 * bf16_bits_to_f32(layer.x_bits).astype(np.float64)
    h = x @ Wgu.astype(np.float64).T
    want = np.vectorize(oracle_mod.swiglu)(h[:, 0::2], h[:, 1::2]) @ Wd.astype(np.float64).T
    assert rel_l2(got, want) < 1e-12


def test_weight_on_input_bias_added_unweighted(oracle_mod):
    layer = make_layer(T=6, H=64, I=64, E=3, k=2, seed=13)
    ids, w = oracle_mod.route(layer.logits, 2)
    base = oracle_mod.forward_tokens(*_args(layer, ids, w), weight_on_input=True)
    args = list(_args(layer, ids, w))
    d = np.random.default_rng(7).standard_normal(layer.down_bias.shape).astype(np.float32)
    args[8] = layer.down_bias + d
    got = oracle_mod.forward_tokens(*args, weight_on_input=True)
    delta_b = (layer.down_bias + d).astype(np.float64) - layer.down_bias.astype(np.float64)
    want = delta_b[ids].sum(axis=1)
    np.testing.assert_allclose(got - base, want, rtol=1e-9, atol=1e-9 * np.abs(base).max())


def test_clamp_is_exercised_on_tiny_config(oracle_mod, tiny_woo):
    # Non-vacuity: under the workload distributions some gate pre-activations lie
    # above the limit and some below, so the clamp both acts and does not act.
    layer = tiny_woo
    ids, _ = oracle_mod.route(layer.logits, layer.k)
    H, I, E = layer.H, layer.I, layer.E
    Wgu = bf16_bits_to_f32(oracle_mod.dequantize(layer.gate_up.blocks, layer.gate_up.scales, E, 2 * I, H))
    x = bf16_bits_to_f32(layer.x_bits).astype(np.float64)
    gates = []
    for t in range(layer.T):
        for e in ids[t]:
            h = Wgu[e].astype(np.float64) @ x[t] + layer.gate_up_bias[e]
            gates.append(h[0::2])
    g = np.concatenate(gates)
    frac = np.mean(g > layer.limit)
    assert 0.02 < frac < 0.98


@pytest.mark.parametrize("defect,layer_name", [
    ("DEFECT_NIBBLE_SWAP", "tiny_woo"),
    ("DEFECT_E8M0_BIAS_126", "tiny_woo"),
    ("DEFECT_GATE_ZERO", "tiny_woo"),
    ("DEFECT_NO_CLAMP", "tiny_woo"),
    ("DEFECT_UNINTERLEAVED", "tiny_woo"),
    ("DEFECT_DOWN_BIAS_UNWEIGHTED", "tiny_bias_heavy"),
    ("DEFECT_DOWN_BIAS_IN_SCALE", "tiny_bias_heavy"),
    ("DEFECT_NIBBLE_SWAP", "tiny_woi"),
    ("DEFECT_NO_CLAMP", "tiny_woi"),
])
def test_planted_mistakes_exceed_layer_tolerance(oracle_mod, defect, layer_name):
    # Each planted mistake must move the layer output beyond the parity tolerance,
    # so a CUDA path carrying it could not pass the parity tests.
    layer = workload(layer_name)
    ids, w = oracle_mod.route(layer.logits, layer.k)
    good = oracle_mod.forward_tokens(*_args(layer, ids, w), weight_on_input=layer.weight_on_input)
    bad = oracle_mod.forward_tokens(*_args(layer, ids, w), weight_on_input=layer.weight_on_input,
                                    defect=getattr(oracle_mod, defect))
    assert rel_l2(bad, good) > REL_L2_TOL or max_abs_over_rms(bad, good) > MAX_ABS_OVER_RMS_TOL


def test_config_biases_are_too_small_for_the_layer_tolerance(oracle_mod):
    # Why the bias-heavy test case exists: with N(0, 0.02) biases a misplaced down
    # bias stays far inside the layer tolerance, so bias semantics need their own case.
    layer = workload("tiny_woo")
    ids, w = oracle_mod.route(layer.logits, layer.k)
    good = oracle_mod.forward_tokens(*_args(layer, ids, w))
    bad = oracle_mod.forward_tokens(*_args(layer, ids, w),
                                    defect=oracle_mod.DEFECT_DOWN_BIAS_UNWEIGHTED)
    assert rel_l2(bad, good) < REL_L2_TOL


def test_planted_woi_bias_mistake_is_caught(oracle_mod):
    # The apply_router_weight_on_input review item: a weighted down bias in that mode.
    layer = make_layer(T=8, H=128, I=128, E=4, k=2, seed=0)
    ids, w = oracle_mod.route(layer.logits, 2)
    good = oracle_mod.forward_tokens(*_args(layer, ids, w), weight_on_input=True)
    bad = oracle_mod.forward_tokens(*_args(layer, ids, w), weight_on_input=True,
                                    defect=oracle_mod.DEFECT_WOI_BIAS_WEIGHTED)
    # biases are small (N(0, 0.02)); the mistake must still be visible per element
    assert np.max(np.abs(bad - good)) > 1e-3


def test_envelope_bounds_output_and_matches_dense_special_case(oracle_mod, tiny_woo):
    # Triangle inequality: |out| <= env elementwise.
    layer = tiny_woo
    ids, w = oracle_mod.route(layer.logits, layer.k)
    out, env = oracle_mod.forward_tokens(*_args(layer, ids, w), envelope=True)
    assert np.all(np.abs(out) <= env * (1 + 1e-12))
    np.testing.assert_array_equal(out, oracle_mod.forward_tokens(*_args(layer, ids, w)))
    # Dense special case (E = k = 1, w = 1): env = |W_d| @ |a| + |b_d| with numpy.
    layer = make_layer(T=4, H=64, I=96, E=1, k=1, seed=21)
    ids1 = np.zeros((4, 1), np.int32)
    w1 = np.ones((4, 1), np.float32)
    _, env = oracle_mod.forward_tokens(*_args(layer, ids1, w1), envelope=True)
    H, I = layer.H, layer.I
    Wgu = bf16_bits_to_f32(oracle_mod.dequantize(layer.gate_up.blocks, layer.gate_up.scales, 1, 2 * I, H))[0]
    Wd = bf16_bits_to_f32(oracle_mod.dequantize(layer.down.blocks, layer.down.scales, 1, H, I))[0]
    x = bf16_bits_to_f32(layer.x_bits).astype(np.float64)
    h = x @ Wgu.astype(np.float64).T + layer.gate_up_bias[0].astype(np.float64)
    act = np.vectorize(oracle_mod.swiglu)(h[:, 0::2], h[:, 1::2])
    want = np.abs(act) @ np.abs(Wd.astype(np.float64)).T + np.abs(layer.down_bias[0].astype(np.float64))
    assert rel_l2(env, want) < 1e-12


@pytest.mark.parametrize("layer_name", ["tiny_wide", "20b_decode_wide_T8"])
def test_dropped_second_split_term_exceeds_layer_tolerance(oracle_mod, layer_name):
    # The decode tiles feed the tensor core two E4M3 terms per activation element at a
    # power-of-two scale per 32-element block; on blocks spanning 2^20 a kernel that
    # kept only the first term would be off by far more than the layer tolerance, so
    # the GPU test on these layers (tests/test_gpu_forward.py) fails if it does.
    layer = workload(layer_name)
    ids, w = oracle_mod.route(layer.logits, layer.k)
    args = (layer.x_bits, ids, w, layer.gate_up.blocks, layer.gate_up.scales, layer.gate_up_bias,
            layer.down.blocks, layer.down.scales, layer.down_bias)
    want = oracle_mod.forward_tokens(*args)
    bad = oracle_mod.forward_tokens(*args, defect=oracle_mod.DEFECT_OPERAND_E4M3_HI_ONLY)
    assert rel_l2(bad, want) > 2 * REL_L2_TOL
    assert max_abs_over_rms(bad, want) > 2 * MAX_ABS_OVER_RMS_TOL
