"""The edge-shape parity bound is not so loose that it hides a mistake.

The GPU edge-shape tests (small H or I, unit biases) compare the layer against the
oracle with the bound of tests/_metrics.py, which widens the configured max-abs
bound by 2^-8 (|want| + env) to absorb the bf16 rounding of the activation operand.
Here, on the CPU and on exactly those shapes, every planted mistake of the oracle
that changes the layer's structure (nibble order, E8M0 bias, gate projection,
clamp, gate/up interleave) must still be rejected by that bound; and every planted
mistake that the configured bound rejects with a margin must be rejected by the
widened one too.

Bias-placement mistakes cannot be resolved on shapes whose output RMS is ~100 times
the unit bias (a misplaced bias then moves the output by well under 1 %, inside any
1 % tolerance); they are pinned on the bias-heavy tiny layer by
tests/test_oracle_pins.py instead.  No GPU needed.
"""
import numpy as np
import pytest

from mxfp4_expert_ffn_moe_b200.workloads import make_layer
from tests._metrics import (MAX_ABS_OVER_RMS_TOL, REL_L2_TOL, max_abs_over_rms, rel_l2,
                            within_envelope_tolerance)

# the MXFP4 edge shapes of tests/test_gpu_forward.py (T, H, I, E, k, weight on input)
EDGE_SHAPES = [
    (1, 64, 64, 1, 1, False),
    (37, 192, 320, 5, 3, False),
    (130, 128, 64, 3, 2, True),
    (3, 256, 128, 16, 4, False),
    (200, 64, 128, 2, 2, False),
    (3, 8192, 64, 4, 2, False),
]
STRUCTURAL = ["DEFECT_NIBBLE_SWAP", "DEFECT_E8M0_BIAS_126", "DEFECT_GATE_ZERO", "DEFECT_NO_CLAMP",
              "DEFECT_UNINTERLEAVED"]
BIAS = ["DEFECT_DOWN_BIAS_UNWEIGHTED", "DEFECT_DOWN_BIAS_IN_SCALE"]


def _layer_and_want(oracle, shape):
    T, H, I, E, k, woi = shape
    L = make_layer(T, H, I, E, k, seed=T + H, biases=not woi, weight_on_input=woi, bias_std=1.0,
                   name=f"edge_{T}_{H}_{I}_{E}_{k}")
    ids, w = oracle.route(L.logits, L.k)
    args = (L.x_bits, ids, w, L.gate_up.blocks, L.gate_up.scales, L.gate_up_bias, L.down.blocks,
            L.down.scales, L.down_bias)
    want, env = oracle.forward_tokens(*args, weight_on_input=woi, envelope=True)
    return args, woi, want, env


@pytest.mark.parametrize("shape", EDGE_SHAPES, ids=lambda s: "x".join(map(str, s[:5])) + ("_woi" if s[5] else ""))
def test_edge_bound_rejects_planted_mistakes(oracle_mod, shape):
    args, woi, want, env = _layer_and_want(oracle_mod, shape)
    assert within_envelope_tolerance(want, want, env)
    for name in STRUCTURAL + BIAS:
        bad = oracle_mod.forward_tokens(*args, weight_on_input=woi, defect=getattr(oracle_mod, name))
        plain_rejects_with_margin = (rel_l2(bad, want) > REL_L2_TOL or
                                     max_abs_over_rms(bad, want) > 1.5 * MAX_ABS_OVER_RMS_TOL)
        if name in STRUCTURAL or plain_rejects_with_margin:
            assert not within_envelope_tolerance(bad, want, env), (name, shape)
