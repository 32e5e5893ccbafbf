"""Pins for the router linear layer of the CPU oracle (logits = x . W_r^T + b_r, the
gpt-oss mlp.router with its bias; FreeToken PR #838).  Hand values, numpy matrix
products over the decoded bf16 operands, and planted mistakes.  No GPU needed."""
import numpy as np

from mxfp4_expert_ffn_moe_b200.workloads import bf16_bits_to_f32, f32_to_bf16_bits, make_router


def test_router_hand_values(oracle_mod):
    # x = [1, 2], W_r = [[1, 0.5], [-1, 3]], b = [0.25, -1]:
    #   logit 0 = 1 + 1 + 0.25 = 2.25, logit 1 = -1 + 6 - 1 = 4
    x = f32_to_bf16_bits(np.float32([[1.0, 2.0]]))
    w = f32_to_bf16_bits(np.float32([[1.0, 0.5], [-1.0, 3.0]]))
    got = oracle_mod.router_logits(x, w, np.float32([0.25, -1.0]))
    np.testing.assert_array_equal(got, [[2.25, 4.0]])
    np.testing.assert_array_equal(oracle_mod.router_logits(x, w, None), [[2.0, 5.0]])


def test_router_matches_numpy_matmul(oracle_mod):
    r = make_router(T=7, H=320, E=12, k=3, seed=5)
    got = oracle_mod.router_logits(r.x_bits, r.w_bits, r.bias)
    x = bf16_bits_to_f32(r.x_bits).astype(np.float64)
    w = bf16_bits_to_f32(r.w_bits).astype(np.float64)
    want = x @ w.T + r.bias.astype(np.float64)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-13)


def test_router_planted_mistakes_differ(oracle_mod):
    # the bias dropped, or W_r read transposed (square case), moves every logit row
    r = make_router(T=6, H=64, E=64, k=2, seed=6)
    good = oracle_mod.router_logits(r.x_bits, r.w_bits, r.bias)
    no_bias = oracle_mod.router_logits(r.x_bits, r.w_bits, None)
    assert np.all(np.abs(good - no_bias).max(axis=1) > 1e-3)
    transposed = oracle_mod.router_logits(r.x_bits, np.ascontiguousarray(r.w_bits.T), r.bias)
    assert np.all(np.abs(good - transposed).max(axis=1) > 1e-2)


def test_router_workload_logits_have_unit_scale(oracle_mod):
    # the synthetic router gives logits of about unit spread (as the layer workloads'
    # N(0, 1) logits), so top-k decisions are neither all ties nor all far apart
    r = make_router(T=64, H=2880, E=32, k=4, seed=0)
    l = oracle_mod.router_logits(r.x_bits, r.w_bits, r.bias)
    assert 0.7 < float(l.std()) < 1.4
