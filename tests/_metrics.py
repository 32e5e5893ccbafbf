"""Parity metrics shared by the tests (no layer arithmetic here)."""
import numpy as np

# Layer-output tolerance: bf16 output against the double-precision oracle.
REL_L2_TOL = 1e-2
MAX_ABS_OVER_RMS_TOL = 2e-2


def rel_l2(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def max_abs_over_rms(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(got - ref)) / max(rms, 1e-300))


def within_layer_tolerance(got, ref):
    return rel_l2(got, ref) <= REL_L2_TOL and max_abs_over_rms(got, ref) <= MAX_ABS_OVER_RMS_TOL


# Edge shapes outside the configured workloads (small H or I, unit biases, outputs
# whose max reaches ~10x their RMS) use a bound derived from the arithmetic: the
# bf16 rounding of the output moves a value v by up to 2^-8 |v|, and rounding each
# activation a_i (and, with the router weight on the input, each w*x) to the bf16
# MMA operand moves the down projection by at most 2^-9 sum_i |a_i W_i| per
# rounding, i.e. within 2^-8 of the magnitude envelope env the oracle reports (the
# fp32-golden plus magnitude-envelope parity test of MoE-Infinity PR #152).  So,
# elementwise, |got - want| <= 2e-2 RMS(want) + 2^-8 (|want| + env), rel-L2 <= 1e-2.
BF16_U2 = 2.0 ** -8


def envelope_excess_over_rms(got, want, env):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    rms = float(np.sqrt(np.mean(want * want)))
    excess = np.abs(got - want) - BF16_U2 * (np.abs(want) + np.asarray(env, np.float64))
    return float(np.max(excess)) / max(rms, 1e-300)


def within_envelope_tolerance(got, want, env):
    return rel_l2(got, want) <= REL_L2_TOL and envelope_excess_over_rms(got, want, env) <= MAX_ABS_OVER_RMS_TOL
