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
