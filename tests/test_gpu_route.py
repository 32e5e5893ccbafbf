"""moe_route on the GPU against the CPU oracle: ids bit-exact, weights to fp32 rounding."""
import numpy as np
import pytest

from mxfp4_expert_ffn_moe_b200.workloads import workload
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu


def _route(moe, logits, k):
    import torch
    ids, w = moe.moe_route(to_dev(logits), k)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("T,E,k", [(1, 4, 1), (8, 4, 2), (37, 32, 4), (4096, 32, 4),
                                   (300, 128, 4), (65, 200, 8), (5, 256, 8), (9, 7, 7)])
def test_route_matches_oracle(moe_gpu, oracle_mod, T, E, k):
    rng = np.random.default_rng(T * 7 + E)
    logits = rng.standard_normal((T, E), dtype=np.float32)
    logits[0, :] = 0.25                       # a fully tied row
    if T > 2:
        logits[2, ::3] = logits[2, 1]         # partial ties
    ids, w = _route(moe_gpu, logits, k)
    ids_o, w_o = oracle_mod.route(logits, k)
    np.testing.assert_array_equal(ids, ids_o)
    np.testing.assert_allclose(w, w_o, rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(w.astype(np.float64).sum(axis=1), 1.0, atol=1e-6)


@pytest.mark.parametrize("name", ["20b_prefill_T4096", "120b_zipf_T8192"])
def test_route_full_size_workloads(moe_gpu, oracle_mod, name):
    layer = workload(name)
    ids, w = _route(moe_gpu, layer.logits, layer.k)
    ids_o, w_o = oracle_mod.route(layer.logits, layer.k)
    np.testing.assert_array_equal(ids, ids_o)
    np.testing.assert_allclose(w, w_o, rtol=1e-6, atol=1e-7)


def test_nan_logits_are_never_chosen_and_short_rows_are_flagged(moe_gpu, oracle_mod):
    # NaN logits are skipped; a token with at least k other logits routes exactly as
    # the oracle does over its non-NaN logits, a token with fewer gets id -1 and weight
    # 0 in its empty slots (softmax over the chosen ones) and raises the logit flag
    T, E, k = 6, 8, 4
    rng = np.random.default_rng(21)
    logits = rng.standard_normal((T, E), dtype=np.float32)
    logits[0, [1, 5]] = np.nan                    # 6 finite logits left: full routing
    logits[1, :6] = np.nan                        # 2 left: two empty slots
    logits[2, :] = np.nan                         # none left
    moe_gpu.moe_get_device_error()
    ids, w = _route(moe_gpu, logits, k)
    assert moe_gpu.moe_get_device_error() & moe_gpu.MOE_DEVERR_BAD_LOGIT
    for t in (0, 3, 4, 5):
        row = np.where(np.isnan(logits[t]), -np.inf, logits[t])[None, :]
        ids_o, w_o = oracle_mod.route(row.astype(np.float32), k)
        np.testing.assert_array_equal(ids[t], ids_o[0])
        np.testing.assert_allclose(w[t], w_o[0], rtol=1e-6, atol=1e-7)
    ids_o, w_o = oracle_mod.route(logits[1:2, 6:], 2)
    np.testing.assert_array_equal(ids[1], np.concatenate([ids_o[0] + 6, [-1, -1]]))
    np.testing.assert_allclose(w[1], np.concatenate([w_o[0], [0.0, 0.0]]), rtol=1e-6, atol=1e-7)
    np.testing.assert_array_equal(ids[2], [-1] * k)
    np.testing.assert_array_equal(w[2], [0.0] * k)
