"""moe_router_route (router linear layer fused with routing) on the GPU against the
CPU oracle.

The logits are fp32 sums of exact bf16 products on the tensor cores, compared with
the double-precision oracle within the accumulation bound (H + 1) * 2^-23 * env,
env = |x| . |W_r|^T + |b_r|.  The routing decision is taken in the kernel's
precision: the oracle's routing of the GPU's own logits must give the same ids bit
for bit (weights to fp32 rounding), and the standalone routing kernel on those
logits the same bits.  Tokens whose k-th and (k+1)-th oracle logits are further
apart than twice the bound must also pick the oracle's experts.
"""
import numpy as np
import pytest

from mxfp4_expert_ffn_moe_b200.workloads import bf16_bits_to_f32, make_router, router_workload
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu


def _run(moe, r, want_logits=True, bias=True):
    import torch
    x = to_dev(r.x_bits, torch.bfloat16)
    w = to_dev(r.w_bits, torch.bfloat16)
    b = to_dev(r.bias) if (bias and r.bias is not None) else None
    res = moe.moe_router_route(x, w, b, r.k, want_logits=want_logits)
    torch.cuda.synchronize()
    return res


def _check(moe, oracle, r, rows=None, bias=True):
    import torch
    ids_d, w_d, lg_d = _run(moe, r, bias=bias)
    ids, w, lg = ids_d.cpu().numpy(), w_d.cpu().numpy(), lg_d.cpu().numpy()
    b = r.bias if bias else None
    rows = np.arange(r.x_bits.shape[0]) if rows is None else rows
    want = oracle.router_logits(r.x_bits[rows], r.w_bits, b)
    x = np.abs(bf16_bits_to_f32(r.x_bits[rows]).astype(np.float64))
    wa = np.abs(bf16_bits_to_f32(r.w_bits).astype(np.float64))
    env = x @ wa.T + (np.abs(b.astype(np.float64)) if b is not None else 0.0)
    H = r.x_bits.shape[1]
    bound = (H + 1) * 2.0 ** -23 * env
    err = np.abs(lg[rows].astype(np.float64) - want)
    assert np.all(err <= bound), float(np.max(err / bound))
    # the decision in the kernel's precision
    ids_o, w_o = oracle.route(lg, r.k)
    np.testing.assert_array_equal(ids, ids_o)
    np.testing.assert_allclose(w, w_o, rtol=1e-6, atol=1e-7)
    ids2, w2 = moe.moe_route(lg_d, r.k)
    assert torch.equal(ids2, ids_d) and torch.equal(w2.view(torch.int32), w_d.view(torch.int32))
    # clear decisions agree with the oracle's own logits
    srt = -np.sort(-want, axis=1)
    if r.k < want.shape[1]:
        clear = (srt[:, r.k - 1] - srt[:, r.k]) > 2 * bound.max(axis=1)
        ids_w, _ = oracle.route(want.astype(np.float32), r.k)
        np.testing.assert_array_equal(np.sort(ids[rows][clear], axis=1), np.sort(ids_w[clear], axis=1))
        if clear.size >= 32:
            assert clear.mean() > 0.5
    assert moe.moe_get_device_error() == 0


# the K loop is split over clusters of 1, 2, 4 or 8 CTAs depending on T and H (8 for
# few tiles and long K, 1 once the tiles fill the SMs: the last case); top-k lists of
# 4 (k <= 4) and 8
@pytest.mark.parametrize("T,H,E,k", [(1, 64, 4, 1), (37, 192, 32, 4), (130, 64, 7, 7), (300, 2880, 128, 4),
                                     (5, 128, 256, 8), (129, 2880, 200, 8), (256, 448, 64, 2),
                                     (18949, 256, 8, 2)])
def test_router_matches_oracle(moe_gpu, oracle_mod, T, H, E, k):
    _check(moe_gpu, oracle_mod, make_router(T, H, E, k, seed=T + E))


def test_router_without_bias(moe_gpu, oracle_mod):
    _check(moe_gpu, oracle_mod, make_router(70, 256, 32, 4, seed=3), bias=False)


@pytest.mark.parametrize("name,n_rows", [("router_20b_T4096", None), ("router_20b_T8", None),
                                         ("router_120b_T8192", 256)])
def test_router_full_size(moe_gpu, oracle_mod, name, n_rows):
    r = router_workload(name)
    T = r.x_bits.shape[0]
    rows = None
    if n_rows is not None:
        rng = np.random.default_rng(4)
        rows = np.sort(np.concatenate([[0, T - 1], rng.choice(np.arange(1, T - 1), n_rows - 2, replace=False)]))
    _check(moe_gpu, oracle_mod, r, rows=rows)


def test_router_ids_only_and_bad_sizes(moe_gpu, oracle_mod):
    import torch
    r = make_router(40, 128, 16, 2, seed=8)
    ids_a, w_a = _run(moe_gpu, r, want_logits=False)
    ids_b, w_b, _ = _run(moe_gpu, r, want_logits=True)
    assert torch.equal(ids_a, ids_b) and torch.equal(w_a, w_b)
    x = to_dev(make_router(4, 96, 8, 2).x_bits, torch.bfloat16)       # H % 64 != 0
    w = to_dev(make_router(4, 96, 8, 2).w_bits, torch.bfloat16)
    with pytest.raises(moe_gpu.MoEError) as ei:
        moe_gpu.moe_router_route(x, w, None, 2)
    assert ei.value.status == -1


def test_router_nan_logits_follow_the_routing_rule(moe_gpu):
    # a NaN router bias makes that expert's logit NaN for every token: it is never
    # chosen; with E = k + 1 and two NaN columns every token has one empty slot
    import torch
    r = make_router(40, 128, 5, 4, seed=3)
    x = to_dev(r.x_bits, torch.bfloat16)
    w = to_dev(r.w_bits, torch.bfloat16)
    b = r.bias.copy()
    b[[1, 3]] = np.nan
    moe_gpu.moe_get_device_error()
    ids, wt, lg = moe_gpu.moe_router_route(x, w, to_dev(b), r.k, want_logits=True)
    assert moe_gpu.moe_get_device_error() & moe_gpu.MOE_DEVERR_BAD_LOGIT
    ids, wt = ids.cpu().numpy(), wt.cpu().numpy()
    assert np.all(ids[:, 3] == -1) and np.all(wt[:, 3] == 0.0)
    assert not np.isin(ids[:, :3], [1, 3]).any()
    np.testing.assert_allclose(wt.astype(np.float64).sum(axis=1), 1.0, atol=1e-6)
    ids2, w2 = moe_gpu.moe_route(lg, r.k)
    assert torch.equal(ids2.cpu(), torch.from_numpy(ids)) and torch.equal(w2.cpu(), torch.from_numpy(wt))
    assert moe_gpu.moe_get_device_error() & moe_gpu.MOE_DEVERR_BAD_LOGIT   # read (and clear) the word
