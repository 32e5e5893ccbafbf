"""moe_permute on the GPU: the grouping of (token, slot) pairs by expert, checked
exactly against a numpy restatement of its definition.

Pair p = t*k + j goes to expert ids[p]; counts are the per-expert histogram,
offsets and tile_offsets its exclusive scans (the latter over whole token tiles),
sorted_pairs lists every valid pair once in expert order with ascending p inside
an expert (a stable order, FreeToken PR #838's expert-ordered views), pair_rows
is its inverse.  Integer bookkeeping: bit-exact, no tolerance.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _expected(ids, E, tile_rows):
    flat = ids.reshape(-1).astype(np.int64)
    valid = (flat >= 0) & (flat < E)
    counts = np.bincount(flat[valid], minlength=E).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    tiles = (counts + tile_rows - 1) // tile_rows
    tile_offsets = np.concatenate([[0], np.cumsum(tiles)])
    p = np.nonzero(valid)[0]
    order = p[np.argsort(flat[p], kind="stable")]      # expert order, ascending p inside
    return counts, offsets, tile_offsets, order


def _run(moe, ids_np, E, tile_rows):
    import torch
    ids = torch.from_numpy(ids_np.astype(np.int32)).cuda()
    res = moe.moe_permute(ids, E, tile_rows)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy().astype(np.int64) for k, v in res.items()}


def _check(moe, ids_np, E, tile_rows):
    counts, offsets, tile_offsets, order = _expected(ids_np, E, tile_rows)
    got = _run(moe, ids_np, E, tile_rows)
    np.testing.assert_array_equal(got["counts"], counts)
    np.testing.assert_array_equal(got["offsets"], offsets)
    np.testing.assert_array_equal(got["tile_offsets"], tile_offsets)
    rows = int(offsets[-1])
    sp = got["sorted_pairs"][:rows]
    np.testing.assert_array_equal(sp, order)
    # bijection between the valid pairs and the rows, and the inverse map
    P = ids_np.size
    inv = got["pair_rows"]
    flat = ids_np.reshape(-1)
    valid = (flat >= 0) & (flat < E)
    assert np.all(inv[~valid] == -1)
    np.testing.assert_array_equal(sp[inv[valid]], np.nonzero(valid)[0])
    assert np.unique(inv[valid]).size == int(valid.sum()) == rows
    assert P >= rows


@pytest.mark.parametrize("T,k,E,tile_rows", [
    (1, 1, 1, 32),          # a single pair
    (3, 2, 5, 32),          # most experts empty
    (37, 3, 7, 32),         # ragged tails
    (4096, 4, 32, 256),     # the gpt-oss-20b prefill layer's shape
    (2048, 8, 256, 32),     # largest E and k
    (15000, 4, 64, 256),    # 60,000 pairs: 30 CTAs, each placing its own range
    (40000, 4, 128, 256),   # 160,000 pairs: the 64-CTA cap, sub-chunks of 79 pairs
])
def test_permute_uniform_ids(moe_gpu, T, k, E, tile_rows):
    rng = np.random.default_rng(T * 7 + E)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)])   # k distinct experts per token
    _check(moe_gpu, ids, E, tile_rows)
    assert moe_gpu.moe_get_device_error() == 0


def test_permute_skewed_ids(moe_gpu):
    # one hot expert takes most pairs (the Zipf-skewed gpt-oss-120b layer's pattern),
    # several experts stay empty
    rng = np.random.default_rng(11)
    T, k, E = 8192, 4, 128
    hot = rng.random((T, k)) < 0.8
    ids = np.where(hot, 0, rng.integers(1, E // 2, size=(T, k))).astype(np.int32)
    _check(moe_gpu, ids, E, 256)
    assert moe_gpu.moe_get_device_error() == 0


def test_permute_drops_out_of_range_ids(moe_gpu):
    rng = np.random.default_rng(3)
    T, k, E = 300, 4, 16
    ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
    ids[5, 1] = -1
    ids[17, 3] = E
    ids[200, 0] = 1 << 30
    _check(moe_gpu, ids, E, 32)
    assert moe_gpu.moe_get_device_error() & moe_gpu.MOE_DEVERR_BAD_EXPERT_ID


def test_permute_is_deterministic_with_repeated_experts(moe_gpu):
    # every pair on the same expert: the stable order is the identity
    T, k, E = 5000, 2, 4
    ids = np.full((T, k), 2, np.int32)
    got = _run(moe_gpu, ids, E, 32)
    np.testing.assert_array_equal(got["sorted_pairs"], np.arange(T * k))
    np.testing.assert_array_equal(got["pair_rows"], np.arange(T * k))
    assert moe_gpu.moe_get_device_error() == 0
