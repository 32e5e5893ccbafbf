"""mxfp4_dequantize on the GPU against the CPU oracle: bit-exact (rel-err 0.0)."""
import numpy as np
import pytest

from mxfp4_expert_ffn_moe_b200.workloads import make_bank, make_dequant_bank
from tests.gpu_util import bits_of, to_dev

pytestmark = pytest.mark.gpu


def _gpu_dequant(moe, blocks, scales):
    import torch
    out = moe.mxfp4_dequantize(to_dev(blocks), to_dev(scales))
    torch.cuda.synchronize()
    return bits_of(out)


def test_every_code_and_every_scale_byte(moe_gpu, oracle_mod):
    # 256 rows, row n uses scale byte n in every block: all E8M0 bytes including
    # the subnormal (0, 1), overflow (253, 254) and invalid (255) ones.
    E, N, K = 1, 256, 64
    rng = np.random.default_rng(0)
    blocks = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    blocks[0, :, 0] = 0x10      # codes 0 and 1
    blocks[0, :, 1:9] = np.array([0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE, 0xE1], np.uint8)
    scales = np.repeat(np.arange(256, dtype=np.uint8)[None, :, None], K // 32, axis=2)
    got = _gpu_dequant(moe_gpu, blocks, scales)
    want = oracle_mod.dequantize(blocks, scales, E, N, K)
    np.testing.assert_array_equal(got, want)
    assert moe_gpu.moe_get_device_error() & moe_gpu.MOE_DEVERR_BAD_SCALE
    assert moe_gpu.moe_get_device_error() == 0   # the read cleared it


@pytest.mark.parametrize("E,N,K", [(1, 1, 32), (3, 5, 96), (2, 7, 2880), (4, 129, 160)])
def test_ragged_shapes(moe_gpu, oracle_mod, E, N, K):
    rng = np.random.default_rng(E * 1000 + N)
    bank = make_bank(rng, E, N, K, 0, 254)
    got = _gpu_dequant(moe_gpu, bank.blocks, bank.scales)
    np.testing.assert_array_equal(got, oracle_mod.dequantize(bank.blocks, bank.scales, E, N, K))
    assert moe_gpu.moe_get_device_error() == 0


def test_full_gpt_oss_20b_bank_bit_exact(moe_gpu, oracle_mod):
    # The standalone dequant workload at full size: gate_up [32, 5760, 2880] and
    # down [32, 2880, 2880], scale bytes in [110, 130]; every element of both banks
    # is compared with the oracle bit for bit.
    import torch
    gu, dn = make_dequant_bank(seed=0)
    for bank in (gu, dn):
        E, N, K = bank.shape
        out = moe_gpu.mxfp4_dequantize(to_dev(bank.blocks), to_dev(bank.scales))
        torch.cuda.synchronize()
        got = bits_of(out)
        del out
        want = oracle_mod.dequantize(bank.blocks, bank.scales, E, N, K)
        assert np.array_equal(got, want), f"{int(np.count_nonzero(got != want))} elements differ"
        del got, want
    assert moe_gpu.moe_get_device_error() == 0
