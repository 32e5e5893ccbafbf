"""Dequant-on-copy from host memory on the GPU: the packed bank stays in page-locked
host memory and the decode kernel reads it through its device mapping.  The result
must be bit for bit the oracle's (and the device-memory call's); host memory the
device cannot address is refused before anything runs."""
import numpy as np
import pytest

from mxfp4_expert_ffn_moe_b200.workloads import make_bank, make_dequant_bank, make_nvfp4_dequant_bank
from tests.gpu_util import bits_of, to_dev

pytestmark = pytest.mark.gpu


def _pinned(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).pin_memory()


@pytest.mark.parametrize("E,N,K", [(1, 1, 32), (3, 5, 96), (4, 129, 160)])
def test_mxfp4_from_host_matches_oracle(moe_gpu, oracle_mod, E, N, K):
    import torch
    rng = np.random.default_rng(E * 31 + N)
    bank = make_bank(rng, E, N, K, 0, 254)
    out = moe_gpu.mxfp4_dequantize_from_host(_pinned(bank.blocks), _pinned(bank.scales))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bits_of(out), oracle_mod.dequantize(bank.blocks, bank.scales, E, N, K))
    assert moe_gpu.moe_get_device_error() == 0


@pytest.mark.parametrize("E,N,K", [(1, 1, 16), (3, 5, 96), (70, 3, 48)])
def test_nvfp4_from_host_matches_oracle(moe_gpu, oracle_mod, E, N, K):
    import torch
    rng = np.random.default_rng(E * 37 + N)
    blocks = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    scales = rng.integers(0, 0x7F, size=(E, N, K // 16), dtype=np.uint8)
    s2 = rng.uniform(0.25, 2.0, size=E).astype(np.float32)
    out = moe_gpu.nvfp4_dequantize_from_host(_pinned(blocks), _pinned(scales), to_dev(s2))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bits_of(out), oracle_mod.nvfp4_dequantize(blocks, scales, s2, E, N, K))
    assert moe_gpu.moe_get_device_error() == 0


def test_full_20b_down_bank_from_host_equals_device_path(moe_gpu, oracle_mod):
    # the gpt-oss-20b down bank [32, 2880, 2880] from host memory: identical bits to
    # the device-memory call, and every element bit-exact against the oracle
    import torch
    _, dn = make_dequant_bank(seed=0)
    E, N, K = dn.shape
    host_out = moe_gpu.mxfp4_dequantize_from_host(_pinned(dn.blocks), _pinned(dn.scales))
    dev_out = moe_gpu.mxfp4_dequantize(to_dev(dn.blocks), to_dev(dn.scales))
    torch.cuda.synchronize()
    assert torch.equal(host_out.view(torch.int16), dev_out.view(torch.int16))
    del dev_out
    got = bits_of(host_out)
    del host_out
    want = oracle_mod.dequantize(dn.blocks, dn.scales, E, N, K)
    assert np.array_equal(got, want), f"{int(np.count_nonzero(got != want))} elements differ"
    del got, want
    gu, _ = make_nvfp4_dequant_bank(seed=1, E=4)
    E, N, K = gu.shape
    s2 = to_dev(gu.scale2)
    a = moe_gpu.nvfp4_dequantize_from_host(_pinned(gu.blocks), _pinned(gu.scales), s2)
    b = moe_gpu.nvfp4_dequantize(to_dev(gu.blocks), to_dev(gu.scales), s2)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert moe_gpu.moe_get_device_error() == 0


def test_memory_the_device_cannot_address_is_refused(moe_gpu):
    import ctypes

    import torch
    bank = make_bank(np.random.default_rng(0), 2, 4, 64, 100, 130)
    out = torch.empty((2, 4, 64), dtype=torch.bfloat16, device="cuda")
    lib = moe_gpu.load_library()
    # pageable (not page-locked) host memory
    hb = np.ascontiguousarray(bank.blocks)
    hs = np.ascontiguousarray(bank.scales)
    rc = lib.mxfp4_dequantize_from_host(ctypes.c_void_p(hb.ctypes.data), ctypes.c_void_p(hs.ctypes.data),
                                        ctypes.c_void_p(out.data_ptr()), 2, 4, 64, None)
    assert rc == -1
    # device memory passed where host memory is expected
    db, ds = to_dev(bank.blocks), to_dev(bank.scales)
    rc = lib.mxfp4_dequantize_from_host(ctypes.c_void_p(db.data_ptr()), ctypes.c_void_p(ds.data_ptr()),
                                        ctypes.c_void_p(out.data_ptr()), 2, 4, 64, None)
    assert rc == -1
    torch.cuda.synchronize()
    assert moe_gpu.moe_get_device_error() == 0
