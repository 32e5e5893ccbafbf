"""The C-ABI library: it builds, loads, exports every declared entry point, and its
host-side argument checks reject bad calls before touching a device.  No GPU."""
import ctypes
import os
import re
import subprocess

import pytest

import mxfp4_expert_ffn_moe_b200 as moe
from mxfp4_expert_ffn_moe_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_mxfp4.h")


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z][a-z0-9_]*)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_expected_calls():
    assert set(declared_functions()) == set(moe.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", moe.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in declared_functions():
        assert name in exported, name


def test_status_strings(lib):
    assert moe.moe_status_string(0) == "success"
    assert "invalid" in moe.moe_status_string(-1)
    assert moe.moe_status_string(12345) == "unknown status"


def test_workspace_size_host_logic(lib):
    s = moe.moe_mxfp4_workspace_size(4096, 2880, 2880, 32, 4)
    P = 4096 * 4
    assert s >= P * 2880 * 2 + P * 2880 * 2 + P * 2880 * 4
    assert s % 256 == 0
    assert moe.moe_mxfp4_workspace_size(0, 2880, 2880, 32, 4) == 0      # T < 1
    assert moe.moe_mxfp4_workspace_size(8, 2880, 2880, 4, 5) == 0       # k > E
    assert moe.moe_mxfp4_workspace_size(8, 100, 128, 4, 2) == 0         # H % 64
    assert moe.moe_mxfp4_workspace_size(8, 128, 128, 300, 2) == 0       # E > 256


def test_argument_checks_need_no_device(lib):
    # These fail in the host-side validation, before any CUDA call.
    p = ctypes.c_void_p(0x1000)          # never dereferenced
    null = None
    assert lib.mxfp4_dequantize(null, p, p, 1, 1, 32, null) == -1
    assert lib.mxfp4_dequantize(p, p, p, 1, 1, 48, null) == -1          # K % 32
    assert lib.mxfp4_dequantize(p, p, ctypes.c_void_p(0x1008), 1, 1, 32, null) == -1  # alignment
    assert lib.moe_route(p, 4, 8, 9, p, p, null) == -1                   # k > E
    assert lib.moe_route(p, 4, 300, 2, p, p, null) == -2                 # E > 256
    args = [p, 8, 128, 128, 4, 2, p, p, p, p, None, p, p, None, ctypes.c_float(1.702),
            ctypes.c_float(7.0), p]
    bad = list(args)
    bad[0] = None
    assert lib.moe_mxfp4_forward(*bad, null) == -1
    bad = list(args)
    bad[2] = 96                                                           # H % 64
    assert lib.moe_mxfp4_forward(*bad, null) == -1
    # router weight on the input with a bias present is refused
    bad = list(args)
    bad[10] = p
    assert lib.moe_mxfp4_forward_ex(*bad, ctypes.c_uint32(1), None, 0, null) == -1
    # unknown flag bits are refused
    assert lib.moe_mxfp4_forward_ex(*args, ctypes.c_uint32(6), None, 0, null) == -1
    # a caller workspace that is too small is refused before anything runs
    assert lib.moe_mxfp4_forward_ex(*args, ctypes.c_uint32(0), ctypes.c_void_p(0x100000), 64,
                                    null) == -4


def test_profiler_stage_mask_host_logic(lib):
    # host-side state only: no event is recorded while no launch happens
    assert lib.moe_profile_enable_stages(ctypes.c_uint32(1 << 7)) == -1        # past the stages
    assert lib.moe_profile_enable_stages(ctypes.c_uint32(1 << 3)) == 0         # gate_up only
    moe.moe_profile_enable_stages(["gate_up", "down"])
    moe.moe_profile_enable_stages([])
    moe.moe_profile_enable(False)
    ms = (ctypes.c_double * 7)()
    launches = (ctypes.c_int64 * 7)()
    assert lib.moe_profile_read(ms, launches) == 0
    with pytest.raises(ValueError):
        moe.moe_profile_enable_stages(["no_such_stage"])


def test_nvfp4_router_and_host_copy_argument_checks_need_no_device(lib):
    # The NVFP4, router and host-copy entry points reject bad calls in the host-side
    # validation, before any CUDA call.
    p = ctypes.c_void_p(0x1000)          # never dereferenced
    null = None
    # nvfp4_dequantize
    assert lib.nvfp4_dequantize(null, p, null, p, 1, 1, 16, null) == -1
    assert lib.nvfp4_dequantize(p, p, null, p, 1, 1, 24, null) == -1                    # K % 16
    assert lib.nvfp4_dequantize(p, p, ctypes.c_void_p(0x1002), p, 1, 1, 16, null) == -1  # scale2 alignment
    # moe_nvfp4_forward_ex: x, T, H, I, E, k, ids, w, gu blocks/scales/scale2/bias, d blocks/scales/scale2/bias
    args = [p, 8, 128, 128, 4, 2, p, p, p, p, None, None, p, p, None, None, ctypes.c_float(1.702),
            ctypes.c_float(7.0), p, ctypes.c_uint32(0), None, 0, null]
    bad = list(args)
    bad[0] = None
    assert lib.moe_nvfp4_forward_ex(*bad) == -1
    bad = list(args)
    bad[2] = 96                                                                             # H % 64
    assert lib.moe_nvfp4_forward_ex(*bad) == -1
    bad = list(args)
    bad[11], bad[19] = p, ctypes.c_uint32(1)                         # weight on input with a bias
    assert lib.moe_nvfp4_forward_ex(*bad) == -1
    bad = list(args)
    bad[10] = ctypes.c_void_p(0x1002)                                                       # scale2 alignment
    assert lib.moe_nvfp4_forward_ex(*bad) == -1
    bad = list(args)
    bad[20], bad[21] = ctypes.c_void_p(0x100000), 64                                        # workspace too small
    assert lib.moe_nvfp4_forward_ex(*bad) == -4
    # moe_router_route: x, w, b, T, H, E, k, logits, ids, weights
    assert lib.moe_router_route(null, p, null, 8, 128, 32, 4, null, p, p, null) == -1
    assert lib.moe_router_route(p, p, null, 8, 96, 32, 4, null, p, p, null) == -1          # H % 64
    assert lib.moe_router_route(p, p, null, 8, 128, 4, 5, null, p, p, null) == -1          # k > E
    assert lib.moe_router_route(p, p, null, 8, 128, 300, 4, null, p, p, null) == -2        # E > 256
    assert lib.moe_router_route(ctypes.c_void_p(0x1008), p, null, 8, 128, 32, 4, null, p, p, null) == -1
    # *_dequantize_from_host: sizes are checked before the host pointers are looked at
    assert lib.mxfp4_dequantize_from_host(p, p, p, 1, 1, 48, null) == -1                  # K % 32
    assert lib.mxfp4_dequantize_from_host(null, p, p, 1, 1, 32, null) == -1
    assert lib.nvfp4_dequantize_from_host(p, p, null, p, 1, 1, 24, null) == -1            # K % 16
    assert lib.nvfp4_dequantize_from_host(p, null, null, p, 1, 1, 16, null) == -1


@pytest.mark.parametrize("env,T,want", [(None, 1, 32), (None, 4096, 256), ("0", 1, 256), ("2000", 4096, 32),
                                        ("junk", 1, 32), ("-5", 4096, 256)])
def test_decode_switch_environment_override(env, T, want):
    # MOE_DECODE_MAX_TOKENS_PER_EXPERT moves the decode/prefill tile switch (read once
    # per process, so each case runs in a fresh interpreter); host-only, no device
    import subprocess
    import sys
    code = ("import sys; sys.path.insert(0, %r); import mxfp4_expert_ffn_moe_b200 as m; "
            "print(m.moe_token_tile_rows(%d, 2880, 2880, 32, 4))" % (ROOT, T))
    e = dict(os.environ)
    e.pop("MOE_DECODE_MAX_TOKENS_PER_EXPERT", None)
    if env is not None:
        e["MOE_DECODE_MAX_TOKENS_PER_EXPERT"] = env
    r = subprocess.run([sys.executable, "-c", code], env=e, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr[-400:]
    assert int(r.stdout.strip().splitlines()[-1]) == want
