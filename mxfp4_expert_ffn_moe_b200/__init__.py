"""B200-native MXFP4 expert-FFN MoE layer: thin Python binding of the C ABI.

The functions below carry the same names as the C entry points declared in
``include/moe_mxfp4.h`` and only marshal arguments: shapes and raw device pointers
from torch tensors, the current CUDA stream, and the status code back as an
exception.  Every step of the layer runs in the CUDA kernels of
``libmoe_mxfp4.so``; there is no CPU fallback, and calling any function without the
built library raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "MoEError", "load_library", "library_path", "mxfp4_dequantize", "moe_route",
    "moe_mxfp4_forward", "moe_mxfp4_forward_ex", "moe_mxfp4_workspace_size",
    "moe_status_string", "moe_get_device_error", "MOE_FLAG_WEIGHT_ON_INPUT",
    "MOE_DEVERR_BAD_EXPERT_ID", "MOE_DEVERR_BAD_SCALE", "MOE_DEVERR_TIMEOUT",
    "EXPORTED_SYMBOLS", "PROFILE_STAGES", "moe_profile_enable", "moe_profile_enable_stages",
    "moe_profile_read",
    "moe_mxfp4_forward_noalloc", "MOE_NOALLOC_SCRATCH_BYTES",
    "nvfp4_dequantize", "moe_nvfp4_forward_ex", "moe_router_route",
    "mxfp4_dequantize_from_host", "nvfp4_dequantize_from_host", "moe_permute", "moe_token_tile_rows",
    "MOE_DEVERR_BAD_LOGIT", "MOE_DEVERR_OUT_OF_BOUNDS", "use_checked_library", "moe_gather_pairs", "moe_mxfp4_expert_rows",
    "moe_combine_pairs",
]

MOE_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024

MOE_FLAG_WEIGHT_ON_INPUT = 0x1
MOE_DEVERR_BAD_EXPERT_ID = 0x1
MOE_DEVERR_BAD_SCALE = 0x2
MOE_DEVERR_TIMEOUT = 0x4
MOE_DEVERR_BAD_LOGIT = 0x8
MOE_DEVERR_OUT_OF_BOUNDS = 0x10

EXPORTED_SYMBOLS = (
    "mxfp4_dequantize", "moe_route", "moe_mxfp4_forward", "moe_mxfp4_forward_ex",
    "moe_mxfp4_workspace_size", "moe_status_string", "moe_get_device_error",
    "moe_profile_enable", "moe_profile_enable_stages", "moe_profile_read", "moe_mxfp4_forward_noalloc",
    "nvfp4_dequantize", "moe_nvfp4_forward_ex", "moe_router_route",
    "mxfp4_dequantize_from_host", "nvfp4_dequantize_from_host", "moe_permute", "moe_token_tile_rows",
    "moe_gather_pairs", "moe_mxfp4_expert_rows", "moe_combine_pairs",
)
PROFILE_STAGES = ("route", "permute", "gather", "gate_up", "down", "combine", "dequant")

_PKG = os.path.dirname(os.path.abspath(__file__))
_lib = None
_libs = {}
_use_checked = False


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {moe_status_string(status)} ({status})")
        self.status = status


def library_path(checked: bool = False) -> str:
    return os.path.join(_PKG, "libmoe_mxfp4_checked.so" if checked else "libmoe_mxfp4.so")


def use_checked_library(on: bool) -> bool:
    """Route every call of this binding to the bounds-checked build of the library
    (built by build.build(checked=True); each data-dependent global index is tested
    and MOE_DEVERR_OUT_OF_BOUNDS raised instead of an access outside a buffer), or
    back to the normal build.  Returns the previous setting."""
    global _use_checked, _lib
    prev = _use_checked
    _use_checked = bool(on)
    _lib = None
    return prev


def load_library():
    """Load the in-tree CUDA library (the variant use_checked_library selects); raise if
    it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path(_use_checked)
    if path in _libs:
        _lib = _libs[path]
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} (run __graft_entry__.build())")
    lib = ctypes.CDLL(path)
    p, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    lib.mxfp4_dequantize.argtypes = [p, p, p, i64, i64, i64, p]
    lib.mxfp4_dequantize.restype = i32
    lib.moe_route.argtypes = [p, i64, i64, i32, p, p, p]
    lib.moe_route.restype = i32
    fwd = [p, i64, i64, i64, i64, i32, p, p, p, p, p, p, p, p, f32, f32, p]
    lib.moe_mxfp4_forward.argtypes = fwd + [p]
    lib.moe_mxfp4_forward.restype = i32
    lib.moe_mxfp4_forward_ex.argtypes = fwd + [ctypes.c_uint32, p, ctypes.c_size_t, p]
    lib.moe_mxfp4_forward_ex.restype = i32
    lib.moe_mxfp4_workspace_size.argtypes = [i64, i64, i64, i64, i32]
    lib.moe_mxfp4_workspace_size.restype = ctypes.c_size_t
    lib.moe_status_string.argtypes = [i32]
    lib.moe_status_string.restype = ctypes.c_char_p
    lib.moe_get_device_error.argtypes = [p]
    lib.moe_get_device_error.restype = i32
    lib.moe_mxfp4_forward_noalloc.argtypes = fwd + [ctypes.c_uint32, p]
    lib.moe_mxfp4_forward_noalloc.restype = i32
    lib.moe_profile_enable.argtypes = [i32]
    lib.moe_profile_enable.restype = i32
    lib.moe_profile_enable_stages.argtypes = [ctypes.c_uint32]
    lib.moe_profile_enable_stages.restype = i32
    lib.moe_router_route.argtypes = [p, p, p, i64, i64, i64, i32, p, p, p, p]
    lib.moe_router_route.restype = i32
    lib.mxfp4_dequantize_from_host.argtypes = [p, p, p, i64, i64, i64, p]
    lib.mxfp4_dequantize_from_host.restype = i32
    lib.nvfp4_dequantize_from_host.argtypes = [p, p, p, p, i64, i64, i64, p]
    lib.nvfp4_dequantize_from_host.restype = i32
    lib.nvfp4_dequantize.argtypes = [p, p, p, p, i64, i64, i64, p]
    lib.nvfp4_dequantize.restype = i32
    nv_fwd = [p, i64, i64, i64, i64, i32, p, p, p, p, p, p, p, p, p, p, ctypes.c_float,
              ctypes.c_float, p, ctypes.c_uint32, p, ctypes.c_size_t, p]
    lib.moe_nvfp4_forward_ex.argtypes = nv_fwd
    lib.moe_nvfp4_forward_ex.restype = i32
    lib.moe_permute.argtypes = [p, i64, i32, i64, i32, p, p, p, p, p, p]
    lib.moe_permute.restype = i32
    lib.moe_token_tile_rows.argtypes = [i64, i64, i64, i64, i32, i32]
    lib.moe_token_tile_rows.restype = i32
    lib.moe_gather_pairs.argtypes = [p, i64, i64, i32, p, p, p, p, i64, p, p, p, p]
    lib.moe_gather_pairs.restype = i32
    lib.moe_mxfp4_expert_rows.argtypes = [p, i64, i64, i64, i64, i64, p, p, p, p, p, p, p, p, f32, f32, p,
                                          ctypes.c_uint32, p, ctypes.c_size_t, p]
    lib.moe_mxfp4_expert_rows.restype = i32
    lib.moe_combine_pairs.argtypes = [p, p, i64, i32, i64, p, p]
    lib.moe_combine_pairs.restype = i32
    lib.moe_profile_read.argtypes = [p, p]
    lib.moe_profile_read.restype = i32
    _libs[path] = lib
    _lib = lib
    return lib


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t, dtype, name):
    import torch
    if t is None:
        return None
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor, got {t.dtype} "
                         f"on {t.device} (contiguous={t.is_contiguous()})")
    return ctypes.c_void_p(t.data_ptr())


def _check(fn, rc):
    if rc != 0:
        raise MoEError(fn, rc)


def moe_status_string(status: int) -> str:
    return load_library().moe_status_string(int(status)).decode()


def mxfp4_dequantize(blocks, scales, out=None, stream=None):
    """Packed [E, N, K/2] uint8 + E8M0 [E, N, K/32] uint8 -> bf16 [E, N, K]."""
    import torch
    E, N, Kh = blocks.shape
    K = 2 * Kh
    if out is None:
        out = torch.empty((E, N, K), dtype=torch.bfloat16, device=blocks.device)
    rc = load_library().mxfp4_dequantize(_dev(blocks, torch.uint8, "blocks"),
                                         _dev(scales, torch.uint8, "scales"),
                                         _dev(out, torch.bfloat16, "out"), E, N, K, _stream(stream))
    _check("mxfp4_dequantize", rc)
    return out


def _host(t, dtype, name):
    if not (t.device.type == "cpu" and t.dtype == dtype and t.is_contiguous() and t.is_pinned()):
        raise ValueError(f"{name}: expected a contiguous page-locked CPU {dtype} tensor")
    return ctypes.c_void_p(t.data_ptr())


def mxfp4_dequantize_from_host(blocks, scales, out=None, device=None, stream=None):
    """Dequant-on-copy: packed [E, N, K/2] + E8M0 [E, N, K/32] in pinned host memory ->
    bf16 [E, N, K] on the device (the kernel reads the host bank through its mapping)."""
    import torch
    E, N, Kh = blocks.shape
    K = 2 * Kh
    if out is None:
        out = torch.empty((E, N, K), dtype=torch.bfloat16, device=device or "cuda")
    rc = load_library().mxfp4_dequantize_from_host(_host(blocks, torch.uint8, "blocks"),
                                                   _host(scales, torch.uint8, "scales"),
                                                   _dev(out, torch.bfloat16, "out"), E, N, K, _stream(stream))
    _check("mxfp4_dequantize_from_host", rc)
    return out


def nvfp4_dequantize_from_host(blocks, scales, scale2=None, out=None, device=None, stream=None):
    """Dequant-on-copy of an NVFP4 bank in pinned host memory (E4M3 [E, N, K/16]);
    scale2 is a device fp32 [E] tensor or None."""
    import torch
    E, N, Kh = blocks.shape
    K = 2 * Kh
    if out is None:
        out = torch.empty((E, N, K), dtype=torch.bfloat16, device=device or "cuda")
    rc = load_library().nvfp4_dequantize_from_host(_host(blocks, torch.uint8, "blocks"),
                                                   _host(scales, torch.uint8, "scales"),
                                                   _dev(scale2, torch.float32, "scale2"),
                                                   _dev(out, torch.bfloat16, "out"), E, N, K, _stream(stream))
    _check("nvfp4_dequantize_from_host", rc)
    return out


def moe_route(router_logits, k: int, ids=None, weights=None, stream=None):
    """fp32 logits [T, E] -> (int32 ids [T, k], fp32 weights [T, k])."""
    import torch
    T, E = router_logits.shape
    if ids is None:
        ids = torch.empty((T, k), dtype=torch.int32, device=router_logits.device)
    if weights is None:
        weights = torch.empty((T, k), dtype=torch.float32, device=router_logits.device)
    rc = load_library().moe_route(_dev(router_logits, torch.float32, "router_logits"), T, E, int(k),
                                  _dev(ids, torch.int32, "ids"), _dev(weights, torch.float32, "weights"),
                                  _stream(stream))
    _check("moe_route", rc)
    return ids, weights


def moe_router_route(x, w_router, b_router, k: int, want_logits: bool = False, ids=None,
                     weights=None, logits=None, stream=None):
    """Router linear layer + routing: bf16 x [T, H], bf16 w_router [E, H], fp32 b_router
    [E] or None -> (int32 ids [T, k], fp32 weights [T, k]) and, with want_logits (or a
    logits tensor given), the fp32 logits [T, E] the routing used."""
    import torch
    T, H = x.shape
    E = w_router.shape[0]
    if ids is None:
        ids = torch.empty((T, k), dtype=torch.int32, device=x.device)
    if weights is None:
        weights = torch.empty((T, k), dtype=torch.float32, device=x.device)
    if logits is None and want_logits:
        logits = torch.empty((T, E), dtype=torch.float32, device=x.device)
    rc = load_library().moe_router_route(
        _dev(x, torch.bfloat16, "x"), _dev(w_router, torch.bfloat16, "w_router"),
        _dev(b_router, torch.float32, "b_router"), T, H, E, int(k), _dev(logits, torch.float32, "logits"),
        _dev(ids, torch.int32, "ids"), _dev(weights, torch.float32, "weights"), _stream(stream))
    _check("moe_router_route", rc)
    return (ids, weights, logits) if logits is not None else (ids, weights)


def _fwd_args(x, ids, weights, gate_up_blocks, gate_up_scales, gate_up_bias, down_blocks,
              down_scales, down_bias, alpha, limit, out):
    import torch
    T, H = x.shape
    k = ids.shape[1]
    E, N2, _ = gate_up_blocks.shape
    I = N2 // 2
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    args = [_dev(x, torch.bfloat16, "x"), T, H, I, E, k, _dev(ids, torch.int32, "ids"),
            _dev(weights, torch.float32, "weights"), _dev(gate_up_blocks, torch.uint8, "gate_up_blocks"),
            _dev(gate_up_scales, torch.uint8, "gate_up_scales"),
            _dev(gate_up_bias, torch.float32, "gate_up_bias"), _dev(down_blocks, torch.uint8, "down_blocks"),
            _dev(down_scales, torch.uint8, "down_scales"), _dev(down_bias, torch.float32, "down_bias"),
            float(alpha), float(limit), _dev(out, torch.bfloat16, "out")]
    return args, out


def moe_mxfp4_forward(x, ids, weights, gate_up_blocks, gate_up_scales, gate_up_bias, down_blocks,
                      down_scales, down_bias, alpha: float = 1.702, limit: float = 7.0, out=None,
                      stream=None):
    args, out = _fwd_args(x, ids, weights, gate_up_blocks, gate_up_scales, gate_up_bias,
                          down_blocks, down_scales, down_bias, alpha, limit, out)
    _check("moe_mxfp4_forward", load_library().moe_mxfp4_forward(*args, _stream(stream)))
    return out


def moe_mxfp4_forward_ex(x, ids, weights, gate_up_blocks, gate_up_scales, gate_up_bias,
                         down_blocks, down_scales, down_bias, alpha: float = 1.702,
                         limit: float = 7.0, out=None, flags: int = 0, workspace=None,
                         stream=None):
    import torch
    args, out = _fwd_args(x, ids, weights, gate_up_blocks, gate_up_scales, gate_up_bias,
                          down_blocks, down_scales, down_bias, alpha, limit, out)
    ws = _dev(workspace, torch.uint8, "workspace")
    nbytes = 0 if workspace is None else workspace.numel()
    rc = load_library().moe_mxfp4_forward_ex(*args, ctypes.c_uint32(flags), ws, nbytes, _stream(stream))
    _check("moe_mxfp4_forward_ex", rc)
    return out


def moe_mxfp4_forward_noalloc(x, ids, weights, gate_up_blocks, gate_up_scales, gate_up_bias,
                              down_blocks, down_scales, down_bias, alpha: float = 1.702,
                              limit: float = 7.0, out=None, flags: int = 0, stream=None):
    """The layer for callers that cannot allocate device memory: the library's
    static scratch array stands in for the workspace (see the C header for the
    size limit, the first-call set-up and the sharing rules)."""
    args, out = _fwd_args(x, ids, weights, gate_up_blocks, gate_up_scales, gate_up_bias,
                          down_blocks, down_scales, down_bias, alpha, limit, out)
    rc = load_library().moe_mxfp4_forward_noalloc(*args, ctypes.c_uint32(flags), _stream(stream))
    _check("moe_mxfp4_forward_noalloc", rc)
    return out


def nvfp4_dequantize(blocks, scales, scale2=None, out=None, stream=None):
    """Packed [E, N, K/2] uint8 + E4M3 [E, N, K/16] uint8 (+ fp32 weight_scale_2 [E])
    -> bf16 [E, N, K]."""
    import torch
    E, N, Kh = blocks.shape
    K = 2 * Kh
    if out is None:
        out = torch.empty((E, N, K), dtype=torch.bfloat16, device=blocks.device)
    rc = load_library().nvfp4_dequantize(_dev(blocks, torch.uint8, "blocks"),
                                         _dev(scales, torch.uint8, "scales"),
                                         _dev(scale2, torch.float32, "scale2"),
                                         _dev(out, torch.bfloat16, "out"), E, N, K, _stream(stream))
    _check("nvfp4_dequantize", rc)
    return out


def moe_nvfp4_forward_ex(x, ids, weights, gate_up_blocks, gate_up_scales, gate_up_scale2,
                         gate_up_bias, down_blocks, down_scales, down_scale2, down_bias,
                         alpha: float = 1.702, limit: float = 7.0, out=None, flags: int = 0,
                         workspace=None, stream=None):
    """The layer over NVFP4 banks: E4M3 scales [E, 2I, H/16] / [E, H, I/16] and fp32
    weight_scale_2 [E, 2] (gate, up) / [E], each may be None (= 1)."""
    import torch
    T, H = x.shape
    k = ids.shape[1]
    E, N2, _ = gate_up_blocks.shape
    I = N2 // 2
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    ws = _dev(workspace, torch.uint8, "workspace")
    nbytes = 0 if workspace is None else workspace.numel()
    rc = load_library().moe_nvfp4_forward_ex(
        _dev(x, torch.bfloat16, "x"), T, H, I, E, k, _dev(ids, torch.int32, "ids"),
        _dev(weights, torch.float32, "weights"), _dev(gate_up_blocks, torch.uint8, "gate_up_blocks"),
        _dev(gate_up_scales, torch.uint8, "gate_up_scales"),
        _dev(gate_up_scale2, torch.float32, "gate_up_scale2"),
        _dev(gate_up_bias, torch.float32, "gate_up_bias"), _dev(down_blocks, torch.uint8, "down_blocks"),
        _dev(down_scales, torch.uint8, "down_scales"), _dev(down_scale2, torch.float32, "down_scale2"),
        _dev(down_bias, torch.float32, "down_bias"), float(alpha), float(limit),
        _dev(out, torch.bfloat16, "out"), ctypes.c_uint32(flags), ws, nbytes, _stream(stream))
    _check("moe_nvfp4_forward_ex", rc)
    return out


def moe_permute(ids, E: int, tile_rows: int, want_pair_rows: bool = True, stream=None):
    """Group the (token, slot) pairs of int32 ids [T, k] by expert.  Returns a dict of
    int32 device tensors: counts [E], offsets [E + 1], tile_offsets [E + 1],
    sorted_pairs [T*k] and (with want_pair_rows) pair_rows [T*k]."""
    import torch
    T, k = ids.shape
    dev = ids.device
    out = {"counts": torch.empty(E, dtype=torch.int32, device=dev),
           "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
           "tile_offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
           "sorted_pairs": torch.empty(T * k, dtype=torch.int32, device=dev)}
    if want_pair_rows:
        out["pair_rows"] = torch.empty(T * k, dtype=torch.int32, device=dev)
    rc = load_library().moe_permute(
        _dev(ids, torch.int32, "ids"), T, int(k), int(E), int(tile_rows),
        *[_dev(out[n], torch.int32, n) for n in ("counts", "offsets", "tile_offsets", "sorted_pairs")],
        _dev(out.get("pair_rows"), torch.int32, "pair_rows"), _stream(stream))
    _check("moe_permute", rc)
    return out


def moe_gather_pairs(x, ids, weights, perm, E: int, stream=None):
    """Rows of x in the expert order of `perm` (moe_permute's dict), with their expert
    ids and routing weights: (bf16 [T*k, H], int32 [T*k], fp32 [T*k]); only the first
    perm["offsets"][E] rows are written."""
    import torch
    T, H = x.shape
    k = ids.shape[1]
    x_rows = torch.empty((T * k, H), dtype=torch.bfloat16, device=x.device)
    row_ids = torch.empty(T * k, dtype=torch.int32, device=x.device)
    row_w = torch.empty(T * k, dtype=torch.float32, device=x.device)
    rc = load_library().moe_gather_pairs(
        _dev(x, torch.bfloat16, "x"), T, H, int(k), _dev(ids, torch.int32, "ids"),
        _dev(weights, torch.float32, "weights"), _dev(perm["sorted_pairs"], torch.int32, "sorted_pairs"),
        _dev(perm["offsets"], torch.int32, "offsets"), int(E), _dev(x_rows, torch.bfloat16, "x_rows"),
        _dev(row_ids, torch.int32, "row_ids"), _dev(row_w, torch.float32, "row_weights"), _stream(stream))
    _check("moe_gather_pairs", rc)
    return x_rows, row_ids, row_w


def moe_mxfp4_expert_rows(x_rows, row_ids, row_weights, expert_base: int, gate_up_blocks, gate_up_scales,
                          gate_up_bias, down_blocks, down_scales, down_bias, alpha: float = 1.702,
                          limit: float = 7.0, flags: int = 0, y_rows=None, workspace=None, stream=None):
    """Rows x_rows [R, H] through experts row_ids - expert_base of the given banks ->
    fp32 [R, H] (one weighted slot of the layer per row, no combine)."""
    import torch
    R, H = x_rows.shape
    E, N2, _ = gate_up_blocks.shape
    if y_rows is None:
        y_rows = torch.empty((R, H), dtype=torch.float32, device=x_rows.device)
    ws = _dev(workspace, torch.uint8, "workspace")
    nbytes = 0 if workspace is None else workspace.numel()
    rc = load_library().moe_mxfp4_expert_rows(
        _dev(x_rows, torch.bfloat16, "x_rows"), R, H, N2 // 2, E, int(expert_base),
        _dev(row_ids, torch.int32, "row_ids"), _dev(row_weights, torch.float32, "row_weights"),
        _dev(gate_up_blocks, torch.uint8, "gate_up_blocks"), _dev(gate_up_scales, torch.uint8, "gate_up_scales"),
        _dev(gate_up_bias, torch.float32, "gate_up_bias"), _dev(down_blocks, torch.uint8, "down_blocks"),
        _dev(down_scales, torch.uint8, "down_scales"), _dev(down_bias, torch.float32, "down_bias"),
        float(alpha), float(limit), _dev(y_rows, torch.float32, "y_rows"), ctypes.c_uint32(flags), ws, nbytes,
        _stream(stream))
    _check("moe_mxfp4_expert_rows", rc)
    return y_rows


def moe_combine_pairs(y_rows, pair_rows, T: int, k: int, out=None, stream=None):
    """out[t] = sum_j y_rows[pair_rows[t*k + j]] (fp32 sum in slot order, bf16 out)."""
    import torch
    H = y_rows.shape[1]
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=y_rows.device)
    rc = load_library().moe_combine_pairs(_dev(y_rows, torch.float32, "y_rows"),
                                          _dev(pair_rows, torch.int32, "pair_rows"), int(T), int(k), H,
                                          _dev(out, torch.bfloat16, "out"), _stream(stream))
    _check("moe_combine_pairs", rc)
    return out


def moe_token_tile_rows(T: int, H: int, I: int, E: int, k: int, nvfp4: bool = False) -> int:
    """Token-tile height the forward uses for these sizes on the current device."""
    rc = int(load_library().moe_token_tile_rows(T, H, I, E, k, 1 if nvfp4 else 0))
    _check("moe_token_tile_rows", rc if rc < 0 else 0)
    return rc


def moe_mxfp4_workspace_size(T: int, H: int, I: int, E: int, k: int) -> int:
    return int(load_library().moe_mxfp4_workspace_size(T, H, I, E, k))


def moe_get_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the sticky device error bits."""
    rc = load_library().moe_get_device_error(_stream(stream))
    if rc < 0:
        raise MoEError("moe_get_device_error", rc)
    return rc


def moe_profile_enable(on: bool = True) -> None:
    """Start (or stop) CUDA-event timing of every kernel the library launches."""
    _check("moe_profile_enable", load_library().moe_profile_enable(1 if on else 0))


def moe_profile_enable_stages(stages) -> None:
    """Time only the named stages (an iterable of PROFILE_STAGES names); empty stops."""
    mask = 0
    for name in stages:
        mask |= 1 << PROFILE_STAGES.index(name)
    _check("moe_profile_enable_stages", load_library().moe_profile_enable_stages(ctypes.c_uint32(mask)))


def moe_profile_read():
    """Per-stage (kernel ms, launch count) since the previous read, as a dict."""
    n = len(PROFILE_STAGES)
    ms = (ctypes.c_double * n)()
    launches = (ctypes.c_int64 * n)()
    _check("moe_profile_read", load_library().moe_profile_read(ms, launches))
    return {name: (float(ms[i]), int(launches[i])) for i, name in enumerate(PROFILE_STAGES)}
