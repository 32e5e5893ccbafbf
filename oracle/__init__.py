"""CPU oracle for the MXFP4 expert-FFN MoE layer (ctypes wrapper around moe_oracle.c).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the package smoke check and
the benchmark's CPU-baseline leg may import this module.  It shares nothing with the
CUDA path: the arithmetic lives in ``moe_oracle.c`` (plain C, double precision), and
this file only marshals numpy arrays into it.

What each entry point follows is cited in ``moe_oracle.c``; in short:

* ``dequantize``  -- MoE-Infinity PR #152 "expert offloading Phase 2 -- MXFP4
  dequant-on-copy execution", Changes (golden test, rel-err 0.0); onnxruntime/mobius
  PR #719 "Add native GPT-OSS MXFP4 QMoE export", Summary/Validation (block layout,
  E8M0 byte validity); OCP MX v1.0 for the E2M1 and E8M0 element definitions.
* ``route``       -- top-k over router logits then softmax over the k chosen
  (transformers PR #49431: the MXFP4 experts take routing ids + weights).
* ``router_logits`` -- the router linear layer before it, x . W_r^T + b_r (FreeToken
  PR #838: the gpt-oss router is mlp.router, with a bias).
* ``forward_tokens`` / ``forward_grouped`` -- FreeToken PR #838 "feat(gguf): serve
  gpt-oss gguf checkpoints on gpt_oss", review items on the down bias and on
  apply_router_weight_on_input, and "What it does" (alpha 1.702, limit 7, bias roles).
* ``e4m3_value`` / ``nvfp4_dequantize`` / ``nvfp4_forward_tokens`` -- the NVFP4 expert
  variant: E2M1 codes with one E4M3 scale per 16 elements (OCP OFP8 v1.0 for E4M3)
  and a per-expert fp32 weight_scale_2 that multiplies each projection before its
  bias (FreeToken PR #838, review item "NVFP4 down scale vs. down bias").

Every function here is pinned by the CPU tests against hand-written values, closed
forms, invariants or a library routine; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

DEFECT_NONE = 0
DEFECT_NIBBLE_SWAP = 1
DEFECT_E8M0_BIAS_126 = 2
DEFECT_GATE_ZERO = 3
DEFECT_NO_CLAMP = 4
DEFECT_UNINTERLEAVED = 5
DEFECT_DOWN_BIAS_UNWEIGHTED = 6
DEFECT_WOI_BIAS_WEIGHTED = 7
DEFECT_DOWN_BIAS_IN_SCALE = 8
DEFECT_NVFP4_SCALE_AFTER_BIAS = 9
DEFECT_NVFP4_BLOCK32 = 10
DEFECT_NVFP4_GU_SCALE_SWAP = 11
DEFECT_OPERAND_E4M3_HI_ONLY = 12

FLAG_WEIGHT_ON_INPUT = 1


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so beside it (gcc, OpenMP, strict FP)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", _SRC, "-o", _LIB, "-lm"]
    subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        p = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.oracle_e2m1_value.restype = ctypes.c_double
        lib.oracle_e2m1_value.argtypes = [ctypes.c_int]
        lib.oracle_e8m0_value.restype = ctypes.c_double
        lib.oracle_e8m0_value.argtypes = [ctypes.c_int, ctypes.c_int]
        lib.oracle_double_to_bf16.restype = ctypes.c_uint16
        lib.oracle_double_to_bf16.argtypes = [ctypes.c_double]
        lib.oracle_bf16_to_double.restype = ctypes.c_double
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_swiglu.restype = ctypes.c_double
        lib.oracle_swiglu.argtypes = [ctypes.c_double] * 4 + [ctypes.c_int]
        lib.oracle_dequantize.restype = None
        lib.oracle_dequantize.argtypes = [p, p, p, i64, i64, i64, ctypes.c_int]
        lib.oracle_route.restype = None
        lib.oracle_route.argtypes = [p, i64, i64, ctypes.c_int, p, p]
        lib.oracle_forward_tokens.restype = None
        lib.oracle_forward_tokens.argtypes = [p, i64, i64, i64, i64, ctypes.c_int, p, p,
                                              p, p, p, p, p, p, ctypes.c_double, ctypes.c_double,
                                              ctypes.c_int, p, i64, p, p, ctypes.c_int]
        lib.oracle_forward_grouped.restype = ctypes.c_int
        lib.oracle_forward_grouped.argtypes = [p, i64, i64, i64, i64, ctypes.c_int, p, p,
                                               p, p, p, p, p, p, ctypes.c_double, ctypes.c_double,
                                               ctypes.c_int, p]
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_e4m3_value.argtypes = [ctypes.c_int]
        lib.oracle_nvfp4_dequantize.restype = None
        lib.oracle_nvfp4_dequantize.argtypes = [p, p, p, p, i64, i64, i64, ctypes.c_int]
        lib.oracle_nvfp4_forward_tokens.restype = None
        lib.oracle_nvfp4_forward_tokens.argtypes = [p, i64, i64, i64, i64, ctypes.c_int, p, p,
                                                    p, p, p, p, p, p, p, p, ctypes.c_double,
                                                    ctypes.c_double, ctypes.c_int, p, i64, p, p,
                                                    ctypes.c_int]
        lib.oracle_router_logits.restype = None
        lib.oracle_router_logits.argtypes = [p, p, p, i64, i64, i64, p]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def e2m1_value(code: int) -> float:
    return _load().oracle_e2m1_value(int(code))


def e8m0_value(b: int, defect: int = DEFECT_NONE) -> float:
    return _load().oracle_e8m0_value(int(b), int(defect))


def double_to_bf16(v: float) -> int:
    return int(_load().oracle_double_to_bf16(float(v)))


def bf16_to_double(bits: int) -> float:
    return _load().oracle_bf16_to_double(int(bits))


def swiglu(gate: float, up: float, alpha: float = 1.702, limit: float = 7.0,
           defect: int = DEFECT_NONE) -> float:
    return _load().oracle_swiglu(float(gate), float(up), float(alpha), float(limit), int(defect))


def dequantize(blocks, scales, E: int, N: int, K: int, defect: int = DEFECT_NONE) -> np.ndarray:
    """Packed [E,N,K/2] + E8M0 [E,N,K/32] -> bf16 bit patterns, uint16 [E,N,K]."""
    blocks = _c(blocks, np.uint8)
    scales = _c(scales, np.uint8)
    assert blocks.size == E * N * K // 2 and scales.size == E * N * K // 32
    out = np.empty((E, N, K), dtype=np.uint16)
    _load().oracle_dequantize(_ptr(blocks), _ptr(scales), _ptr(out), E, N, K, int(defect))
    return out


def route(logits, k: int):
    """fp32 logits [T,E] -> (ids int32 [T,k], weights float32 [T,k])."""
    logits = _c(logits, np.float32)
    T, E = logits.shape
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float32)
    _load().oracle_route(_ptr(logits), T, E, int(k), _ptr(ids), _ptr(w))
    return ids, w


def forward_tokens(x_bits, ids, weights, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales,
                   d_bias, alpha=1.702, limit=7.0, weight_on_input=False, tokens=None,
                   defect: int = DEFECT_NONE, envelope: bool = False):
    """Formulation A.  x_bits: bf16 bits uint16 [T,H].  Returns float64 [len(tokens), H],
    or (out, env) with the down projection's magnitude envelope when envelope=True."""
    x_bits = _c(x_bits, np.uint16)
    T, H = x_bits.shape
    ids = _c(ids, np.int32)
    k = ids.shape[1]
    weights = _c(weights, np.float32)
    gu_blocks = _c(gu_blocks, np.uint8)
    E = gu_blocks.shape[0]
    I = gu_blocks.shape[1] // 2
    if tokens is None:
        tokens = np.arange(T, dtype=np.int64)
    tokens = _c(tokens, np.int64)
    out = np.empty((tokens.size, H), dtype=np.float64)
    env = np.empty((tokens.size, H), dtype=np.float64) if envelope else None
    _load().oracle_forward_tokens(
        _ptr(x_bits), T, H, I, E, k, _ptr(ids), _ptr(weights), _ptr(gu_blocks),
        _ptr(_c(gu_scales, np.uint8)), _ptr(_c(gu_bias, np.float32)), _ptr(_c(d_blocks, np.uint8)),
        _ptr(_c(d_scales, np.uint8)), _ptr(_c(d_bias, np.float32)), float(alpha), float(limit),
        FLAG_WEIGHT_ON_INPUT if weight_on_input else 0, _ptr(tokens), tokens.size, _ptr(out),
        _ptr(env), int(defect))
    return (out, env) if envelope else out


def forward_grouped(x_bits, ids, weights, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales,
                    d_bias, alpha=1.702, limit=7.0, weight_on_input=False) -> np.ndarray:
    """Formulation B (pairs grouped by expert over a decoded bank).  float64 [T,H]."""
    x_bits = _c(x_bits, np.uint16)
    T, H = x_bits.shape
    ids = _c(ids, np.int32)
    k = ids.shape[1]
    gu_blocks = _c(gu_blocks, np.uint8)
    E = gu_blocks.shape[0]
    I = gu_blocks.shape[1] // 2
    out = np.empty((T, H), dtype=np.float64)
    rc = _load().oracle_forward_grouped(
        _ptr(x_bits), T, H, I, E, k, _ptr(ids), _ptr(_c(weights, np.float32)), _ptr(gu_blocks),
        _ptr(_c(gu_scales, np.uint8)), _ptr(_c(gu_bias, np.float32)), _ptr(_c(d_blocks, np.uint8)),
        _ptr(_c(d_scales, np.uint8)), _ptr(_c(d_bias, np.float32)), float(alpha), float(limit),
        FLAG_WEIGHT_ON_INPUT if weight_on_input else 0, _ptr(out))
    if rc != 0:
        raise MemoryError("oracle_forward_grouped: allocation failed")
    return out


def router_logits(x_bits, w_bits, bias=None) -> np.ndarray:
    """Router linear layer: bf16 x [T,H] and W_r [E,H] (bits), fp32 bias [E] or None
    -> float64 logits [T,E]."""
    x_bits = _c(x_bits, np.uint16)
    w_bits = _c(w_bits, np.uint16)
    T, H = x_bits.shape
    E = w_bits.shape[0]
    assert w_bits.shape[1] == H
    out = np.empty((T, E), dtype=np.float64)
    _load().oracle_router_logits(_ptr(x_bits), _ptr(w_bits), _ptr(_c(bias, np.float32)), T, H, E,
                                 _ptr(out))
    return out


def e4m3_value(b: int) -> float:
    return _load().oracle_e4m3_value(int(b))


def nvfp4_dequantize(blocks, scales, scale2, E: int, N: int, K: int,
                     defect: int = DEFECT_NONE) -> np.ndarray:
    """Packed [E,N,K/2] + E4M3 [E,N,K/16] (+ fp32 [E] or None) -> bf16 bits uint16 [E,N,K]."""
    blocks = _c(blocks, np.uint8)
    scales = _c(scales, np.uint8)
    scale2 = _c(scale2, np.float32)
    assert blocks.size == E * N * K // 2 and scales.size == E * N * K // 16
    assert scale2 is None or scale2.size == E
    out = np.empty((E, N, K), dtype=np.uint16)
    _load().oracle_nvfp4_dequantize(_ptr(blocks), _ptr(scales), _ptr(scale2), _ptr(out), E, N, K,
                                    int(defect))
    return out


def nvfp4_forward_tokens(x_bits, ids, weights, gu_blocks, gu_scales, gu_scale2, gu_bias,
                         d_blocks, d_scales, d_scale2, d_bias, alpha=1.702, limit=7.0,
                         weight_on_input=False, tokens=None, defect: int = DEFECT_NONE,
                         envelope: bool = False):
    """Formulation A with NVFP4 experts.  gu_scale2 fp32 [E, 2] (gate, up) and d_scale2
    fp32 [E] may be None (1).  Returns float64 [len(tokens), H] (and the envelope)."""
    x_bits = _c(x_bits, np.uint16)
    T, H = x_bits.shape
    ids = _c(ids, np.int32)
    k = ids.shape[1]
    weights = _c(weights, np.float32)
    gu_blocks = _c(gu_blocks, np.uint8)
    E = gu_blocks.shape[0]
    I = gu_blocks.shape[1] // 2
    gu_scale2 = _c(gu_scale2, np.float32)
    d_scale2 = _c(d_scale2, np.float32)
    assert gu_scale2 is None or gu_scale2.size == 2 * E
    assert d_scale2 is None or d_scale2.size == E
    if tokens is None:
        tokens = np.arange(T, dtype=np.int64)
    tokens = _c(tokens, np.int64)
    out = np.empty((tokens.size, H), dtype=np.float64)
    env = np.empty((tokens.size, H), dtype=np.float64) if envelope else None
    _load().oracle_nvfp4_forward_tokens(
        _ptr(x_bits), T, H, I, E, k, _ptr(ids), _ptr(weights), _ptr(gu_blocks),
        _ptr(_c(gu_scales, np.uint8)), _ptr(gu_scale2), _ptr(_c(gu_bias, np.float32)),
        _ptr(_c(d_blocks, np.uint8)), _ptr(_c(d_scales, np.uint8)), _ptr(d_scale2),
        _ptr(_c(d_bias, np.float32)), float(alpha), float(limit),
        FLAG_WEIGHT_ON_INPUT if weight_on_input else 0, _ptr(tokens), tokens.size, _ptr(out),
        _ptr(env), int(defect))
    return (out, env) if envelope else out


def num_threads() -> int:
    return int(_load().oracle_num_threads())
