"""Seeded synthetic inputs for the MXFP4 expert-FFN MoE layer.

This module only draws random inputs with the shapes and value distributions of
gpt-oss-shaped MoE layers; it contains none of the layer's arithmetic.  Both the
CUDA path's tests/benchmark and the CPU oracle consume the same arrays from here.

Recipe (every array from ``numpy.random.default_rng(seed)``, drawn in this order):

* ``x``       bf16 [T, H], N(0, 1) rounded to bf16 (nearest, ties to even)
* ``logits``  fp32 [T, E], N(0, 1); with ``zipf`` > 0 each column e gets the offset
              ``zipf * log(1 / (e + 1))`` so that expert 0 is the most popular
* gate_up     packed uint8 [E, 2I, H/2] uniform over all bytes (two uniform E2M1
              codes per byte), E8M0 scales uint8 [E, 2I, H/32] uniform in
              [scale_lo, scale_hi], bias fp32 [E, 2I] N(0, bias_std^2), bias_std = 0.02
* down        packed uint8 [E, H, I/2], scales [E, H, I/32], bias fp32 [E, H], same laws

NVFP4 layers (``fmt="nvfp4"``) draw in the same order with one E4M3 scale byte per 16
elements ([E, N, K/16], uniform in [e4m3_lo, e4m3_hi] = [0x08, 0x37]: 2^-6 .. 0.9375,
sign clear), then append the per-expert fp32 weight_scale_2 draws: gate_up [E, 2]
(gate, up) and down [E], uniform in [0.5, 1).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round finite float32 values to bfloat16 bit patterns (nearest, ties to even)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class ExpertBank:
    """One packed projection bank: blocks [E, N, K/2] and scales, E8M0 [E, N, K/32]
    (MXFP4) or E4M3 [E, N, K/16] with a per-expert fp32 ``scale2`` (NVFP4)."""
    blocks: np.ndarray
    scales: np.ndarray
    scale2: Optional[np.ndarray] = None

    @property
    def shape(self):
        E, N, Kh = self.blocks.shape
        return E, N, 2 * Kh


@dataclass
class MoELayer:
    T: int
    H: int
    I: int
    E: int
    k: int
    x_bits: np.ndarray            # uint16 [T, H] (bf16 bit patterns)
    logits: np.ndarray            # float32 [T, E]
    gate_up: ExpertBank           # [E, 2I, H/2] / [E, 2I, H/32]
    gate_up_bias: Optional[np.ndarray]  # float32 [E, 2I] or None
    down: ExpertBank              # [E, H, I/2] / [E, H, I/32]
    down_bias: Optional[np.ndarray]     # float32 [E, H] or None
    alpha: float = 1.702
    limit: float = 7.0
    weight_on_input: bool = False
    name: str = field(default="")
    fmt: str = "mxfp4"


E4M3_LO, E4M3_HI = 0x08, 0x37


def make_bank(rng: np.random.Generator, E: int, N: int, K: int, scale_lo: int,
              scale_hi: int, block: int = 32) -> ExpertBank:
    blocks = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    scales = rng.integers(scale_lo, scale_hi + 1, size=(E, N, K // block), dtype=np.uint8)
    return ExpertBank(blocks, scales)


def make_layer(T: int, H: int, I: int, E: int, k: int, seed: int = 0, scale_lo: int = 118,
               scale_hi: int = 126, zipf: float = 0.0, biases: bool = True,
               weight_on_input: bool = False, bias_std: float = 0.02,
               name: str = "", fmt: str = "mxfp4", x_dist: str = "normal") -> MoELayer:
    assert fmt in ("mxfp4", "nvfp4") and x_dist in ("normal", "wide")
    if fmt == "nvfp4":
        return _make_nvfp4_layer(T, H, I, E, k, seed, zipf, biases, weight_on_input, bias_std, name)
    rng = np.random.default_rng(seed)
    if x_dist == "wide":
        x_bits = _wide_range_rows(rng, T, H)
    else:
        x_bits = f32_to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    logits = rng.standard_normal((T, E), dtype=np.float32)
    if zipf:
        rank = np.arange(1, E + 1, dtype=np.float64)
        logits = (logits + (zipf * np.log(1.0 / rank)).astype(np.float32)[None, :]).astype(np.float32)
    gu = make_bank(rng, E, 2 * I, H, scale_lo, scale_hi)
    gu_bias = (bias_std * rng.standard_normal((E, 2 * I))).astype(np.float32)
    dn = make_bank(rng, E, H, I, scale_lo, scale_hi)
    d_bias = (bias_std * rng.standard_normal((E, H))).astype(np.float32)
    if not biases:
        gu_bias = None
        d_bias = None
    return MoELayer(T, H, I, E, k, x_bits, logits, gu, gu_bias, dn, d_bias,
                    weight_on_input=weight_on_input, name=name)


def _wide_range_rows(rng: np.random.Generator, T: int, H: int) -> np.ndarray:
    """bf16 rows whose 32-element blocks each hold one large element (magnitude
    2^u, u uniform in [0, 3)) at a random position and 31 smaller ones spread
    log-uniformly from it down to 2^-20 of it, random signs."""
    nb = H // 32
    big = 2.0 ** rng.uniform(0.0, 3.0, size=(T, nb, 1))
    below = rng.uniform(0.0, 20.0, size=(T, nb, 32))
    pos = rng.integers(0, 32, size=(T, nb))
    np.put_along_axis(below, pos[..., None], 0.0, axis=2)
    sign = np.where(rng.integers(0, 2, size=(T, nb, 32)) == 1, -1.0, 1.0)
    x = (sign * big * 2.0 ** (-below)).reshape(T, H).astype(np.float32)
    return f32_to_bf16_bits(x)


def _make_nvfp4_layer(T, H, I, E, k, seed, zipf, biases, weight_on_input, bias_std, name):
    rng = np.random.default_rng(seed)
    x_bits = f32_to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    logits = rng.standard_normal((T, E), dtype=np.float32)
    if zipf:
        rank = np.arange(1, E + 1, dtype=np.float64)
        logits = (logits + (zipf * np.log(1.0 / rank)).astype(np.float32)[None, :]).astype(np.float32)
    gu = make_bank(rng, E, 2 * I, H, E4M3_LO, E4M3_HI, block=16)
    gu_bias = (bias_std * rng.standard_normal((E, 2 * I))).astype(np.float32)
    dn = make_bank(rng, E, H, I, E4M3_LO, E4M3_HI, block=16)
    d_bias = (bias_std * rng.standard_normal((E, H))).astype(np.float32)
    gu.scale2 = rng.uniform(0.5, 1.0, size=(E, 2)).astype(np.float32)
    dn.scale2 = rng.uniform(0.5, 1.0, size=(E,)).astype(np.float32)
    if not biases:
        gu_bias = None
        d_bias = None
    return MoELayer(T, H, I, E, k, x_bits, logits, gu, gu_bias, dn, d_bias,
                    weight_on_input=weight_on_input, name=name, fmt="nvfp4")


def make_nvfp4_dequant_bank(seed: int = 0, E: int = 32, H: int = 2880, I: int = 2880):
    """gpt-oss-20b-shaped NVFP4 expert bank for the standalone dequant workload."""
    rng = np.random.default_rng(seed)
    gu = make_bank(rng, E, 2 * I, H, E4M3_LO, E4M3_HI, block=16)
    dn = make_bank(rng, E, H, I, E4M3_LO, E4M3_HI, block=16)
    gu.scale2 = rng.uniform(0.5, 1.0, size=(E,)).astype(np.float32)
    dn.scale2 = rng.uniform(0.5, 1.0, size=(E,)).astype(np.float32)
    return gu, dn


def make_dequant_bank(seed: int = 0, E: int = 32, H: int = 2880, I: int = 2880,
                      scale_lo: int = 110, scale_hi: int = 130):
    """gpt-oss-20b-shaped expert bank for the standalone dequant-on-copy workload."""
    rng = np.random.default_rng(seed)
    gu = make_bank(rng, E, 2 * I, H, scale_lo, scale_hi)
    dn = make_bank(rng, E, H, I, scale_lo, scale_hi)
    return gu, dn


# Named workloads: gpt-oss-20b (E=32) and gpt-oss-120b (E=128) shaped layers.
WORKLOADS = {
    "tiny_woo": dict(T=8, H=128, I=128, E=4, k=2, biases=True, weight_on_input=False),
    "tiny_woi": dict(T=8, H=128, I=128, E=4, k=2, biases=False, weight_on_input=True),
    # test case only: biases as large as the expert outputs, so that a mistake in
    # where the biases enter is visible at the layer-output tolerance
    "tiny_bias_heavy": dict(T=8, H=128, I=128, E=4, k=2, biases=True, bias_std=8.0),
    "20b_decode_T1": dict(T=1, H=2880, I=2880, E=32, k=4),
    "20b_decode_T8": dict(T=8, H=2880, I=2880, E=32, k=4),
    "20b_decode_T64": dict(T=64, H=2880, I=2880, E=32, k=4),
    "20b_prefill_T4096": dict(T=4096, H=2880, I=2880, E=32, k=4),
    "120b_zipf_T256": dict(T=256, H=2880, I=2880, E=128, k=4, zipf=1.5),
    "120b_zipf_T8192": dict(T=8192, H=2880, I=2880, E=128, k=4, zipf=1.5),
    # test cases only: activation blocks spanning 2^20 (one large element, the rest
    # down to 2^-20 of it) and heavy gate_up biases (gate values far below zero give
    # activations near zero beside large ones), the hardest inputs for an operand
    # kept as a few significant bits per block scale
    "tiny_wide": dict(T=16, H=256, I=256, E=4, k=2, x_dist="wide", bias_std=3.0),
    "20b_decode_wide_T8": dict(T=8, H=2880, I=2880, E=32, k=4, x_dist="wide", bias_std=3.0),
    # the NVFP4 expert variant of the same layers
    "nvfp4_tiny_woo": dict(T=8, H=128, I=128, E=4, k=2, biases=True, fmt="nvfp4"),
    "nvfp4_tiny_woi": dict(T=8, H=128, I=128, E=4, k=2, biases=False, weight_on_input=True,
                           fmt="nvfp4"),
    "nvfp4_tiny_bias_heavy": dict(T=8, H=128, I=128, E=4, k=2, biases=True, bias_std=8.0,
                                  fmt="nvfp4"),
    "nvfp4_20b_decode_T8": dict(T=8, H=2880, I=2880, E=32, k=4, fmt="nvfp4"),
    "nvfp4_20b_prefill_T4096": dict(T=4096, H=2880, I=2880, E=32, k=4, fmt="nvfp4"),
}


@dataclass
class Router:
    """Router linear layer inputs: x bf16 bits [T, H], W_r bf16 bits [E, H], b_r fp32 [E]."""
    x_bits: np.ndarray
    w_bits: np.ndarray
    bias: Optional[np.ndarray]
    k: int


def make_router(T: int, H: int, E: int, k: int, seed: int = 0, bias: bool = True) -> Router:
    """x ~ N(0, 1), W_r ~ N(0, 1/H) (logits of unit scale), b_r ~ N(0, 0.1^2); in that order."""
    rng = np.random.default_rng(seed)
    x_bits = f32_to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    w_bits = f32_to_bf16_bits((rng.standard_normal((E, H)) / np.sqrt(H)).astype(np.float32))
    b = (0.1 * rng.standard_normal(E)).astype(np.float32)
    return Router(x_bits, w_bits, b if bias else None, k)


ROUTERS = {
    "router_20b_T4096": dict(T=4096, H=2880, E=32, k=4),
    "router_20b_T8": dict(T=8, H=2880, E=32, k=4),
    "router_120b_T8192": dict(T=8192, H=2880, E=128, k=4),
}


def router_workload(name: str, seed: int = 0) -> Router:
    return make_router(seed=seed, **ROUTERS[name])


def workload(name: str, seed: int = 0) -> MoELayer:
    return make_layer(seed=seed, name=name, **WORKLOADS[name])
