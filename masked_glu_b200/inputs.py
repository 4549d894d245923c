"""Seeded synthetic inputs for MGLU, shared by the tests, the smoke check and
the benchmark.  This module holds no part of the method's arithmetic: it draws
random numbers and rounds them to the storage precision, nothing else.

Recipe (Llama-style FFN shapes; the pages train on FineWeb-Edu, which is not
used here -- these tensors stand in for a trained layer's inputs):

* ``numpy.random.Generator(PCG64(seed))``;
* x ~ N(0, 1), W and W_down ~ N(0, 0.02^2) (0.02 is a standard deviation);
* masks: n_m independent Bernoulli(p) draws per weight (p = 0.5 unless given);
* floating-point draws are made in float64, rounded to float32 (round to
  nearest even), and for bf16 inputs then rounded from float32 to bf16 (round
  to nearest even).  Both the CUDA path and the oracle consume exactly these
  rounded values.

Layouts: x [T][d]; W [h][d] (nn.Linear(d, h).weight); masks [n_m][h][d] uint8
in {0, 1}; W_down [d][h] (nn.Linear(h, d).weight).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np


def f32_to_bf16_bits(a32: np.ndarray) -> np.ndarray:
    """float32 array -> uint16 bf16 bit patterns, round to nearest even.
    NaN stays NaN (quiet)."""
    a32 = np.ascontiguousarray(a32, dtype=np.float32)
    u = a32.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = (u + 0x7FFF + lsb) >> 16
    nan = np.isnan(a32)
    out = r.astype(np.uint16)
    if nan.any():
        out[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def round_bf16(a: np.ndarray):
    """float64 -> (bf16 values as float64, uint16 bit patterns)."""
    bits = f32_to_bf16_bits(np.asarray(a, dtype=np.float64).astype(np.float32))
    return bf16_bits_to_f64(bits), bits


@dataclass
class Tensor:
    """One input tensor: its exact values (float64) and its storage form
    (uint16 bf16 bits or float32), shape as stored."""

    values: np.ndarray
    storage: np.ndarray
    dtype: str  # "bf16" or "f32"


def _make(a64: np.ndarray, dtype: str) -> Tensor:
    if dtype == "bf16":
        vals, bits = round_bf16(a64)
        return Tensor(vals, bits, "bf16")
    if dtype == "f32":
        s = a64.astype(np.float32)
        return Tensor(s.astype(np.float64), s, "f32")
    raise ValueError(dtype)


def normal(rng: np.random.Generator, shape, std: float, dtype: str) -> Tensor:
    return _make(rng.standard_normal(shape) * std, dtype)


def bernoulli_masks(rng: np.random.Generator, n_m: int, h: int, d: int, p: float) -> np.ndarray:
    """n_m independent Bernoulli(p) masks, [n_m][h][d] uint8 in {0, 1}; drawn
    one mask at a time to bound host memory."""
    out = np.empty((n_m, h, d), dtype=np.uint8)
    for i in range(n_m):
        if p == 0.5:
            out[i] = rng.integers(0, 2, size=(h, d), dtype=np.uint8)
        else:
            out[i] = (rng.random((h, d), dtype=np.float32) < np.float32(p)).astype(np.uint8)
    return out


@dataclass
class Case:
    T: int
    d: int
    h: int
    n_m: int
    dtype: str
    p: float
    seed: int
    x: Tensor
    W: Tensor
    masks: np.ndarray
    W_down: Optional[Tensor] = None
    note: str = field(default="")


def make_case(T: int, d: int, h: int, n_m: int, *, seed: int, p: float = 0.5,
              dtype: str = "bf16", w_std: float = 0.02, x_std: float = 1.0,
              with_down: bool = False) -> Case:
    """Draw one seeded case.  Draw order is fixed: W, masks, x, W_down."""
    rng = np.random.Generator(np.random.PCG64(seed))
    W = normal(rng, (h, d), w_std, dtype)
    masks = bernoulli_masks(rng, n_m, h, d, p)
    x = normal(rng, (T, d), x_std, dtype)
    Wd = normal(rng, (d, h), w_std, dtype) if with_down else None
    return Case(T, d, h, n_m, dtype, p, seed, x, W, masks, Wd)


# The workloads: Llama-style FFN shapes.  Seeds are 1000 + workload index,
# plus T for the token sweeps.
WORKLOADS = {
    "tiny_f32": dict(T=4, d=64, h=128, n_m=2, dtype="f32"),
    "decode_d2048_h8192_nm4": dict(T=1, d=2048, h=8192, n_m=4, dtype="bf16"),
    "decode_d4096_h14336_nm8": dict(T=1, d=4096, h=14336, n_m=8, dtype="bf16"),
    "prefill_T4096_d2048_h8192_nm4": dict(T=4096, d=2048, h=8192, n_m=4, dtype="bf16"),
    "ffn_d4096_h14336_nm8": dict(T=1, d=4096, h=14336, n_m=8, dtype="bf16"),
}
WORKLOAD_SEEDS = {name: 1000 + i for i, name in enumerate(WORKLOADS)}
