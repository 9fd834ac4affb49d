"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds no quantization arithmetic: it only draws random numbers,
applies the structure of each workload (outlier positions, outlier channels)
and converts to the storage type.  Recipe: numpy PCG64 streams, drawn in fp64,
structured in fp64, then rounded once to fp32 (``astype``); bf16 tensors are
the round-to-nearest-even bf16 of that fp32 tensor, kept as uint16 bit
patterns.

Workloads (shapes and distributions):

* ``gaussian``      iid N(0, 1) fp32 (4096 x 4096, seed 0)
* ``student_t``     Student-t(nu=3) x 1e-3 fp32 (8192 x 8192), small enough
                    that plain E4M3 block scales underflow
* ``razer_weight``  N(0, 0.02) with 0.1 % of positions (without replacement)
                    multiplied by 20, bf16 (8192 x 8192)
* ``razer_act``     N(0, 1) bf16 (16384 x 4096)
* ``mx_act``        N(0, 1) with 16 channels (columns) multiplied by 50, bf16
                    (8192 x 4096)
* ``mx_weight``     N(0, 0.02) bf16 (4096 x 4096)
* ``gemm_act``      N(0, 1) with round(0.005 * K) channels multiplied by 30,
                    bf16 (8192 x 4096)
* ``gemm_weight``   N(0, 0.02) bf16 (14336 x 4096)
"""
from __future__ import annotations

import numpy as np

# stream ids: one SeedSequence entropy per workload, so that changing one
# workload's size never changes another's values
_STREAM = {
    "student_t": 2,
    "razer_weight": 31,
    "razer_act": 32,
    "mx_act": 41,
    "mx_weight": 42,
    "gemm_act": 51,
    "gemm_weight": 52,
}

FULL_SHAPES = {
    "gaussian": (4096, 4096),
    "student_t": (8192, 8192),
    "razer_weight": (8192, 8192),
    "razer_act": (16384, 4096),
    "mx_act": (8192, 4096),
    "mx_weight": (4096, 4096),
    "gemm_act": (8192, 4096),
    "gemm_weight": (14336, 4096),
}

BF16_KINDS = {"razer_weight", "razer_act", "mx_act", "mx_weight", "gemm_act", "gemm_weight"}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as uint16 bit patterns (finite inputs)."""
    u = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _rng(kind: str, seed: int | None):
    if kind == "gaussian":
        return np.random.default_rng(0 if seed is None else seed)
    base = _STREAM[kind]
    return np.random.default_rng(np.random.SeedSequence([base] if seed is None else [base, seed]))


def generate(kind: str, rows: int | None = None, cols: int | None = None, seed: int | None = None):
    """Draw workload `kind` at (rows, cols) (default: its full size).

    Returns fp32 for the fp32 workloads and uint16 bf16 bit patterns for the
    bf16 ones.  `seed` selects an independent stream (None = the canonical one).
    """
    fr, fc = FULL_SHAPES[kind]
    rows = fr if rows is None else int(rows)
    cols = fc if cols is None else int(cols)
    g = _rng(kind, seed)
    if kind == "gaussian":
        x = g.standard_normal((rows, cols))
    elif kind == "student_t":
        x = g.standard_t(3.0, size=(rows, cols)) * 1e-3
    elif kind == "razer_weight":
        x = g.standard_normal((rows, cols)) * 0.02
        n_out = int(round(0.001 * rows * cols))
        pos = g.choice(rows * cols, size=n_out, replace=False)
        x.reshape(-1)[pos] *= 20.0
    elif kind in ("razer_act",):
        x = g.standard_normal((rows, cols))
    elif kind == "mx_act":
        x = g.standard_normal((rows, cols))
        ch = g.choice(cols, size=min(16, cols), replace=False)
        x[:, ch] *= 50.0
    elif kind in ("mx_weight", "gemm_weight"):
        x = g.standard_normal((rows, cols)) * 0.02
    elif kind == "gemm_act":
        x = g.standard_normal((rows, cols))
        n_ch = max(1, int(round(0.005 * cols)))
        ch = g.choice(cols, size=n_ch, replace=False)
        x[:, ch] *= 30.0
    else:
        raise KeyError(kind)
    x32 = x.astype(np.float32)
    if kind in BF16_KINDS:
        return f32_to_bf16_bits(x32)
    return x32


def as_f32(a: np.ndarray) -> np.ndarray:
    """fp32 view of a generated tensor (exact widening for bf16 bit patterns)."""
    if a.dtype == np.uint16:
        return bf16_bits_to_f32(a)
    return np.ascontiguousarray(a, np.float32)


def positive_vector(n: int, seed: int = 0, lo: float = 0.25, hi: float = 4.0) -> np.ndarray:
    """Seeded positive fp32 vector (log-uniform in [lo, hi]); stands in for a per-channel scale."""
    g = np.random.default_rng(np.random.SeedSequence([77, seed]))
    return np.exp(g.uniform(np.log(lo), np.log(hi), size=n)).astype(np.float32)
