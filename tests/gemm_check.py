"""Element-wise checks of the tensor-core GEMM outputs against the oracle's fp64
product of the exactly decoded operands (test helper, no tests of its own).

For every checked element, with ref = g * sum_k a_k w_k (fp64) and
S = |g| * sum_k |a_k| |w_k| (the magnitude the fp32 accumulator runs through):

  fp32 accumulation slack   acc = (K / 16) * 2^-23 * S + 2^-22 * |ref|
      one fp32 unit in the last place of S for every 16-element block of K
      (each block's partial product is exact: E2M1 x E2M1 sums times two
      8-bit scales fit fp32's 24 bits; only the additions into the
      accumulator round), plus the two roundings of the global-scale product
  fp32 output   |out - ref| <= acc
  bf16 output   |out - ref| <= 2^-8 (|ref| + acc) + acc
      (round to nearest bf16, unit roundoff 2^-8, of a value within acc of ref)

A 16-element block whose scale is off by a factor 1 + e moves its output
elements by about e * (16 / K) * S, which these bounds see for e of a few
percent, wherever the block sits; a whole-matrix norm would dilute it.
On top: relative Frobenius error <= 1e-5 against the raw fp64 product for
fp32 output, and <= 1e-3 against the bf16-rounded product for bf16 output.

If FP4Q_PARITY_LOG names a file, every check appends one JSON line with the
achieved errors.
"""
import json
import os

import numpy as np
import torch

from block_scaled_fp4_03_b200 import inputs


def bf16_round(x64):
    f = x64.astype(np.float32)
    return inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits(f)).astype(np.float64)


def band_rows(M, salt=0):
    """One row in every 128-row band (the M extent of a CTA's tile), its
    position inside the band varying so that every TMEM lane quarter is hit."""
    bands = np.arange(M // 128)
    return bands * 128 + (bands * 37 + 11 + salt) % 128


def check_gemm(out, da, dw, g, K, label=""):
    """Compare `out` (device tensor, bf16 or fp32, rows x cols) with
    g * da @ dw^T; da / dw are the exactly decoded fp64 operands of the same
    rows / columns."""
    from oracle import oracle as O
    got = out.float().cpu().numpy().astype(np.float64)
    ref = O.gemm_values(da, dw, g, 1.0)
    mag = O.gemm_values(np.abs(da), np.abs(dw), abs(float(g)), 1.0)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), label
    acc = (K / 16.0) * 2.0 ** -23 * mag + 2.0 ** -22 * np.abs(ref)
    fp32 = out.dtype == torch.float32
    tol = acc if fp32 else 2.0 ** -8 * (np.abs(ref) + acc) + acc
    err = np.abs(got - ref)
    ratio = err / np.maximum(tol, np.finfo(np.float64).tiny)
    worst = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
    den = np.linalg.norm(ref)
    e_raw = float(np.linalg.norm(got - ref) / den) if den > 0 else 0.0
    e_b = float(np.linalg.norm(got - bf16_round(ref)) / den) if den > 0 else 0.0
    stats = dict(label=label, dtype="f32" if fp32 else "bf16", shape=list(got.shape), K=int(K),
                 frob_raw=e_raw, frob_vs_bf16=e_b, max_err_over_bound=float(ratio[worst]),
                 max_abs_err=float(err.max()))
    path = os.environ.get("FP4Q_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(stats) + "\n")
    assert ratio[worst] <= 1.0, (label, worst, got[worst], ref[worst], tol[worst], stats)
    if fp32:
        assert e_raw <= 1e-5, stats
    else:
        assert e_b <= 1e-3, stats
    return stats
