"""Pins for the oracle's UE5M3 block scale (the wide-exponent scale format the
"Finer is Better (with the Right Scaling)" summary compares against, findings
on format compatibility) and for the block quantizer run with it.

The page gives no bit layout; the reading (unsigned, 5 exponent bits with bias
15, 3 mantissa bits, subnormals, the all-ones code not a number) is pinned by
structure: counts per binade, the range, containment of every E4M3 scale,
exact nearest-value rounding, and the page's own comparison."""
from fractions import Fraction

import numpy as np
import pytest

from block_scaled_fp4_03_b200 import inputs


def values(O):
    return [Fraction(O.ue5m3_value(c)) for c in range(255)]


def test_table_structure(O):
    v = values(O)
    assert v[0] == 0
    assert all(a < b for a, b in zip(v, v[1:]))            # strictly increasing codes
    # 7 subnormals evenly spaced below the smallest normal, then 8 values per binade
    step = v[1]
    assert [v[k] for k in range(1, 9)] == [step * k for k in range(1, 9)]
    assert v[8] == Fraction(1, 2 ** 14)
    for lo in range(8, 255, 8):
        binade = v[lo:lo + 8]
        assert all(v[lo] <= b < 2 * v[lo] for b in binade)
        assert v[lo] * 2 == (v[lo + 8] if lo + 8 < 255 else v[lo] * 2)
    assert v[254] == Fraction(114688)                      # 1.75 * 2^16
    assert len(v) - 8 == 31 * 8 - 1                        # 31 binades, the last without 0xFF


def test_contains_every_e4m3_scale(O):
    v = set(values(O))
    for c in range(1, 0x7F):
        assert Fraction(O.e4m3_value(c)) in v


def nearest_ref(r, v):
    """Nearest table value by exact rationals, ties to the even code, saturating."""
    r = Fraction(r)
    if r >= v[-1]:
        return len(v) - 1
    for c in range(len(v) - 1):
        if r < v[c + 1]:
            lo, hi = v[c], v[c + 1]
            if 2 * r < lo + hi:
                return c
            if 2 * r > lo + hi:
                return c + 1
            return c if c % 2 == 0 else c + 1
    return len(v) - 1


def test_encode_is_nearest_ties_even(O):
    v = values(O)
    rng = np.random.default_rng(7)
    samples = list(np.float32(10.0) ** rng.uniform(-19, 6, 400).astype(np.float32))
    # every midpoint and its neighbours, and values beyond the range
    for c in range(254):
        mid = (v[c] + v[c + 1]) / 2
        m = np.float32(float(mid))
        samples += [m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(np.inf))]
    samples += [np.float32(0), np.float32(1e9), np.float32(114688), np.float32(120000)]
    for r in samples:
        assert O.ue5m3_encode(float(r)) == nearest_ref(float(r), v), r


def test_brute_force_never_worse_than_e4m3(O):
    """Every E4M3 scale is a UE5M3 scale, so the exhaustive UE5M3 search can only
    match or beat the E4M3 one, block by block (same data, g = 1)."""
    x = inputs.as_f32(inputs.generate("student_t", 8, 256, seed=9))
    for B in (4, 16):
        u = O.block_fp4_quantize(x, B, O.RULE_BRUTE_FORCE, O.SF_UE5M3, 1.0)["mse"]
        e = O.block_fp4_quantize(x, B, O.RULE_BRUTE_FORCE, O.SF_E4M3, 1.0)["mse"]
        assert np.all(u <= e)
        assert np.any(u < e)


def test_e4m3_path_unchanged(O):
    x = inputs.as_f32(inputs.generate("gaussian", 16, 128, seed=3))
    for rule in (O.RULE_ABSMAX, O.RULE_PREVENT_ZERO, O.RULE_FOUR_OVER_SIX, O.RULE_BRUTE_FORCE):
        a = O.nvfp4_quantize(x, 16, rule, g=0.01)
        b = O.block_fp4_quantize(x, 16, rule, O.SF_E4M3, 0.01)
        for k in ("codes", "scales", "deq", "mse"):
            assert np.array_equal(a[k], b[k])


@pytest.mark.parametrize("B", [4, 16, 32])
def test_page_claim_e4m3_recipe_matches_ue5m3(O, B):
    """The summary's finding: E4M3 with 4-over-6 and hierarchical scaling reaches
    the quality of the wide-exponent UE5M3 scale; without a global scale, E4M3
    abs-max underflows on small-magnitude data and UE5M3 does not."""
    x = inputs.as_f32(inputs.generate("student_t", 256, 1024, seed=2))
    g = O.global_scale(O.amax(x))
    ue_abs = O.block_fp4_quantize(x, B, O.RULE_ABSMAX, O.SF_UE5M3, 1.0)["mse"].mean()
    ue_46 = O.block_fp4_quantize(x, B, O.RULE_FOUR_OVER_SIX, O.SF_UE5M3, 1.0)["mse"].mean()
    e4_46h = O.nvfp4_quantize(x, B, O.RULE_FOUR_OVER_SIX, g=g)["mse"].mean()
    e4_abs1 = O.nvfp4_quantize(x, B, O.RULE_ABSMAX, g=1.0)["mse"].mean()
    assert e4_46h <= ue_abs
    assert abs(e4_46h - ue_46) <= 0.02 * ue_46
    assert e4_abs1 > 20 * ue_abs
    zero_scales = (O.block_fp4_quantize(x, B, O.RULE_ABSMAX, O.SF_UE5M3, 1.0)["scales"] == 0).mean()
    assert zero_scales < 1e-3


def _exact_block_sse(xb, s):
    """Exact SSE of block xb at scale s: RNE to the E2M1 grid (ties to the even
    code), saturating at 6 -- written out with rationals, independent of the
    oracle's fp32 arithmetic."""
    grid = [Fraction(v) for v in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]
    tot = Fraction(0)
    for v in xb:
        a = abs(Fraction(float(v)))
        y = a / s
        if y >= 6:
            q = grid[-1]
        else:
            q = min(range(8), key=lambda i: (abs(y - grid[i]), i % 2))
            q = grid[q]
        tot += (a - q * s) ** 2
    return tot


@pytest.mark.parametrize("B,mag", [(4, 1e-5), (8, 1.0), (16, 3e3), (4, 40.0)])
def test_brute_force_tiny_exhaustive_exact(O, B, mag):
    """UE5M3 brute force: over all 254 finite positive scales, the chosen one's
    exact block error is the minimum (to fp32 rounding of the search)."""
    rng = np.random.default_rng(int(B * 7 + mag * 3) % 1000)
    x = (rng.standard_normal((1, 2 * B)) * mag).astype(np.float32)
    r = O.block_fp4_quantize(x, B, O.RULE_BRUTE_FORCE, O.SF_UE5M3, 1.0)
    scales = [Fraction(O.ue5m3_value(c)) for c in range(1, 255)]
    for b in range(2):
        xb = x[0, b * B:(b + 1) * B]
        exact = [_exact_block_sse(xb, s) for s in scales]
        best = min(exact)
        chosen = exact[int(r["scales"][0, b]) - 1]
        assert float(chosen) <= float(best) * (1 + 1e-5) + 1e-45, (b, float(chosen), float(best))
