"""Pins for the oracle's NVFP4 quantizer and its four scale rules.

What the pages fix ("Finer is Better (with the Right Scaling)", Methodology 2
and the findings on regions A/B; RaZeR summary section 1 on positive scales):
scales are non-negative; prevent-zero leaves no zero scale and removes the
underflow error; 4-over-6 picks the lower-error of the 4.0 / 6.0 mappings;
brute force is the minimum; brute-force error falls as blocks shrink.  Hand
examples pin the nibble order, the sign handling and the scale encode.
"""
from fractions import Fraction

import ml_dtypes as md
import numpy as np
import pytest

from block_scaled_fp4_03_b200 import inputs

E2M1 = [Fraction(v) for v in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]
ONE_E4M3 = 0x38   # 1.0 = exponent field 7, mantissa 0


def rules(O):
    return [O.RULE_ABSMAX, O.RULE_PREVENT_ZERO, O.RULE_FOUR_OVER_SIX, O.RULE_BRUTE_FORCE]


def test_exact_block_round_trips(O):
    """A block made of grid values with max 6 has scale 1, zero error, and known codes."""
    x = np.array([[0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.5, -1, -1.5, -2, -3, -4, -6, -0.0]], np.float32)
    for rule in rules(O):
        r = O.nvfp4_quantize(x, 16, rule, g=1.0)
        assert r["scales"][0, 0] == ONE_E4M3
        # element 2i in the low nibble, 2i+1 in the high nibble, sign in bit 3
        assert list(r["codes"][0]) == [0x10, 0x32, 0x54, 0x76, 0xA9, 0xCB, 0xED, 0x8F]
        assert np.array_equal(r["deq"].view(np.uint32), x.view(np.uint32))
        assert r["mse"][0, 0] == 0.0


def test_power_of_two_scale_and_global_scale(O):
    base = np.array([[6, -4, 3, 0.5, -1.5, 2, 1, 0]], np.float32)
    # scale 1/8 -> E4M3 0x20 (exponent field 4); global scale 1
    r = O.nvfp4_quantize(base / 8, 8, O.RULE_ABSMAX, g=1.0)
    assert r["scales"][0, 0] == 0x20 and r["mse"][0, 0] == 0.0
    # same block times 1000 with g = 1000/ (6*448) style global scale: S = sc * g
    g = np.float32(0.25)
    r = O.nvfp4_quantize(base * np.float32(0.25), 8, O.RULE_ABSMAX, g=g)
    assert r["scales"][0, 0] == ONE_E4M3 and r["mse"][0, 0] == 0.0


def test_four_over_six_hand_example(O):
    # block max 4: the 6-mapping scale 4/6 rounds to E4M3 0.6875 and leaves error,
    # the 4-mapping scale is exactly 1 and reproduces the block.
    x = np.array([[4, 2, 1, 3]], np.float32)
    r6 = O.nvfp4_quantize(x, 4, O.RULE_ABSMAX, g=1.0)
    assert O.e4m3_value(int(r6["scales"][0, 0])) == 0.6875
    assert list(O.e2m1_value(c & 0xF) for c in [r6["codes"][0, 0], r6["codes"][0, 1]]) == [6.0, 1.5]
    np.testing.assert_array_equal(r6["deq"][0], np.float32([4.125, 2.0625, 1.03125, 2.75]))
    assert r6["mse"][0, 0] == np.float32((0.125 ** 2 + 0.0625 ** 2 + 0.03125 ** 2 + 0.25 ** 2) / 4)
    r46 = O.nvfp4_quantize(x, 4, O.RULE_FOUR_OVER_SIX, g=1.0)
    assert r46["scales"][0, 0] == ONE_E4M3 and r46["mse"][0, 0] == 0.0


def test_prevent_zero_hand_example(O):
    # block max 1e-3 with g = 1: 1e-3/6 is below half the smallest E4M3 (2^-10), so
    # abs-max gives a zero scale (all codes zero); prevent-zero clamps to 2^-9.
    x = np.array([[1e-3, -5e-4, 2e-4, 0]], np.float32)
    am = O.nvfp4_quantize(x, 4, O.RULE_ABSMAX)
    pz = O.nvfp4_quantize(x, 4, O.RULE_PREVENT_ZERO)
    assert am["scales"][0, 0] == 0 and np.all(am["deq"] == 0)
    assert pz["scales"][0, 0] == 1 and O.e4m3_value(1) == 2.0 ** -9
    # 1e-3 / 2^-9 = 0.512 -> 0.5 ; -5e-4/2^-9 = -0.256 -> -0.5 ; 2e-4 -> 0.1024 -> 0
    np.testing.assert_array_equal(pz["deq"][0], np.float32([2.0 ** -10, -(2.0 ** -10), 0, 0]))
    assert pz["mse"][0, 0] < am["mse"][0, 0]


def test_negative_values_rounding_to_zero_keep_the_sign_bit(O):
    x = np.array([[6, -0.1, 0.1, -0.0]], np.float32)
    r = O.nvfp4_quantize(x, 4, O.RULE_ABSMAX)
    assert r["codes"][0, 0] == (0x7 | (0x8 << 4)) and r["codes"][0, 1] == (0x0 | (0x8 << 4))


def _data(kind, rows, cols, seed=0):
    return inputs.as_f32(inputs.generate(kind, rows, cols, seed=seed))


@pytest.mark.parametrize("B", [4, 8, 16, 32])
@pytest.mark.parametrize("kind,hier", [("student_t", False), ("student_t", True), ("gaussian", True)])
def test_rule_ordering_per_block(O, B, kind, hier):
    x = _data(kind, 48, 256, seed=B)
    g = O.global_scale(O.amax(x)) if hier else np.float32(1.0)
    res = {rule: O.nvfp4_quantize(x, B, rule, g=g) for rule in rules(O)}
    am, pz, fo, bf = (res[r]["mse"] for r in rules(O))
    # scales are never negative (sign bit of the E4M3 byte stays 0)
    for r in res.values():
        assert np.all(r["scales"] < 0x80)
    assert np.all(res[O.RULE_PREVENT_ZERO]["scales"] > 0)
    assert np.all(res[O.RULE_BRUTE_FORCE]["scales"] > 0)
    assert np.all(fo <= am)          # 4-over-6 keeps the 6-mapping unless 4 is better
    assert np.all(bf <= fo)          # brute force scans every candidate 4-over-6 can pick
    assert np.all(bf <= pz)
    assert np.all(pz <= am * (1 + 1e-6))
    # the decision metric is the error the outputs actually have
    err = (x.astype(np.float64) - res[O.RULE_BRUTE_FORCE]["deq"]).reshape(48, -1, B)
    np.testing.assert_allclose((err ** 2).mean(-1), bf, rtol=1e-5, atol=1e-30)


def test_region_a_underflow_and_prevent_zero(O):
    """Student-t x 1e-3 with plain E4M3 scales: many abs-max scales underflow to 0;
    prevent-zero leaves none and the zero-scale blocks' error drops."""
    x = _data("student_t", 64, 512)
    for B in (4, 8, 16, 32):
        am = O.nvfp4_quantize(x, B, O.RULE_ABSMAX)
        pz = O.nvfp4_quantize(x, B, O.RULE_PREVENT_ZERO)
        zero = am["scales"] == 0
        assert zero.sum() > 0
        assert np.all(pz["scales"] > 0)
        assert pz["mse"][zero].sum() < am["mse"][zero].sum()
        # blocks with a non-zero abs-max scale are untouched
        assert np.array_equal(pz["codes"].reshape(64, -1, B // 2)[~zero], am["codes"].reshape(64, -1, B // 2)[~zero])


def test_brute_force_mse_falls_as_blocks_shrink(O):
    """Nested partition: the two halves' optimal scales do at least as well as the parent's."""
    x = _data("gaussian", 64, 512, seed=5)
    tot = []
    for B in (32, 16, 8, 4):
        r = O.nvfp4_quantize(x, B, O.RULE_BRUTE_FORCE, g=1.0, want_deq=False)
        tot.append(r["mse"].astype(np.float64).mean())
    for big, small in zip(tot, tot[1:]):
        assert small <= big * (1 + 1e-6)
    assert tot[-1] < tot[0]


def _exact_block_sse(xb, s):
    """Exact-arithmetic SSE of block xb (Fractions) at effective scale s, RNE-to-grid, saturating."""
    tot = Fraction(0)
    for v in xb:
        v = Fraction(float(v))
        y = abs(v) / s
        if y >= 6:
            q = Fraction(6)
        else:
            best = None
            for i, gv in enumerate(E2M1):
                d = abs(y - gv)
                if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
                    best = (d, i)
            q = E2M1[best[1]]
        tot += (abs(v) - q * s) ** 2
    return tot


@pytest.mark.parametrize("nblocks,B", [(1, 4), (2, 8), (3, 16), (4, 4), (1, 32)])
def test_brute_force_tiny_exhaustive_exact(O, nblocks, B):
    rng = np.random.default_rng(100 + nblocks * B)
    x = (rng.standard_normal((1, nblocks * B)) * rng.choice([1e-3, 1.0, 30.0])).astype(np.float32)
    r = O.nvfp4_quantize(x, B, O.RULE_BRUTE_FORCE, g=1.0)
    e4 = [Fraction(O.e4m3_value(c)) for c in range(1, 0x7F)]
    for b in range(nblocks):
        xb = x[0, b * B:(b + 1) * B]
        exact = [_exact_block_sse(xb, s) for s in e4]
        best = min(exact)
        chosen = exact[int(r["scales"][0, b]) - 1]
        assert float(chosen) <= float(best) * (1 + 1e-5) + 1e-45
        # the oracle's reported mse is its chosen block's exact error (to fp32 accuracy)
        assert abs(float(r["mse"][0, b]) - float(chosen) / B) <= 1e-5 * float(chosen) / B + 1e-45


def test_codes_match_independent_encode(O):
    """Every code equals ml_dtypes' E2M1 cast of x / S computed the oracle's way."""
    x = _data("gaussian", 16, 128, seed=7)
    g = O.global_scale(O.amax(x))
    for rule in rules(O):
        r = O.nvfp4_quantize(x, 16, rule, g=g)
        sc = r["scales"].view(md.float8_e4m3fn).astype(np.float32)
        S = (sc * g).astype(np.float32)
        inv = np.where(S == 0, np.float32(0), np.minimum(np.float32(1) / S, np.finfo(np.float32).max)).astype(np.float32)
        y = (x.reshape(16, -1, 16) * inv[..., None]).astype(np.float32).reshape(16, -1)
        c = y.astype(md.float4_e2m1fn).view(np.uint8) & 0xF
        packed = (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
        assert np.array_equal(packed, r["codes"])
