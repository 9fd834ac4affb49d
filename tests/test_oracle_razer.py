"""Pins for the oracle's RaZeR quantizer (redundant-zero remapping).

RaZeR technical summary, sections 2.1-2.2: weights use an E3M3 scale and 2
free bits choosing one of 4 special values, activations an E4M3 scale whose
sign bit picks one of 2; the -0 code is remapped to the block's special
value, chosen for minimum squared error; +-5 is the best pair.
"""
import json
import os

import numpy as np
import pytest

from block_scaled_fp4_03_b200 import inputs

W_SPECIALS = [5.0, -5.0, 3.5, -3.5]
A_SPECIALS = [5.0, -5.0]
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def _x(kind, rows, cols, seed=0):
    return inputs.as_f32(inputs.generate(kind, rows, cols, seed=seed))


def test_hand_example_positive_and_negative_specials(O):
    # scale 1 (block max 6, g = 1): 5 sits on a tie of the E2M1 grid (4 | 6) and
    # goes to 4 in plain NVFP4; with the +5 special it is exact.
    x = np.zeros((2, 16), np.float32)
    x[0, :3] = [6, 5, 4]
    x[1, :3] = [-6, -5, -4]
    r = O.razer_quantize(x, O.SF_E4M3, A_SPECIALS, g=1.0)
    assert r["meta"][0, 0] == (0 << 7) | 0x38
    assert r["meta"][1, 0] == (1 << 7) | 0x38
    assert r["codes"][0, 0] == (0x7 | (0x8 << 4)) and (r["codes"][0, 1] & 0xF) == 0x6
    assert r["codes"][1, 0] == (0xF | (0x8 << 4)) and (r["codes"][1, 1] & 0xF) == 0xE
    assert np.all(r["mse"] == 0.0)
    assert r["deq"][0, 1] == 5.0 and r["deq"][1, 1] == -5.0
    # plain NVFP4 of the same block errs by 1 on the 5
    p = O.nvfp4_quantize(x, 16, O.RULE_ABSMAX, g=1.0)
    assert p["mse"][0, 0] == np.float32(1.0 / 16)


def test_small_negatives_never_take_the_special_code(O):
    x = np.zeros((1, 16), np.float32)
    x[0, :4] = [6, -0.1, -0.0, 0.1]
    r = O.razer_quantize(x, O.SF_E4M3, A_SPECIALS, g=1.0)
    c = [(r["codes"][0, i // 2] >> (4 * (i % 2))) & 0xF for i in range(4)]
    assert c == [0x7, 0x0, 0x0, 0x0]


def test_weight_meta_byte_layout(O):
    x = _x("razer_weight", 32, 256, seed=3)
    g = O.global_scale(O.amax(x), O.SF_E3M3)
    r = O.razer_quantize(x, O.SF_E3M3, W_SPECIALS, g=g)
    sel, sc = r["meta"] >> 6, r["meta"] & 0x3F
    assert sel.max() <= 3 and sc.max() <= 63
    # the 6-bit scale is the E3M3 abs-max scale of the block
    a = np.abs(x).reshape(32, -1, 16).max(-1)
    expect = np.array([[O.e3m3_encode(float(np.float32(v) / np.float32(6 * g))) for v in row] for row in a])
    assert np.array_equal(sc, expect)


@pytest.mark.parametrize("sf,kind,specials", [(1, "razer_weight", W_SPECIALS), (0, "razer_act", A_SPECIALS)])
def test_never_worse_than_plain_per_block(O, sf, kind, specials):
    x = _x(kind, 64, 512, seed=sf)
    g = O.global_scale(O.amax(x), sf)
    rz = O.razer_quantize(x, sf, specials, g=g)
    # a special value no element can be nearer to reproduces plain block quantization
    plain = O.razer_quantize(x, sf, [100.0], g=g)
    assert np.all(rz["mse"] <= plain["mse"] * (1 + 1e-6))
    assert rz["mse"].astype(np.float64).sum() < plain["mse"].astype(np.float64).sum()
    if sf == O.SF_E4M3:
        nv = O.nvfp4_quantize(x, 16, O.RULE_ABSMAX, g=g)
        assert np.array_equal(nv["mse"].view(np.uint32), plain["mse"].view(np.uint32))
        assert np.array_equal(nv["deq"].view(np.uint32) & 0x7FFFFFFF, plain["deq"].view(np.uint32) & 0x7FFFFFFF)


def test_selection_is_the_per_special_minimum(O):
    x = _x("razer_weight", 16, 256, seed=9)
    g = O.global_scale(O.amax(x), O.SF_E3M3)
    rz = O.razer_quantize(x, O.SF_E3M3, W_SPECIALS, g=g)
    single = np.stack([O.razer_quantize(x, O.SF_E3M3, [v], g=g)["mse"] for v in W_SPECIALS])
    sel = rz["meta"] >> 6
    # first index achieving the minimum
    expect = np.argmin(single, axis=0)
    assert np.array_equal(sel, expect)
    assert np.array_equal(rz["mse"], single.min(axis=0))


def test_plus_minus_five_is_the_best_pair(O):
    fact = json.load(open(GOLDEN))["razer_special_granularity"]
    assert fact["best_pair"] == [5.0, -5.0]
    for sf, kind in ((O.SF_E4M3, "razer_act"), (O.SF_E3M3, "razer_weight")):
        x = _x(kind, 256, 1024, seed=1)
        g = O.global_scale(O.amax(x), sf)
        tot = {v: O.razer_quantize(x, sf, [v, -v], g=g)["mse"].astype(np.float64).mean()
               for v in (2.5, 3.5, 4.5, 5.0, 5.5)}
        assert min(tot, key=tot.get) == 5.0


def _exact_razer_block(xb, S, v):
    """Exact rational SSE of one block under the RaZeR encode of section 2.2 as
    read here: each element takes the nearest E2M1 grid value (ties to the
    even code, saturating at 6) unless it has v's sign, the grid value is not
    zero, and |y| is strictly nearer to |v| than to the grid value -- then it
    takes v.  Written with Fractions, independent of the oracle's fp32 code."""
    from fractions import Fraction
    grid = [Fraction(g) for g in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]
    v = Fraction(v)
    tot = Fraction(0)
    for x in xb:
        xf = Fraction(float(x))
        y = xf / S
        ay = abs(y)
        m = 7 if ay >= 6 else min(range(8), key=lambda i: (abs(ay - grid[i]), i % 2))
        q = grid[m] * (1 if y >= 0 else -1)
        if m != 0 and (y > 0) == (v > 0) and abs(ay - abs(v)) < abs(ay - grid[m]):
            q = v
        tot += (xf - q * S) ** 2
    return tot


@pytest.mark.parametrize("sf,specials", [(0, A_SPECIALS), (1, W_SPECIALS)])
def test_selection_matches_exact_rational_search(O, sf, specials):
    """On tiny inputs whose scaled values are exact (g = 1, scale = block max / 6
    rounded to the format), the chosen special is the exact-arithmetic minimum
    over the table (ties to the earlier entry) and the reported MSE is its error."""
    from fractions import Fraction
    rng = np.random.default_rng(17 + sf)
    x = (rng.standard_normal((6, 16)) * 2.0).astype(np.float32)
    r = O.razer_quantize(x, sf, specials, g=1.0)
    val = O.e3m3_value if sf == 1 else O.e4m3_value
    for b in range(6):
        meta = int(r["meta"][b, 0])
        sel, code = (meta >> 6, meta & 0x3F) if sf == 1 else (meta >> 7, meta & 0x7F)
        S = Fraction(val(code))
        errs = [_exact_razer_block(x[b], S, v) for v in specials]
        best = min(errs)
        assert errs[sel] <= best * (1 + Fraction(1, 10 ** 5)) + Fraction(1, 10 ** 40), (b, sel, errs)
        assert abs(float(r["mse"][b, 0]) - float(errs[sel]) / 16) <= 1e-5 * float(errs[sel]) / 16 + 1e-30
