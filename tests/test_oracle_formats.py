"""Pins for the oracle's number formats (E2M1, E4M3, E3M3, E8M0) and global scale.

Each check compares the C oracle with something that is not the oracle: the
value set the pages print, ml_dtypes' independent implementations of the OCP
formats, and exact rational nearest-value search.
"""
import json
import os
from fractions import Fraction

import ml_dtypes as md
import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def facts():
    with open(GOLDEN) as f:
        return json.load(f)


def nearest_even(r, grid):
    """Exact nearest of r in ascending `grid` (Fractions), ties to the even index, saturating."""
    if np.isinf(r):
        return len(grid) - 1
    r = Fraction(r)
    if r >= grid[-1]:
        return len(grid) - 1
    best = None
    for i, g in enumerate(grid):
        d = abs(r - g)
        if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
            best = (d, i)
    return best[1]


def test_e2m1_value_set_is_the_pages(O):
    printed = facts()["e2m1_values"]["values"]
    vals = [O.e2m1_value(c) for c in range(16)]
    assert sorted(set(vals)) == sorted(set(printed))
    # sign-magnitude: both zeros exist, codes 0 and 8
    assert np.signbit(vals[0]) == False and np.signbit(vals[8]) == True and vals[8] == 0.0
    assert len(vals) == 16


def test_e2m1_decode_matches_ml_dtypes(O):
    ref = np.arange(16, dtype=np.uint8)
    # ml_dtypes packs one e2m1 per byte (low nibble)
    dec = ref.view(md.float4_e2m1fn).astype(np.float32)
    ours = np.array([O.e2m1_value(c) for c in range(16)], np.float32)
    assert np.array_equal(dec.view(np.uint32), ours.view(np.uint32))


def test_e2m1_encode_matches_ml_dtypes(O):
    rng = np.random.default_rng(1)
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    vals = np.concatenate([
        ties, -ties, np.nextafter(ties, np.float32(0)), np.nextafter(ties, np.float32(10)),
        np.array([0.0, -0.0, 6.0, -6.0, 7.0, 1e30, -1e30, np.inf, -np.inf, 1e-40, -1e-40], np.float32),
        rng.standard_normal(2000).astype(np.float32) * 3,
        (rng.uniform(-8, 8, 2000)).astype(np.float32),
    ]).astype(np.float32)
    ref = vals.astype(md.float4_e2m1fn).view(np.uint8) & 0xF
    ours = np.array([O.e2m1_encode(v) for v in vals], np.uint8)
    assert np.array_equal(ref, ours)


def test_e2m1_ties_go_to_even(O):
    # hand list: tie -> neighbour with the even magnitude index
    expect = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for t, v in expect.items():
        assert O.e2m1_value(O.e2m1_encode(t)) == v
        assert O.e2m1_value(O.e2m1_encode(-t)) == -v


def test_e4m3_table_matches_ml_dtypes(O):
    codes = np.arange(0x7F, dtype=np.uint8)
    ref = codes.view(md.float8_e4m3fn).astype(np.float64)
    ours = np.array([O.e4m3_value(int(c)) for c in codes])
    assert np.array_equal(ref, ours)
    pos = ours[1:]
    assert len(pos) == 126 and np.all(np.diff(pos) > 0)
    assert pos[0] == 2.0 ** -9 and pos[-1] == 448.0


def test_e4m3_encode_nearest_even_and_saturating(O):
    rng = np.random.default_rng(2)
    grid = [O.e4m3_value(c) for c in range(0x7F)]
    mids = [(grid[i] + grid[i + 1]) / 2 for i in range(len(grid) - 1)]
    vals = np.concatenate([
        np.array(grid, np.float32), np.array(mids, np.float32),
        np.exp(rng.uniform(np.log(1e-5), np.log(500), 3000)).astype(np.float32),
        np.array([0.0, 1e-30, 448.0, 449.0, 464.0, 480.0, 1e9, np.inf], np.float32),
    ])
    fr = [Fraction(g) for g in grid]
    for v in vals:
        c = O.e4m3_encode(float(v))
        assert c == nearest_even(float(v), fr), v
    # ml_dtypes agrees below the saturation point (its cast gives NaN above 448)
    small = vals[vals <= 448].astype(np.float32)
    ref = small.astype(md.float8_e4m3fn).view(np.uint8)
    ours = np.array([O.e4m3_encode(float(v)) for v in small], np.uint8)
    assert np.array_equal(ref, ours)


def test_e3m3_is_the_coarse_subset_of_e4m3(O):
    vals = [O.e3m3_value(c) for c in range(64)]
    assert vals[0] == 0.0 and len(set(vals)) == 64 and np.all(np.diff(vals) > 0)
    e4 = [O.e4m3_value(c) for c in range(1, 0x7F)]
    # E3M3 (3 exponent bits, 3 mantissa bits, 6 bits in all) has exactly the
    # E4M3 values from 2^-5 to 30 that are multiples of 2^-5.
    subset = [v for v in e4 if 2.0 ** -5 <= v <= 30.0 and (v * 32.0) == int(v * 32.0)]
    assert vals[1:] == subset
    assert vals[1] == 2.0 ** -5 and vals[-1] == 30.0


def test_e3m3_encode_nearest_even(O):
    rng = np.random.default_rng(3)
    grid = [O.e3m3_value(c) for c in range(64)]
    fr = [Fraction(g) for g in grid]
    mids = [(grid[i] + grid[i + 1]) / 2 for i in range(63)]
    vals = np.concatenate([np.array(grid + mids, np.float32),
                           np.exp(rng.uniform(np.log(1e-4), np.log(40), 3000)).astype(np.float32),
                           np.array([0.0, 31.0, 32.0, 1e9], np.float32)])
    for v in vals:
        assert O.e3m3_encode(float(v)) == nearest_even(float(v), fr), v


def test_e8m0_matches_ml_dtypes(O):
    b = np.arange(255, dtype=np.uint8)
    ref = b.view(md.float8_e8m0fnu).astype(np.float64)
    ours = np.array([O.e8m0_value(int(x)) for x in b])
    assert np.array_equal(ref, ours)


def test_global_scale_closed_form(O):
    assert O.global_scale(2688.0, O.SF_E4M3) == np.float32(1.0)
    assert O.global_scale(180.0, O.SF_E3M3) == np.float32(1.0)
    assert O.global_scale(0.0) == np.float32(1.0)
    assert O.global_scale(1.0) == np.float32(1.0) / np.float32(2688.0)
    assert O.global_scale(5376.0) == np.float32(2.0)


def test_amax(O):
    x = np.array([[1.0, -7.5, 3.0, 0.0]], np.float32)
    assert O.amax(x) == np.float32(7.5)
    assert O.amax(np.zeros((2, 4), np.float32)) == 0.0
