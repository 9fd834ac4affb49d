"""Pins for the oracle's dequantization (with per-block MSE) and W4A4 GEMM reference.

The dequantizer re-derives values from packed codes and scale bytes, a code
path separate from the quantizers; it must reproduce their fused outputs bit
for bit.  The GEMM reference (fp64 product of exactly decoded operands) is
checked against a plain triple loop over ml_dtypes-decoded operands.
"""
import ml_dtypes as md
import numpy as np
import pytest

from block_scaled_fp4_03_b200 import inputs


def _x(kind, rows, cols, seed=0):
    return inputs.as_f32(inputs.generate(kind, rows, cols, seed=seed))


@pytest.mark.parametrize("B", [4, 8, 16, 32])
@pytest.mark.parametrize("rule", [0, 1, 2, 3])
def test_dequant_reproduces_nvfp4(O, B, rule):
    x = _x("gaussian", 24, 128, seed=B + rule)
    g = O.global_scale(O.amax(x))
    q = O.nvfp4_quantize(x, B, rule, g=g)
    d = O.dequant_mse(q["codes"], q["scales"], 24, 128, B, O.SF_E4M3, None, g=g, ref=x)
    assert np.array_equal(d["deq"].view(np.uint32), q["deq"].view(np.uint32))
    assert np.array_equal(d["mse"].view(np.uint32), q["mse"].view(np.uint32))


@pytest.mark.parametrize("sf,kind,specials", [(1, "razer_weight", [5.0, -5.0, 3.5, -3.5]),
                                              (0, "razer_act", [5.0, -5.0])])
def test_dequant_reproduces_razer(O, sf, kind, specials):
    x = _x(kind, 24, 256, seed=sf)
    g = O.global_scale(O.amax(x), sf)
    q = O.razer_quantize(x, sf, specials, g=g)
    d = O.dequant_mse(q["codes"], q["meta"], 24, 256, 16, sf, specials, g=g, ref=x)
    assert np.array_equal(d["deq"].view(np.uint32), q["deq"].view(np.uint32))
    assert np.array_equal(d["mse"].view(np.uint32), q["mse"].view(np.uint32))


def test_dequant_reproduces_mxfp4(O):
    x = _x("mx_act", 24, 256, seed=1)
    t = inputs.positive_vector(256, seed=4)
    q = O.mxfp4_quantize(x, t, True, O.RULE_ABSMAX)
    y = O.mx_transform(x, t, True)
    d = O.dequant_mse(q["codes"], q["scales"], 24, 256, 32, O.SF_E8M0, None, ref=y)
    assert np.array_equal(d["deq"].view(np.uint32), q["deq"].view(np.uint32))
    assert np.array_equal(d["mse"].view(np.uint32), q["mse"].view(np.uint32))


def test_dequant_independent_decode(O):
    """deq = RN32(v * RN32(sc * g)) with v, sc decoded by ml_dtypes."""
    x = _x("gaussian", 8, 64, seed=3)
    g = O.global_scale(O.amax(x))
    q = O.nvfp4_quantize(x, 16, O.RULE_FOUR_OVER_SIX, g=g)
    lo, hi = q["codes"] & 0xF, q["codes"] >> 4
    c = np.empty((8, 64), np.uint8)
    c[:, 0::2], c[:, 1::2] = lo, hi
    v = c.view(md.float4_e2m1fn).astype(np.float32)
    S = (q["scales"].view(md.float8_e4m3fn).astype(np.float32) * np.float32(g)).astype(np.float32)
    deq = (v * np.repeat(S, 16, axis=1)).astype(np.float32)
    assert np.array_equal(deq.view(np.uint32), q["deq"].view(np.uint32))


def test_gemm_reference_matches_triple_loop(O):
    a = _x("gemm_act", 6, 64, seed=1)
    w = _x("gemm_weight", 5, 64, seed=1)
    ga = O.global_scale(O.amax(a))
    gw = O.global_scale(O.amax(w))
    qa = O.nvfp4_quantize(a, 16, O.RULE_FOUR_OVER_SIX, g=ga)
    qw = O.nvfp4_quantize(w, 16, O.RULE_ABSMAX, g=gw)
    ref = O.gemm_ref(qa["codes"], qa["scales"], ga, qw["codes"], qw["scales"], gw)

    def decode(q, rows):
        c = np.empty((rows, 64), np.uint8)
        c[:, 0::2], c[:, 1::2] = q["codes"] & 0xF, q["codes"] >> 4
        v = c.view(md.float4_e2m1fn).astype(np.float64)
        s = q["scales"].view(md.float8_e4m3fn).astype(np.float64)
        return v, s

    va, sa = decode(qa, 6)
    vw, sw = decode(qw, 5)
    for m in range(6):
        for n in range(5):
            acc = 0.0
            for k in range(64):
                acc += (va[m, k] * sa[m, k // 16]) * (vw[n, k] * sw[n, k // 16])
            assert abs(ref[m, n] - float(ga) * float(gw) * acc) <= 1e-12 * max(1.0, abs(ref[m, n]))
    # and it approximates the unquantized product at FP4 accuracy
    exact = a.astype(np.float64) @ w.astype(np.float64).T
    assert np.linalg.norm(ref - exact) <= 0.2 * np.linalg.norm(exact)
    sub = O.gemm_ref(qa["codes"], qa["scales"], ga, qw["codes"], qw["scales"], gw,
                     rows=np.array([1, 4]), cols=np.array([0, 3]))
    assert np.array_equal(sub, ref[np.ix_([1, 4], [0, 3])])


@pytest.mark.parametrize("sf,kind,specials", [(1, "razer_weight", [5.0, -5.0, 3.5, -3.5]),
                                              (0, "razer_act", [5.0, -5.0])])
def test_razer_decode_exact_matches_quantizer(O, sf, kind, specials):
    """With g = 1 every RaZeR value v * sc is exact in fp32, so the exact decode
    equals the quantizer's own fused dequantization (separate C code path)."""
    x = _x(kind, 16, 256, seed=7 + sf)
    q = O.razer_quantize(x, sf, specials, g=1.0)
    d = O.razer_decode_exact(q["codes"], q["meta"], sf, specials)
    assert np.array_equal(d, q["deq"].astype(np.float64))
    lo, hi = q["codes"] & 0xF, q["codes"] >> 4
    assert ((lo == 8) | (hi == 8)).any()           # specials do occur


def test_razer_gemm_reference_matches_triple_loop(O):
    a = _x("razer_act", 6, 64, seed=2)
    w = _x("razer_weight", 5, 64, seed=2)
    spa, spw = [5.0, -5.0], [5.0, -5.0, 3.5, -3.5]
    ga = O.global_scale(O.amax(a), O.SF_E4M3)
    gw = O.global_scale(O.amax(w), O.SF_E3M3)
    qa = O.razer_quantize(a, O.SF_E4M3, spa, g=ga)
    qw = O.razer_quantize(w, O.SF_E3M3, spw, g=gw)
    ref = O.gemm_values(O.razer_decode_exact(qa["codes"], qa["meta"], O.SF_E4M3, spa),
                        O.razer_decode_exact(qw["codes"], qw["meta"], O.SF_E3M3, spw), ga, gw)
    # operand values from the C dequantizer at g = 1 (exact v * sc)
    va = O.dequant_mse(qa["codes"], qa["meta"], 6, 64, 16, O.SF_E4M3, spa)["deq"].astype(np.float64)
    vw = O.dequant_mse(qw["codes"], qw["meta"], 5, 64, 16, O.SF_E3M3, spw)["deq"].astype(np.float64)
    for m in range(6):
        for n in range(5):
            acc = 0.0
            for k in range(64):
                acc += va[m, k] * vw[n, k]
            assert abs(ref[m, n] - float(ga) * float(gw) * acc) <= 1e-12 * max(1.0, abs(ref[m, n]))
    exact = a.astype(np.float64) @ w.astype(np.float64).T
    assert np.linalg.norm(ref - exact) <= 0.2 * np.linalg.norm(exact)


def test_mx_decode_exact_matches_dequantizer(O):
    """v * 2^e is exact in fp32 here, so the fp64 decode equals the C
    dequantizer's E8M0 output; and the MX product of the transformed operands
    approximates X W^T (the rotation and 1/t cancel)."""
    x = _x("mx_act", 64, 256, seed=5)
    w = _x("mx_weight", 48, 256, seed=6)
    t = inputs.positive_vector(256, seed=7)
    qa = O.mxfp4_quantize(x, t, True, O.RULE_ABSMAX)
    d = O.mx_decode_exact(qa["codes"], qa["scales"])
    deq = O.dequant_mse(qa["codes"], qa["scales"], 64, 256, 32, O.SF_E8M0, None)["deq"]
    assert np.array_equal(d, deq.astype(np.float64))
    tinv = (1.0 / t.astype(np.float64)).astype(np.float32)
    qw = O.mxfp4_quantize(w, tinv, True, O.RULE_ABSMAX)
    ref = O.gemm_values(d, O.mx_decode_exact(qw["codes"], qw["scales"]), 1.0, 1.0)
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    e_ref = np.linalg.norm(ref - exact) / np.linalg.norm(exact)
    # without the matching 1/t on the weights the product is far off (t spans
    # [1/4, 4], which also makes 4-bit blocks coarse: e_ref is about 0.46)
    qw_bad = O.mxfp4_quantize(w, None, True, O.RULE_ABSMAX)
    bad = O.gemm_values(d, O.mx_decode_exact(qw_bad["codes"], qw_bad["scales"]), 1.0, 1.0)
    e_bad = np.linalg.norm(bad - exact) / np.linalg.norm(exact)
    assert e_ref <= 0.6 and e_bad >= 2 * e_ref, (e_ref, e_bad)
