"""Pins for the oracle's MXFP4 path: online scale, block-Hadamard, E8M0
exponent, Hessian-weighted exponent choice, Hessian blocks and channel scale.

MACaQ review, section 1 (MXFP4 = E2M1 + one E8M0 scale per 32 elements; the
online per-channel scale D and size-32 block-Hadamard B, with W D^-1 B on
the weight side; the exponent chosen among the standard one plus
{+1, 0, -1} by the H = X^T X weighted error) and section 3 (alpha = 0.75,
rms from the Hessian diagonal).
"""
import ml_dtypes as md
import numpy as np

from block_scaled_fp4_03_b200 import inputs


def sylvester(n):
    h = np.array([[1]], np.int64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def _x(kind, rows, cols, seed=0):
    return inputs.as_f32(inputs.generate(kind, rows, cols, seed=seed))


def test_hadamard_is_orthogonal_and_matches_dense(O):
    H = sylvester(32)
    assert np.array_equal(H.T @ H, 32 * np.eye(32, dtype=np.int64))
    x = _x("mx_act", 64, 256, seed=1)
    y = O.mx_transform(x, None, True).astype(np.float64)
    dense = np.concatenate([x[:, k:k + 32].astype(np.float64) @ H.T / np.sqrt(32.0)
                            for k in range(0, 256, 32)], axis=1)
    assert np.abs(y - dense).max() <= 1e-6 * np.abs(dense).max()
    nx = np.linalg.norm(x.astype(np.float64).reshape(64, -1, 32), axis=-1)
    ny = np.linalg.norm(y.reshape(64, -1, 32), axis=-1)
    np.testing.assert_allclose(ny, nx, rtol=1e-6)
    # a unit vector maps to a column of H / sqrt(32)
    e = np.zeros((1, 32), np.float32)
    e[0, 5] = 1
    col = O.mx_transform(e, None, True)[0].astype(np.float64)
    np.testing.assert_allclose(col, H[:, 5] / np.sqrt(32.0), rtol=1e-7)


def test_channel_scale_applies_before_rotation(O):
    x = _x("mx_act", 8, 128, seed=2)
    t = inputs.positive_vector(128, seed=1)
    a = O.mx_transform(x, t, True)
    b = O.mx_transform((x * t).astype(np.float32), None, True)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert np.array_equal(O.mx_transform(x, t, False), (x * t).astype(np.float32))


def test_standard_exponent_puts_block_max_in_4_to_8(O):
    x = _x("mx_act", 64, 512, seed=3)
    r = O.mxfp4_quantize(x, None, True, O.RULE_ABSMAX)
    y = O.mx_transform(x, None, True)
    a = np.abs(y).reshape(64, -1, 32).max(-1).astype(np.float64)
    e = r["scales"].astype(np.int64) - 127
    q = a * np.exp2(-e.astype(np.float64))
    assert np.all((q >= 4) & (q < 8))
    # scale bytes decode through ml_dtypes' E8M0
    sv = r["scales"].view(md.float8_e8m0fnu).astype(np.float64)
    np.testing.assert_array_equal(sv, np.exp2(e.astype(np.float64)))


def test_mx_codes_match_independent_encode(O):
    x = _x("mx_act", 16, 256, seed=4)
    t = inputs.positive_vector(256, seed=2)
    r = O.mxfp4_quantize(x, t, True, O.RULE_ABSMAX)
    y = O.mx_transform(x, t, True)
    e = r["scales"].astype(np.int64) - 127
    q = (y.reshape(16, -1, 32).astype(np.float64) * np.exp2(-e)[..., None]).astype(np.float32).reshape(16, -1)
    c = q.astype(md.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal((c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8), r["codes"])
    v = c.view(md.float4_e2m1fn).astype(np.float64).reshape(16, -1, 32)
    deq = (v * np.exp2(e)[..., None]).reshape(16, -1)
    np.testing.assert_array_equal(r["deq"].astype(np.float64), deq)


def test_all_zero_block_and_clamp(O):
    x = np.zeros((2, 32), np.float32)
    x[1, 0] = 1e-39   # subnormal: exponent clamps to -127
    r = O.mxfp4_quantize(x, None, False, O.RULE_ABSMAX)
    assert r["scales"][0, 0] == 0 and r["scales"][1, 0] == 0
    assert np.all(r["mse"][0] == 0)


def _fp64_block_sse(y, e):
    q = (y.astype(np.float64) * 2.0 ** (-e)).astype(np.float32)
    v = q.astype(md.float4_e2m1fn).astype(np.float64)
    return ((y.astype(np.float64) - v * 2.0 ** e) ** 2).sum()


def test_hessian_identity_is_min_sse_over_offsets(O):
    x = _x("mx_weight", 64, 256, seed=5)
    kb = 256 // 32
    hess = np.tile(np.eye(32, dtype=np.float32), (kb, 1, 1))
    r = O.mxfp4_quantize(x, None, True, O.RULE_HESSIAN_EXP, hess)
    std = O.mxfp4_quantize(x, None, True, O.RULE_ABSMAX)
    y = O.mx_transform(x, None, True)
    e_chosen = r["scales"].astype(np.int64) - 127
    e0 = std["scales"].astype(np.int64) - 127
    moved = 0
    for i in range(64):
        for k in range(kb):
            yb = y[i, 32 * k:32 * (k + 1)]
            cands = [e0[i, k] + o for o in (0, 1, -1)]
            sses = [_fp64_block_sse(yb, int(ec)) for ec in cands]
            best = int(np.argmin(sses))
            srt = sorted(sses)
            if srt[1] - srt[0] > 1e-6 * max(srt[0], 1e-30):
                assert e_chosen[i, k] == cands[best]
            moved += e_chosen[i, k] != e0[i, k]
    assert moved > 0
    # with identity weighting the oracle's choice never has a higher error than the standard one
    assert np.all(r["mse"] <= std["mse"])


def test_hessian_weighted_choice_minimises_the_quadratic_form(O):
    x = _x("mx_weight", 32, 128, seed=6)
    act = _x("mx_act", 512, 128, seed=6)
    hess = O.hessian_blocks(act, None, True).astype(np.float32)
    r = O.mxfp4_quantize(x, None, True, O.RULE_HESSIAN_EXP, hess)
    std = O.mxfp4_quantize(x, None, True, O.RULE_ABSMAX)
    y = O.mx_transform(x, None, True).astype(np.float64)
    H = hess.astype(np.float64)

    def cost(deq):
        d = (y - deq.astype(np.float64)).reshape(32, -1, 32)
        return np.einsum("rki,kij,rkj->rk", d, H, d)

    c_h, c_s = cost(r["deq"]), cost(std["deq"])
    assert np.all(c_h <= c_s * (1 + 1e-5) + 1e-12)
    assert c_h.sum() < c_s.sum()
    e_h = r["scales"].astype(np.int64) - std["scales"].astype(np.int64)
    assert set(np.unique(e_h)) <= {-1, 0, 1}


def test_hessian_blocks_match_brute_force(O):
    x = _x("mx_act", 40, 64, seed=7)
    t = inputs.positive_vector(64, seed=3)
    hb = O.hessian_blocks(x, t, True)
    y = O.mx_transform(x, t, True).astype(np.float64)
    for k in range(2):
        for i in (0, 7, 31):
            for j in (0, 13, 31):
                s = sum(y[n, 32 * k + i] * y[n, 32 * k + j] for n in range(40))
                assert abs(hb[k, i, j] - s) <= 1e-12 * max(1.0, abs(s))
    assert np.allclose(hb, np.transpose(hb, (0, 2, 1)))
    assert np.all(np.linalg.eigvalsh(hb) > -1e-9 * np.abs(hb).max())


def test_channel_scale_closed_form(O):
    # activations with constant columns c_j -> rms_j = |c_j|; weights whose column j
    # alternates +-s_j -> population std s_j.  t_j = (s_j / |c_j|)^0.75.
    c = np.array([1.0, 2.0, 0.5, 4.0], np.float32)
    s = np.array([0.02, 0.08, 0.01, 0.0], np.float32)
    x = np.tile(c, (6, 1))
    w = np.stack([s, -s, s, -s])
    t, ti = O.channel_scale(x, w, 0.75)
    expect = np.array([(0.02 / 1.0) ** 0.75, (0.08 / 2.0) ** 0.75, (0.01 / 0.5) ** 0.75, 1.0], np.float32)
    np.testing.assert_allclose(t, expect, rtol=1e-6)
    assert np.array_equal(ti, np.float32(1) / t)


def test_transform_preserves_the_layer_product(O):
    """X' W'^T = X W^T with X' = X D B and W' = W D^-1 B (before quantization)."""
    x = _x("mx_act", 64, 128, seed=8)
    w = _x("mx_weight", 48, 128, seed=8)
    t, ti = O.channel_scale(x, w, 0.75)
    xp = O.mx_transform(x, t, True).astype(np.float64)
    wp = O.mx_transform(w, ti, True).astype(np.float64)
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    got = xp @ wp.T
    assert np.linalg.norm(got - ref) <= 1e-5 * np.linalg.norm(ref)
