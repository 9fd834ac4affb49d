"""Pins for the oracle's Flip-Refinement ("MACaQ" review, section 1 Key Terms
and section 3 Method): greedy moves of single MXFP4 codes to a neighbouring
E2M1 level, chosen per output row by the largest closed-form decrease of the
Hessian-weighted reconstruction error.

The checks below do not reuse the gain formula: they measure the objective
sum_k d_k^T H'_k d_k directly in fp64 on the codes the oracle returns, and
search every single move by brute force."""
import numpy as np
import pytest

from block_scaled_fp4_03_b200 import inputs

# E2M1 values by code, the printed magnitude set with the sign bit
MAG = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
VALUE = np.concatenate([MAG, -MAG])
# the ladder of distinct values in increasing order
LADDER = np.array([-6, -4, -3, -2, -1.5, -1, -0.5, 0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def unpack(codes, cols):
    c = np.empty((codes.shape[0], cols), np.int64)
    c[:, 0::2] = codes & 15
    c[:, 1::2] = codes >> 4
    return c


def objective(u, c, scales, hess):
    """sum over blocks of d^T H d per row, fp64, d = u - value(code) * 2^e."""
    rows, cols = u.shape
    e = scales.astype(np.int64) - 127
    deq = VALUE[c] * np.exp2(np.repeat(e, 32, axis=1).astype(np.float64))
    d = (u.astype(np.float64) - deq).reshape(rows, cols // 32, 32)
    H = hess.astype(np.float64)
    return np.einsum("rki,kij,rkj->r", d, H, d)


def neighbours(code):
    v = VALUE[code]
    i = int(np.argmin(np.abs(LADDER - v)))
    return [LADDER[j] for j in (i - 1, i + 1) if 0 <= j < len(LADDER)]


def layer(O, rows, cols, seed):
    w = inputs.as_f32(inputs.generate("mx_weight", rows, cols, seed=seed))
    x = inputs.as_f32(inputs.generate("mx_act", 256, cols, seed=seed + 1))
    t, ti = O.channel_scale(x, w, 0.75)
    hess = O.hessian_blocks(x, t, True).astype(np.float32)
    q = O.mxfp4_quantize(w, ti, True, O.RULE_HESSIAN_EXP, hess)
    u = O.mx_transform(w, ti, True)
    return w, ti, hess, q, u


def test_identity_hessian_keeps_round_to_nearest(O):
    """With H'_k = I every element's error is independent and the nearest level
    is optimal: no move can gain, so the codes come back unchanged."""
    w = inputs.as_f32(inputs.generate("mx_weight", 16, 128, seed=4))
    q = O.mxfp4_quantize(w, None, True, O.RULE_ABSMAX)
    eye = np.tile(np.eye(32, dtype=np.float32)[None] * 3.0, (4, 1, 1))
    c, moves = O.mxfp4_flip_refine(w, None, True, eye, q["codes"], q["scales"], 64)
    assert np.all(moves == 0)
    assert np.array_equal(c, q["codes"])


def test_zero_moves_is_identity(O):
    w, ti, hess, q, u = layer(O, 4, 64, seed=1)
    c, moves = O.mxfp4_flip_refine(w, ti, True, hess, q["codes"], q["scales"], 0)
    assert np.all(moves == 0) and np.array_equal(c, q["codes"])


def test_each_move_is_the_best_single_move(O):
    """Brute force: from the codes after m moves, the (m+1)-th accepted move is
    the single neighbouring-level change with the largest fp64 decrease of
    the objective, and that decrease is positive."""
    w, ti, hess, q, u = layer(O, 3, 64, seed=2)
    cols = 64
    prev = q["codes"]
    for m in range(1, 7):
        cur, moves = O.mxfp4_flip_refine(w, ti, True, hess, q["codes"], q["scales"], m)
        cp, cc = unpack(prev, cols), unpack(cur, cols)
        f_prev = objective(u, cp, q["scales"], hess)
        for r in range(3):
            diff = np.nonzero(VALUE[cp[r]] != VALUE[cc[r]])[0]
            if moves[r] < m:            # the row had stopped: nothing changed
                assert diff.size == 0
                continue
            assert diff.size == 1, (m, r, diff)
            i = diff[0]
            # every candidate single move, measured exactly
            best = -np.inf
            for j in range(cols):
                for v in neighbours(cp[r, j]):
                    trial = cp[r].copy()
                    trial[j] = int(np.nonzero(VALUE == v)[0][0])
                    dec = f_prev[r] - objective(u[r:r + 1], trial[None], q["scales"][r:r + 1], hess)[0]
                    best = max(best, dec)
            got = f_prev[r] - objective(u[r:r + 1], cc[r][None], q["scales"][r:r + 1], hess)[0]
            scale = max(1e-30, abs(f_prev[r]))
            assert got > 0
            assert got >= best - 1e-5 * scale, (m, r, i, got, best)
            # a single neighbouring-level step
            assert VALUE[cc[r, i]] in neighbours(cp[r, i])
        prev = cur


def test_objective_decreases_and_stops_at_a_local_minimum(O):
    w, ti, hess, q, u = layer(O, 6, 96, seed=3)
    c0 = unpack(q["codes"], 96)
    f0 = objective(u, c0, q["scales"], hess)
    c, moves = O.mxfp4_flip_refine(w, ti, True, hess, q["codes"], q["scales"], 100000)
    cu = unpack(c, 96)
    f1 = objective(u, cu, q["scales"], hess)
    assert np.all(f1 <= f0 + 1e-9 * np.abs(f0))
    assert np.any(f1 < f0)
    assert np.all(moves < 100000)
    # local minimum: no single neighbouring move decreases f by more than rounding
    for r in range(6):
        for j in range(96):
            for v in neighbours(cu[r, j]):
                trial = cu[r].copy()
                trial[j] = int(np.nonzero(VALUE == v)[0][0])
                fr = objective(u[r:r + 1], trial[None], q["scales"][r:r + 1], hess)[0]
                assert fr >= f1[r] - 1e-5 * abs(f1[r])


@pytest.mark.parametrize("K", [1, 5, 40])
def test_move_budget_and_code_validity(O, K):
    w, ti, hess, q, u = layer(O, 8, 128, seed=5)
    c, moves = O.mxfp4_flip_refine(w, ti, True, hess, q["codes"], q["scales"], K)
    assert np.all(moves <= K) and np.all(moves >= 0)
    cu, c0 = unpack(c, 128), unpack(q["codes"], 128)
    changed = (VALUE[cu] != VALUE[c0]).sum(axis=1)
    assert np.all(changed <= moves)
    # a changed element sits at most `moves` ladder steps from its start
    lad = lambda v: np.searchsorted(LADDER, v)
    steps = np.abs(lad(VALUE[cu]) - lad(VALUE[c0])).sum(axis=1)
    assert np.all(steps <= moves) and np.all(steps % 2 == moves % 2)
