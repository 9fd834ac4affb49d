"""GPU parity: the CUDA library against the CPU oracle, element by element.

Codes, scale bytes, dequantized values, block MSE and global scales must be
bit-identical (the decisions are fp32 sequences fixed by the definition);
Hessian blocks and the channel scale are fp32/fp64 reductions compared within
a stated tolerance.  Small cases span several CUDA blocks with a ragged tail;
full-size cases (the benchmark workloads, in the benchmark's launch
configuration) are checked on sampled rows, which the oracle computes alone
because blocks are independent.
"""
import numpy as np
import pytest
import torch

from block_scaled_fp4_03_b200 import binding as fq
from block_scaled_fp4_03_b200 import inputs

pytestmark = pytest.mark.gpu


def dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def host(t):
    return t.detach().cpu().numpy()


def bits(a):
    a = np.ascontiguousarray(a)
    return a.view(np.uint32) if a.dtype == np.float32 else a


def assert_bits(got, exp, what):
    g, e = bits(host(got) if torch.is_tensor(got) else got), bits(exp)
    assert g.shape == e.shape, (what, g.shape, e.shape)
    bad = np.argwhere(g != e)
    assert bad.size == 0, "%s: %d mismatches, first at %s: gpu %r oracle %r" % (
        what, len(bad), bad[0], g[tuple(bad[0])], e[tuple(bad[0])])


def make(kind, rows, cols, seed, dtype):
    """Input in the requested storage type: returns (device tensor, fp32 numpy for the oracle)."""
    a = inputs.generate(kind, rows, cols, seed=seed)
    f32 = inputs.as_f32(a)
    if dtype == "bf16":
        b = inputs.f32_to_bf16_bits(f32) if a.dtype != np.uint16 else a
        return dev(b), inputs.bf16_bits_to_f32(b)
    return dev(f32), f32


RULES = [fq.ABSMAX, fq.PREVENT_ZERO, fq.FOUR_OVER_SIX, fq.BRUTE_FORCE]


def oracle_g(O, x32, gs_mode, sf=0, given=None):
    if gs_mode == fq.GS_NONE:
        return np.float32(1.0)
    if gs_mode == fq.GS_GIVEN:
        return np.float32(given)
    return O.global_scale(O.amax(x32), sf)


# ------------------------------------------------------------------ NVFP4
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("rule", RULES)
@pytest.mark.parametrize("B", [4, 8, 16, 32])
@pytest.mark.parametrize("gs_mode", [fq.GS_NONE, fq.GS_AMAX, fq.GS_GIVEN])
def test_nvfp4_small(O, B, rule, dtype, gs_mode):
    kind = "student_t" if gs_mode == fq.GS_NONE else "gaussian"
    x, x32 = make(kind, 67, 320, seed=B * 10 + rule, dtype=dtype)
    given = torch.tensor([0.0123], dtype=torch.float32, device="cuda")
    r = fq.nvfp4_quantize(x, block=B, rule=rule, gs_mode=gs_mode,
                          global_scale=given if gs_mode == fq.GS_GIVEN else None,
                          dequant=True, mse=True)
    torch.cuda.synchronize()
    g = oracle_g(O, x32, gs_mode, given=np.float32(0.0123))
    if gs_mode == fq.GS_AMAX:
        assert_bits(r["global_scale"], np.array([g], np.float32), "global scale")
    ref = O.nvfp4_quantize(x32, B, rule, g=g)
    assert_bits(r["codes"], ref["codes"], "codes")
    assert_bits(r["scales"], ref["scales"], "scales")
    assert_bits(r["dequant"], ref["deq"], "dequant")
    assert_bits(r["mse"], ref["mse"], "mse")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("rule", RULES)
@pytest.mark.parametrize("B", [4, 8, 16, 32])
@pytest.mark.parametrize("gs_mode", [fq.GS_NONE, fq.GS_AMAX])
def test_ue5m3_small(O, B, rule, dtype, gs_mode):
    """The same rules with UE5M3 block scales (fp4_block_quantize)."""
    kind = "student_t" if gs_mode == fq.GS_NONE else "gaussian"
    x, x32 = make(kind, 67, 320, seed=B * 10 + rule + 5, dtype=dtype)
    r = fq.nvfp4_quantize(x, block=B, rule=rule, gs_mode=gs_mode, dequant=True, mse=True,
                          scale_fmt=fq.SF_UE5M3)
    torch.cuda.synchronize()
    g = np.float32(1.0) if gs_mode == fq.GS_NONE else O.global_scale(O.amax(x32), O.SF_UE5M3)
    if gs_mode == fq.GS_AMAX:
        assert_bits(r["global_scale"], np.array([g], np.float32), "global scale")
    ref = O.block_fp4_quantize(x32, B, rule, O.SF_UE5M3, g=g)
    assert_bits(r["codes"], ref["codes"], "codes")
    assert_bits(r["scales"], ref["scales"], "scales")
    assert_bits(r["dequant"], ref["deq"], "dequant")
    assert_bits(r["mse"], ref["mse"], "mse")


def test_ue5m3_edge_values(O):
    """Scales at the ends of the UE5M3 range: tiny blocks (subnormal scales),
    huge blocks (saturation), zeros, and midpoints between scale values."""
    rng = np.random.default_rng(5)
    x32 = (rng.standard_normal((8, 64)) * np.float32(1e-5)).astype(np.float32)
    x32[1] *= np.float32(1e-3)
    x32[2] = 0
    x32[3] *= np.float32(3e10)
    x32[4, :16] = np.float32(6 * 1.0625)      # a/6 at the midpoint between 1 and 1.125
    for rule in RULES:
        r = fq.nvfp4_quantize(dev(x32), block=16, rule=rule, gs_mode=fq.GS_NONE, dequant=True, mse=True,
                              scale_fmt=fq.SF_UE5M3)
        torch.cuda.synchronize()
        ref = O.block_fp4_quantize(x32, 16, rule, O.SF_UE5M3, g=1.0)
        for k, rk in (("codes", "codes"), ("scales", "scales"), ("dequant", "deq"), ("mse", "mse")):
            assert_bits(r[k], ref[rk], "%s rule=%d" % (k, rule))


def test_dequant_ue5m3(O):
    x, x32 = make("student_t", 33, 128, seed=4, dtype="f32")
    q = O.block_fp4_quantize(x32, 16, O.RULE_FOUR_OVER_SIX, O.SF_UE5M3, g=1.0)
    r = fq.dequant_mse(dev(q["codes"]), dev(q["scales"]), 33, 128, 16, fq.SF_UE5M3, None, None, ref=x)
    torch.cuda.synchronize()
    assert_bits(r["dequant"], q["deq"], "dequant")
    assert_bits(r["mse"], q["mse"], "mse")


def test_nvfp4_mma_scale_layout(O):
    x, x32 = make("gemm_act", 256, 512, seed=3, dtype="bf16")
    rm = fq.nvfp4_quantize(x, 16, fq.FOUR_OVER_SIX)
    mm = fq.nvfp4_quantize(x, 16, fq.FOUR_OVER_SIX, sf_layout=fq.SF_MMA)
    torch.cuda.synchronize()
    assert_bits(mm["codes"], host(rm["codes"]), "codes")
    s_rm = host(rm["scales"])
    s_mm = host(mm["scales"]).reshape(-1)
    rows, kb = s_rm.shape
    r = np.arange(rows)[:, None]
    c = np.arange(kb)[None, :]
    off = ((r // 128) * (kb // 4) + c // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + c % 4
    assert_bits(s_mm[off], s_rm, "MMA-layout scales")


@pytest.mark.parametrize("rule", RULES)
def test_nvfp4_edge_values(O, rule):
    rng = np.random.default_rng(11)
    x32 = np.zeros((5, 64), np.float32)
    x32[1] = rng.standard_normal(64) * 1e30          # saturating scales
    x32[2] = rng.standard_normal(64) * 1e-38         # subnormal-range inputs
    x32[3, ::2] = -0.0
    x32[3, 1::2] = 6.0 * 2.0 ** -9                   # exactly representable at the smallest scale
    x32[4] = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 8)  # E2M1 ties
    for gs_mode in (fq.GS_NONE, fq.GS_AMAX):
        for B in (4, 16, 32):
            r = fq.nvfp4_quantize(dev(x32), B, rule, gs_mode=gs_mode, dequant=True, mse=True)
            torch.cuda.synchronize()
            g = oracle_g(O, x32, gs_mode)
            ref = O.nvfp4_quantize(x32, B, rule, g=g)
            for k, rk in (("codes", "codes"), ("scales", "scales"), ("dequant", "deq"), ("mse", "mse")):
                assert_bits(r[k], ref[rk], "%s B=%d gs=%d" % (k, B, gs_mode))


def test_nvfp4_empty_and_zero(O):
    z = torch.zeros((0, 64), dtype=torch.float32, device="cuda")
    r = fq.nvfp4_quantize(z, 16, fq.ABSMAX, gs_mode=fq.GS_AMAX)
    torch.cuda.synchronize()
    assert r["codes"].numel() == 0 and host(r["global_scale"])[0] == 1.0
    x = torch.zeros((3, 64), dtype=torch.float32, device="cuda")
    r = fq.nvfp4_quantize(x, 16, fq.BRUTE_FORCE, gs_mode=fq.GS_AMAX, dequant=True, mse=True)
    torch.cuda.synchronize()
    ref = O.nvfp4_quantize(np.zeros((3, 64), np.float32), 16, O.RULE_BRUTE_FORCE, g=1.0)
    assert_bits(r["scales"], ref["scales"], "scales")
    assert np.all(host(r["mse"]) == 0) and np.all(host(r["codes"]) == 0)


def test_brute_force_evaluation_counter(O):
    """The evaluation count a brute-force call adds to its workspace counter:
    at least the one seed per block, at most all 126 codes plus the all-zero
    candidate per block, identical across repeated calls, and added to
    (not reset) by each call."""
    x, x32 = make("student_t", 96, 512, seed=3, dtype="f32")
    ws = torch.zeros(fq.workspace_size(fq.OP_QUANTIZE, 1, 1), dtype=torch.uint8, device="cuda")
    counts = []
    for B in (4, 16):
        ws.zero_()
        r = fq.nvfp4_quantize(x, B, fq.BRUTE_FORCE, gs_mode=fq.GS_NONE, workspace=ws)
        torch.cuda.synchronize()
        n1 = int(host(ws)[fq.WS_BF_EVALS:fq.WS_BF_EVALS + 8].view(np.uint64)[0])
        fq.nvfp4_quantize(x, B, fq.BRUTE_FORCE, gs_mode=fq.GS_NONE, workspace=ws)
        torch.cuda.synchronize()
        n2 = int(host(ws)[fq.WS_BF_EVALS:fq.WS_BF_EVALS + 8].view(np.uint64)[0])
        nblk = x32.size // B
        assert nblk <= n1 <= 127 * nblk, (B, n1, nblk)
        assert n2 == 2 * n1
        ref = O.nvfp4_quantize(x32, B, O.RULE_BRUTE_FORCE, g=1.0)
        assert_bits(r["scales"], ref["scales"], "scales B=%d" % B)
        counts.append(n1)
    # other rules leave the counter alone
    ws.zero_()
    fq.nvfp4_quantize(x, 16, fq.FOUR_OVER_SIX, gs_mode=fq.GS_NONE, workspace=ws)
    torch.cuda.synchronize()
    assert int(host(ws)[fq.WS_BF_EVALS:fq.WS_BF_EVALS + 8].view(np.uint64)[0]) == 0


def lattice_blocks(O, sf, B, g, rows, seed):
    """Blocks built around power-of-two scales r (the brute-force kernel's
    lattice shortcut): the largest element at 0.97-1.0 of 6 S_r (c6 = r, no
    clipping) or 1.0-1.03 of it (c6 = r, clipping: the shortcut must stay off),
    the others uniform in +-6 S_r, and some placed exactly on the grids of
    neighbouring codes (k S_r v for k in 1..13), so that exact ties between
    codes occur."""
    rng = np.random.default_rng(seed)
    val = O.ue5m3_value if sf == O.SF_UE5M3 else O.e4m3_value
    last = 254 if sf == O.SF_UE5M3 else 126
    pow2 = [c for c in range(1, last + 1) if float(np.frexp(val(c))[0]) == 0.5]
    pow2 = [c for c in pow2 if c < last - 8]
    grid = np.array([0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    n = rows * 256 // B
    x = np.empty((n, B), np.float64)
    for i in range(n):
        S = val(int(rng.choice(pow2))) * float(g)
        u = rng.uniform(-6, 6, B)
        top = rng.uniform(0.97, 1.0) if i % 4 else rng.uniform(1.0, 1.03)
        u[rng.integers(B)] = 6 * top * rng.choice([-1, 1])
        for j in np.nonzero(rng.random(B) < 0.4)[0]:
            if abs(u[j]) < 6 * 0.97:
                k = int(rng.integers(1, 14))
                p = k * rng.choice(grid) * rng.choice([-1, 1])
                if abs(p) < 5.8:
                    u[j] = p
        x[i] = u * S
    return x.reshape(rows, 256).astype(np.float32)


@pytest.mark.parametrize("sf", [0, 3])
@pytest.mark.parametrize("B", [4, 8, 16, 32])
@pytest.mark.parametrize("g", [1.0, 0.125])
def test_brute_force_lattice_shortcut_cases(O, sf, B, g):
    """Brute force on blocks whose abs-max scale is a power of two: codes, scale
    bytes, dequant and MSE equal the oracle's full scan of every code, with g = 1
    (GS_NONE) and with a power-of-two g given."""
    x32 = lattice_blocks(O, O.SF_UE5M3 if sf == 3 else O.SF_E4M3, B, g, 48, seed=100 + B + sf)
    given = torch.tensor([g], dtype=torch.float32, device="cuda")
    gs_mode = fq.GS_NONE if g == 1.0 else fq.GS_GIVEN
    r = fq.nvfp4_quantize(dev(x32), block=B, rule=fq.BRUTE_FORCE, gs_mode=gs_mode,
                          global_scale=given if gs_mode == fq.GS_GIVEN else None,
                          dequant=True, mse=True, scale_fmt=fq.SF_UE5M3 if sf == 3 else fq.SF_E4M3)
    torch.cuda.synchronize()
    ref = O.block_fp4_quantize(x32, B, O.RULE_BRUTE_FORCE, O.SF_UE5M3 if sf == 3 else O.SF_E4M3,
                               g=np.float32(g))
    assert_bits(r["codes"], ref["codes"], "codes")
    assert_bits(r["scales"], ref["scales"], "scales")
    assert_bits(r["dequant"], ref["deq"], "dequant")
    assert_bits(r["mse"], ref["mse"], "mse")


# ------------------------------------------------------------------ RaZeR
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("sf,kind,specials", [(fq.SF_E3M3, "razer_weight", [5.0, -5.0, 3.5, -3.5]),
                                              (fq.SF_E4M3, "razer_act", [5.0, -5.0]),
                                              (fq.SF_E3M3, "razer_weight", [4.5, -2.5])])
@pytest.mark.parametrize("gs_mode", [fq.GS_AMAX, fq.GS_NONE])
def test_razer_small(O, sf, kind, specials, dtype, gs_mode):
    x, x32 = make(kind, 71, 256, seed=sf + 5, dtype=dtype)
    r = fq.razer_quantize(x, sf, specials, gs_mode=gs_mode, dequant=True, mse=True)
    torch.cuda.synchronize()
    g = oracle_g(O, x32, gs_mode, sf=sf)
    ref = O.razer_quantize(x32, sf, specials, g=g)
    assert_bits(r["codes"], ref["codes"], "codes")
    assert_bits(r["meta"], ref["meta"], "meta")
    assert_bits(r["dequant"], ref["deq"], "dequant")
    assert_bits(r["mse"], ref["mse"], "mse")


# ------------------------------------------------------------------ MXFP4
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("use_t,had", [(False, False), (False, True), (True, True)])
def test_mxfp4_absmax_small(O, dtype, use_t, had):
    x, x32 = make("mx_act", 83, 256, seed=7, dtype=dtype)
    t = inputs.positive_vector(256, seed=5) if use_t else None
    r = fq.mxfp4_quantize(x, None if t is None else dev(t), had, fq.ABSMAX, dequant=True, mse=True)
    torch.cuda.synchronize()
    ref = O.mxfp4_quantize(x32, t, had, O.RULE_ABSMAX)
    assert_bits(r["codes"], ref["codes"], "codes")
    assert_bits(r["scales"], ref["scales"], "scales")
    assert_bits(r["dequant"], ref["deq"], "dequant")
    assert_bits(r["mse"], ref["mse"], "mse")


def test_mxfp4_absmax_wide_rows(O):
    """Rows of more than 512 column blocks (16416 columns): the one-lane-per-block
    kernel, with t and the rotation, bit for bit."""
    x, x32 = make("mx_act", 9, 16416, seed=17, dtype="bf16")
    t = inputs.positive_vector(16416, seed=18)
    r = fq.mxfp4_quantize(x, dev(t), True, fq.ABSMAX, dequant=True, mse=True)
    torch.cuda.synchronize()
    ref = O.mxfp4_quantize(x32, t, True, O.RULE_ABSMAX)
    assert_bits(r["codes"], ref["codes"], "codes")
    assert_bits(r["scales"], ref["scales"], "scales")
    assert_bits(r["dequant"], ref["deq"], "dequant")
    assert_bits(r["mse"], ref["mse"], "mse")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_mxfp4_hessian_small(O, dtype):
    w, w32 = make("mx_weight", 300, 256, seed=8, dtype=dtype)
    act = inputs.as_f32(inputs.generate("mx_act", 512, 256, seed=8))
    t, ti = O.channel_scale(act, w32, 0.75)
    hess = O.hessian_blocks(act, t, True).astype(np.float32)
    r = fq.mxfp4_quantize(w, dev(ti), True, fq.HESSIAN_EXP, hess=dev(hess), dequant=True, mse=True)
    torch.cuda.synchronize()
    ref = O.mxfp4_quantize(w32, ti, True, O.RULE_HESSIAN_EXP, hess)
    assert_bits(r["codes"], ref["codes"], "codes")
    assert_bits(r["scales"], ref["scales"], "scales")
    assert_bits(r["dequant"], ref["deq"], "dequant")
    assert_bits(r["mse"], ref["mse"], "mse")
    std = O.mxfp4_quantize(w32, ti, True, O.RULE_ABSMAX)
    assert np.any(ref["scales"] != std["scales"])     # the Hessian rule moved some exponents


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_hessian_blocks(O, dtype):
    x, x32 = make("mx_act", 700, 128, seed=9, dtype=dtype)
    t = inputs.positive_vector(128, seed=6)
    ws = torch.empty(fq.workspace_size(fq.OP_HESSIAN, 700, 128), dtype=torch.uint8, device="cuda")
    h = fq.hessian_blocks(x, dev(t), True, workspace=ws)
    assert fq.hessian_status(ws) == 0
    ref = O.hessian_blocks(x32, t, True)
    got = host(h).astype(np.float64)
    for k in range(ref.shape[0]):
        err = np.linalg.norm(got[k] - ref[k]) / np.linalg.norm(ref[k])
        assert err <= 1e-5, (k, err)


def test_channel_scale(O):
    x, x32 = make("mx_act", 1000, 256, seed=10, dtype="bf16")
    w, w32 = make("mx_weight", 300, 256, seed=10, dtype="bf16")
    t, ti = fq.channel_scale(x, w, 0.75)
    torch.cuda.synchronize()
    rt, rti = O.channel_scale(x32, w32, 0.75)
    np.testing.assert_allclose(host(t), rt, rtol=3e-7)
    assert_bits(ti, (np.float32(1) / host(t)).astype(np.float32), "t_inv is the fp32 reciprocal of t")


# ------------------------------------------------------- Flip-Refinement
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("K", [0, 1, 7, 128, 100000])
def test_flip_refine_small(O, dtype, K):
    """37 rows (ragged against the 4 rows of a CTA) x 256 columns: refined
    codes and per-row move counts equal the oracle's."""
    w, w32 = make("mx_weight", 37, 256, seed=11, dtype=dtype)
    xa, xa32 = make("mx_act", 300, 256, seed=12, dtype="f32")
    t, ti = O.channel_scale(xa32, w32, 0.75)
    hin = O.hessian_blocks(xa32, t, True).astype(np.float32)
    q = O.mxfp4_quantize(w32, ti, True, O.RULE_HESSIAN_EXP, hin, want_deq=False)
    codes = dev(q["codes"].copy())
    mv = fq.mxfp4_flip_refine(w, codes, dev(q["scales"]), dev(hin), chan_scale=dev(ti), max_moves=K)
    torch.cuda.synchronize()
    rc, rm = O.mxfp4_flip_refine(w32, ti, True, hin, q["codes"], q["scales"], K)
    assert_bits(host(mv), rm, "moves per row")
    assert_bits(codes, rc, "refined codes")
    if K >= 7:
        assert np.all(rm > 0)


@pytest.mark.parametrize("K", [5, 10, 100000])
def test_flip_refine_long_block_sequences(O, K):
    """Blocks whose own greedy runs for many moves (every element just below a
    rounding midpoint, H' dominated by the all-ones direction): past the moves
    precomputed per block the rows take the direct per-row path; results are
    the same either way."""
    rng = np.random.default_rng(3)
    w32 = np.zeros((6, 64), np.float32)
    for r in range(6):
        for k in range(2):
            w32[r, 32 * k:32 * k + 32] = (np.float32(4.9 * 2.0 ** (r - 2)) *
                                          (1 + 0.001 * rng.standard_normal(32)).astype(np.float32))
    H = np.tile((np.ones((32, 32), np.float32) + 0.05 * np.eye(32, dtype=np.float32))[None], (2, 1, 1))
    q = O.mxfp4_quantize(w32, None, False, O.RULE_HESSIAN_EXP, H, want_deq=False)
    codes = dev(q["codes"].copy())
    mv = fq.mxfp4_flip_refine(dev(w32), codes, dev(q["scales"]), dev(H), hadamard=False, max_moves=K)
    torch.cuda.synchronize()
    rc, rm = O.mxfp4_flip_refine(w32, None, False, H, q["codes"], q["scales"], K)
    assert_bits(host(mv), rm, "moves per row")
    assert_bits(codes, rc, "refined codes")
    assert np.all(rm == min(K, 28))


def test_flip_refine_without_transform(O):
    w, w32 = make("mx_weight", 9, 128, seed=13, dtype="f32")
    xa, xa32 = make("mx_act", 200, 128, seed=14, dtype="f32")
    hin = O.hessian_blocks(xa32, None, False).astype(np.float32)
    q = O.mxfp4_quantize(w32, None, False, O.RULE_HESSIAN_EXP, hin, want_deq=False)
    codes = dev(q["codes"].copy())
    mv = fq.mxfp4_flip_refine(w, codes, dev(q["scales"]), dev(hin), hadamard=False, max_moves=64)
    torch.cuda.synchronize()
    rc, rm = O.mxfp4_flip_refine(w32, None, False, hin, q["codes"], q["scales"], 64)
    assert_bits(host(mv), rm, "moves per row")
    assert_bits(codes, rc, "refined codes")


# ------------------------------------------------------------- dequant
@pytest.mark.parametrize("B", [4, 8, 16, 32])
def test_dequant_nvfp4(O, B):
    x, x32 = make("gaussian", 45, 256, seed=B, dtype="f32")
    g = O.global_scale(O.amax(x32))
    q = O.nvfp4_quantize(x32, B, O.RULE_FOUR_OVER_SIX, g=g)
    gd = torch.tensor([g], dtype=torch.float32, device="cuda")
    r = fq.dequant_mse(dev(q["codes"]), dev(q["scales"]), 45, 256, B, fq.SF_E4M3, None, gd, ref=x)
    torch.cuda.synchronize()
    ref = O.dequant_mse(q["codes"], q["scales"], 45, 256, B, O.SF_E4M3, None, g=g, ref=x32)
    assert_bits(r["dequant"], ref["deq"], "dequant")
    assert_bits(r["mse"], ref["mse"], "mse")


def test_dequant_razer_and_mx(O):
    w, w32 = make("razer_weight", 40, 256, seed=2, dtype="bf16")
    sp = [5.0, -5.0, 3.5, -3.5]
    g = O.global_scale(O.amax(w32), O.SF_E3M3)
    q = O.razer_quantize(w32, O.SF_E3M3, sp, g=g)
    gd = torch.tensor([g], dtype=torch.float32, device="cuda")
    r = fq.dequant_mse(dev(q["codes"]), dev(q["meta"]), 40, 256, 16, fq.SF_E3M3, sp, gd, ref=w)
    torch.cuda.synchronize()
    assert_bits(r["dequant"], q["deq"], "razer dequant")
    assert_bits(r["mse"], q["mse"], "razer mse")
    a, a32 = make("mx_act", 40, 256, seed=2, dtype="f32")
    qm = O.mxfp4_quantize(a32, None, True, O.RULE_ABSMAX)
    y = O.mx_transform(a32, None, True)
    r = fq.dequant_mse(dev(qm["codes"]), dev(qm["scales"]), 40, 256, 32, fq.SF_E8M0, None, None, ref=dev(y))
    torch.cuda.synchronize()
    assert_bits(r["dequant"], qm["deq"], "mx dequant")
    assert_bits(r["mse"], qm["mse"], "mx mse")


# ------------------------------------------------- full-size workloads
def _rows(n, k, seed):
    return np.sort(np.random.default_rng(seed).choice(n, size=k, replace=False))


def test_full_gaussian_nvfp4_prevent_zero(O):
    """4096 x 4096 fp32 N(0,1), block 16, hierarchical scale: the whole tensor."""
    a = inputs.generate("gaussian")
    r = fq.nvfp4_quantize(dev(a), 16, fq.PREVENT_ZERO, gs_mode=fq.GS_AMAX, dequant=True, mse=True)
    torch.cuda.synchronize()
    g = O.global_scale(O.amax(a))
    assert_bits(r["global_scale"], np.array([g], np.float32), "g")
    ref = O.nvfp4_quantize(a, 16, O.RULE_PREVENT_ZERO, g=g)
    for k, rk in (("codes", "codes"), ("scales", "scales"), ("dequant", "deq"), ("mse", "mse")):
        assert_bits(r[k], ref[rk], k)


@pytest.mark.parametrize("B", [4, 8, 16, 32])
def test_full_student_t_sweep_sampled(O, B):
    """8192 x 8192 Student-t x 1e-3, all four rules, g = 1; 24 sampled rows per rule."""
    a = inputs.generate("student_t")
    x = dev(a)
    rows = _rows(a.shape[0], 24, B)
    for rule in RULES:
        r = fq.nvfp4_quantize(x, B, rule, gs_mode=fq.GS_NONE, mse=True)
        torch.cuda.synchronize()
        ref = O.nvfp4_quantize(a[rows], B, rule, g=1.0, want_deq=False)
        assert_bits(host(r["codes"])[rows], ref["codes"], "codes rule %d" % rule)
        assert_bits(host(r["scales"])[rows], ref["scales"], "scales rule %d" % rule)
        assert_bits(host(r["mse"])[rows], ref["mse"], "mse rule %d" % rule)
    del x
    torch.cuda.empty_cache()


@pytest.mark.parametrize("kind,sf,specials", [("razer_weight", fq.SF_E3M3, [5.0, -5.0, 3.5, -3.5]),
                                              ("razer_act", fq.SF_E4M3, [5.0, -5.0])])
def test_full_razer_sampled(O, kind, sf, specials):
    a = inputs.generate(kind)
    a32 = inputs.as_f32(a)
    r = fq.razer_quantize(dev(a), sf, specials, gs_mode=fq.GS_AMAX, mse=True)
    torch.cuda.synchronize()
    g = O.global_scale(O.amax(a32), sf)
    assert_bits(r["global_scale"], np.array([g], np.float32), "g")
    rows = _rows(a.shape[0], 32, sf)
    ref = O.razer_quantize(a32[rows], sf, specials, g=g, want_deq=False)
    assert_bits(host(r["codes"])[rows], ref["codes"], "codes")
    assert_bits(host(r["meta"])[rows], ref["meta"], "meta")
    assert_bits(host(r["mse"])[rows], ref["mse"], "mse")


def test_full_mxfp4_prep_sampled(O):
    """8192 x 4096 activations and 4096 x 4096 weights: t, H' and both quantizers."""
    xa = inputs.generate("mx_act")
    wa = inputs.generate("mx_weight")
    x32, w32 = inputs.as_f32(xa), inputs.as_f32(wa)
    x, w = dev(xa), dev(wa)
    t, ti = fq.channel_scale(x, w, 0.75)
    h = fq.hessian_blocks(x, t, True)
    qa = fq.mxfp4_quantize(x, t, True, fq.ABSMAX, mse=True)
    torch.cuda.synchronize()
    rt, _ = O.channel_scale(x32, w32, 0.75)
    np.testing.assert_allclose(host(t), rt, rtol=3e-7)
    tg, tig = host(t), host(ti)
    rows = _rows(8192, 32, 1)
    ref = O.mxfp4_quantize(x32[rows], tg, True, O.RULE_ABSMAX, want_deq=False)
    assert_bits(host(qa["codes"])[rows], ref["codes"], "act codes")
    assert_bits(host(qa["scales"])[rows], ref["scales"], "act scales")
    assert_bits(host(qa["mse"])[rows], ref["mse"], "act mse")
    # H' from the GPU's own t, against the oracle on the same t
    href = O.hessian_blocks(x32, tg, True)
    hg = host(h).astype(np.float64)
    for k in range(128):                      # every 32 x 32 block, at the small cases' tolerance
        assert np.linalg.norm(hg[k] - href[k]) / np.linalg.norm(href[k]) <= 1e-5, k
    # weight quantizer: decision parity on the oracle's H' (an input to both)
    hin = href.astype(np.float32)
    qw = fq.mxfp4_quantize(w, ti, True, fq.HESSIAN_EXP, hess=dev(hin), mse=True)
    torch.cuda.synchronize()
    wrows = _rows(4096, 24, 2)
    refw = O.mxfp4_quantize(w32[wrows], tig, True, O.RULE_HESSIAN_EXP, hin, want_deq=False)
    assert_bits(host(qw["codes"])[wrows], refw["codes"], "weight codes")
    assert_bits(host(qw["scales"])[wrows], refw["scales"], "weight scales")
    assert_bits(host(qw["mse"])[wrows], refw["mse"], "weight mse")
    # Flip-Refinement of the whole weight tensor (128 moves per row), sampled rows
    codes = qw["codes"].clone()
    mv = fq.mxfp4_flip_refine(w, codes, qw["scales"], dev(hin), chan_scale=ti, max_moves=128)
    torch.cuda.synchronize()
    rc, rm = O.mxfp4_flip_refine(w32[wrows], tig, True, hin, host(qw["codes"])[wrows],
                                 host(qw["scales"])[wrows], 128)
    assert_bits(host(codes)[wrows], rc, "refined weight codes")
    assert_bits(host(mv)[wrows], rm, "moves per row")
