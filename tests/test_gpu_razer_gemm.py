"""GPU parity of the RaZeR-aware W4A4 GEMM ("RaZeR: Redundant Zero Remapping",
sections 2.2 and 2.3) against the oracle's fp64 product of the exactly decoded
RaZeR operands (the -0 code stands for the block's special value).

The operand split (razer_gemm_prepare) is checked exactly: main + extra
reproduces every RaZeR value in fp64 and the E4M3 scale bytes equal the RaZeR
scales.  The GEMM bars are the ones of the plain W4A4 GEMM (element-wise
bounds from fp32 accumulation over every pass, tests/gemm_check.py, plus the
Frobenius bars), for bf16 and fp32 output.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_scaled_fp4_03_b200 import binding as fq
from block_scaled_fp4_03_b200 import inputs
from gemm_check import band_rows, check_gemm
from test_gpu_gemm import dev, to_mma_layout

pytestmark = pytest.mark.gpu

SPW = [5.0, -5.0, 3.5, -3.5]     # weight table (E3M3 scale, 2-bit selector)
SPA = [5.0, -5.0]                # activation table (E4M3 scale, 1-bit selector)


def from_mma_layout(flat, rows, kb):
    r = np.arange(rows)[:, None]
    c = np.arange(kb)[None, :]
    off = ((r // 128) * (kb // 4) + c // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + c % 4
    return np.asarray(flat)[off]


def unpack(codes):
    c = np.empty((codes.shape[0], codes.shape[1] * 2), np.int64)
    c[:, 0::2] = codes & 0xF
    c[:, 1::2] = codes >> 4
    return c


def razer_operand(O, x32, sf, specials):
    g = O.global_scale(O.amax(x32), sf)
    q = O.razer_quantize(x32, sf, specials, g=g, want_deq=False, want_mse=False)
    return q, g


def prepared(q, sf, specials):
    return fq.razer_gemm_prepare(dev(q["codes"]), dev(q["meta"]), sf, specials)


@pytest.mark.parametrize("sf,kind,specials", [(1, "razer_weight", SPW), (0, "razer_act", SPA),
                                              (1, "gemm_weight", [5.5, -5.5, 2.5, -4.5])])
def test_prepare_split_is_exact(O, sf, kind, specials):
    rows, cols = 256, 512
    x32 = inputs.as_f32(inputs.generate(kind, rows, cols, seed=3))
    q, _ = razer_operand(O, x32, sf, specials)
    p = prepared(q, sf, specials)
    torch.cuda.synchronize()
    main = p["main"].cpu().numpy()
    extra = p["extra"].cpu().numpy()
    sc = from_mma_layout(p["scales"].cpu().numpy(), rows, cols // 16)
    e2 = np.array([O.e2m1_value(c) for c in range(16)], np.float64)
    e4 = np.array([O.e4m3_value(c) if c < 0x7F else np.nan for c in range(256)], np.float64)
    sc_code = q["meta"] & (0x3F if sf == 1 else 0x7F)
    val = O.e3m3_value if sf == 1 else O.e4m3_value
    want_sc = np.array([[val(int(c)) for c in row] for row in sc_code])
    assert np.array_equal(e4[sc], want_sc)
    S = np.repeat(e4[sc], 16, axis=1)
    got = e2[unpack(main)] * S + e2[unpack(extra)] * S
    ref = O.razer_decode_exact(q["codes"], q["meta"], sf, specials)
    assert np.array_equal(got, ref)
    c = unpack(q["codes"])
    assert (c == 8).any()
    assert np.array_equal(unpack(main)[c != 8], c[c != 8])
    assert np.all(unpack(extra)[c != 8] == 0)


def test_prepare_rejects_bad_tables_and_shapes():
    L = fq.lib()
    fake = ctypes.c_void_p(0x10000)

    def call(rows, cols, sf, sp):
        arr = (ctypes.c_float * len(sp))(*sp)
        return L.razer_gemm_prepare(fake, fake, rows, cols, sf, ctypes.cast(arr, ctypes.c_void_p), len(sp),
                                    fake, fake, fake, None)
    assert call(128, 64, 1, [11.0]) == 3          # 11 is no sum of two E2M1 values
    assert call(128, 64, 1, [0.25]) == 1          # not a multiple of 0.5
    assert call(128, 64, 0, [5.0, -5.0, 3.5]) == 1   # E4M3 meta has one selector bit
    assert call(100, 64, 1, [5.0]) == 1
    assert call(128, 48, 1, [5.0]) == 1
    assert call(128, 64, 2, [5.0]) == 1
    assert call(0, 64, 1, [5.0]) == 0


def gemm_case(O, M, N, K, a_razer, w_razer, seed, out_dtype=fq.BF16):
    a32 = inputs.as_f32(inputs.generate("gemm_act", M, K, seed=seed))
    w32 = inputs.as_f32(inputs.generate("gemm_weight", N, K, seed=seed + 1))
    if a_razer:
        qa, ga = razer_operand(O, a32, 0, SPA)
        pa = prepared(qa, 0, SPA)
        a_args = (pa["main"], pa["scales"], pa["extra"])
        da = O.razer_decode_exact(qa["codes"], qa["meta"], 0, SPA)
    else:
        ga = O.global_scale(O.amax(a32))
        qa = O.nvfp4_quantize(a32, 16, O.RULE_FOUR_OVER_SIX, g=ga, want_deq=False, want_mse=False)
        a_args = (dev(qa["codes"]), dev(to_mma_layout(qa["scales"])), None)
        da = O.nvfp4_decode_exact(qa["codes"], qa["scales"])
    if w_razer:
        qw, gw = razer_operand(O, w32, 1, SPW)
        pw = prepared(qw, 1, SPW)
        w_args = (pw["main"], pw["scales"], pw["extra"])
        dw = O.razer_decode_exact(qw["codes"], qw["meta"], 1, SPW)
    else:
        gw = O.global_scale(O.amax(w32))
        qw = O.nvfp4_quantize(w32, 16, O.RULE_ABSMAX, g=gw, want_deq=False, want_mse=False)
        w_args = (dev(qw["codes"]), dev(to_mma_layout(qw["scales"])), None)
        dw = O.nvfp4_decode_exact(qw["codes"], qw["scales"])
    ws = torch.empty(8192, dtype=torch.uint8, device="cuda")
    out = fq.razer_w4a4_gemm(a_args[0], a_args[1], dev(np.array([ga], np.float32)),
                             w_args[0], w_args[1], dev(np.array([gw], np.float32)),
                             a_extra=a_args[2], w_extra=w_args[2], workspace=ws, out_dtype=out_dtype)
    assert fq.gemm_status(ws) == 0
    return out, da, dw, float(ga) * float(gw)


@pytest.mark.parametrize("out_dtype", [fq.BF16, fq.F32])
@pytest.mark.parametrize("a_razer,w_razer", [(False, True), (True, False), (True, True)])
@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (256, 512, 512), (384, 256, 1024), (512, 768, 768)])
def test_razer_gemm(O, M, N, K, a_razer, w_razer, out_dtype):
    out, da, dw, g = gemm_case(O, M, N, K, a_razer, w_razer, seed=M + N + K, out_dtype=out_dtype)
    passes = (2 if a_razer else 1) * (2 if w_razer else 1)
    check_gemm(out, da, dw, g, K * passes, "razer a=%d w=%d %dx%dx%d" % (a_razer, w_razer, M, N, K))


def test_razer_gemm_beats_dropping_the_specials(O):
    """Treating -0 as zero (what the tensor core alone does) must be measurably
    worse than the two-pass product: the extra pass carries real signal."""
    M, N, K = 256, 256, 512
    a32 = inputs.as_f32(inputs.generate("gemm_act", M, K, seed=4))
    w32 = inputs.as_f32(inputs.generate("gemm_weight", N, K, seed=5))
    ga = O.global_scale(O.amax(a32))
    qa = O.nvfp4_quantize(a32, 16, O.RULE_FOUR_OVER_SIX, g=ga, want_deq=False, want_mse=False)
    qw, gw = razer_operand(O, w32, 1, SPW)
    pw = prepared(qw, 1, SPW)
    args = (dev(qa["codes"]), dev(to_mma_layout(qa["scales"])), dev(np.array([ga], np.float32)))
    gwd = dev(np.array([gw], np.float32))
    two = fq.razer_w4a4_gemm(*args, pw["main"], pw["scales"], gwd, w_extra=pw["extra"])
    ref = O.gemm_values(O.nvfp4_decode_exact(qa["codes"], qa["scales"]),
                        O.razer_decode_exact(qw["codes"], qw["meta"], 1, SPW), ga, gw)
    # -0 decoded as zero: the raw RaZeR codes with the converted scales, one pass
    raw = fq.razer_w4a4_gemm(*args, dev(qw["codes"]), pw["scales"], gwd)
    e_two = np.linalg.norm(two.float().cpu().numpy() - ref) / np.linalg.norm(ref)
    e_raw = np.linalg.norm(raw.float().cpu().numpy() - ref) / np.linalg.norm(ref)
    assert e_two <= 4e-3 and e_raw > 10 * e_two, (e_two, e_raw)


def test_single_pass_equals_w4a4_gemm(O):
    M, N, K = 256, 512, 512
    a32 = inputs.as_f32(inputs.generate("gemm_act", M, K, seed=8))
    w32 = inputs.as_f32(inputs.generate("gemm_weight", N, K, seed=9))
    ga = O.global_scale(O.amax(a32))
    gw = O.global_scale(O.amax(w32))
    qa = O.nvfp4_quantize(a32, 16, O.RULE_ABSMAX, g=ga, want_deq=False, want_mse=False)
    qw = O.nvfp4_quantize(w32, 16, O.RULE_ABSMAX, g=gw, want_deq=False, want_mse=False)
    A, SA = dev(qa["codes"]), dev(to_mma_layout(qa["scales"]))
    W, SW = dev(qw["codes"]), dev(to_mma_layout(qw["scales"]))
    gad, gwd = dev(np.array([ga], np.float32)), dev(np.array([gw], np.float32))
    one = fq.razer_w4a4_gemm(A, SA, gad, W, SW, gwd)
    ref = fq.w4a4_gemm(A, W, SW, gwd, a_scales=SA, a_global_scale=gad)
    assert torch.equal(one.view(torch.int16), ref.view(torch.int16))


def test_razer_gemm_full_size_sampled(O):
    """M=8192 x N=14336 x K=4096: RaZeR weights (E3M3, +-5 / +-3.5), 4-over-6
    NVFP4 activations quantized on the device, two passes."""
    M, N, K = 8192, 14336, 4096
    a = inputs.generate("gemm_act")
    w32 = inputs.as_f32(inputs.generate("gemm_weight"))
    qw, gw = razer_operand(O, w32, 1, SPW)
    pw = prepared(qw, 1, SPW)
    ad = dev(a)
    qa_dev = fq.nvfp4_quantize(ad, 16, fq.FOUR_OVER_SIX, gs_mode=fq.GS_AMAX, sf_layout=fq.SF_MMA)
    ws = torch.empty(8192, dtype=torch.uint8, device="cuda")
    out = fq.razer_w4a4_gemm(qa_dev["codes"], qa_dev["scales"], qa_dev["global_scale"], pw["main"],
                             pw["scales"], dev(np.array([gw], np.float32)), w_extra=pw["extra"], workspace=ws)
    assert fq.gemm_status(ws) == 0
    a32 = inputs.as_f32(a)
    ga = O.global_scale(O.amax(a32))
    rows = band_rows(M, salt=5)
    qa = O.nvfp4_quantize(a32[rows], 16, O.RULE_FOUR_OVER_SIX, g=ga, want_deq=False, want_mse=False)
    dw = O.razer_decode_exact(qw["codes"], qw["meta"], 1, SPW)
    check_gemm(out[torch.from_numpy(rows).cuda()], O.nvfp4_decode_exact(qa["codes"], qa["scales"]), dw,
               float(ga) * float(gw), 2 * K, "razer w full 8192x14336x4096")
