"""GPU parity of the MXFP4 W4A4 GEMM ("MACaQ" review, section 1: MXFP4 operands,
E2M1 values with one E8M0 exponent per 32 elements; the activations rotated
online) against the oracle's fp64 product of the exactly decoded operands.

The prologue (channel scale, 32-block rotation, E8M0 quantization of a dense A
with its scales written in the GEMM's layout) must give exactly the operands
the oracle quantizer gives: the dense-A result equals the packed-A result bit
for bit.  The GEMM bars are the ones of the NVFP4 GEMM (element-wise bounds
from fp32 accumulation, tests/gemm_check.py, plus the Frobenius bars), for
bf16 and fp32 output.
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


def operands(O, M, N, K, seed, rule_w=None):
    x = inputs.generate("mx_act", M, K, seed=seed)            # bf16 bits
    w32 = inputs.as_f32(inputs.generate("mx_weight", N, K, seed=seed + 1))
    t = inputs.positive_vector(K, seed=seed + 2)
    tinv = (1.0 / t.astype(np.float64)).astype(np.float32)
    x32 = inputs.as_f32(x)
    qa = O.mxfp4_quantize(x32, t, True, O.RULE_ABSMAX, want_deq=False, want_mse=False)
    if rule_w == O.RULE_HESSIAN_EXP:
        hess = O.hessian_blocks(x32, t, True).astype(np.float32)
        qw = O.mxfp4_quantize(w32, tinv, True, O.RULE_HESSIAN_EXP, hess, want_deq=False, want_mse=False)
    else:
        qw = O.mxfp4_quantize(w32, tinv, True, O.RULE_ABSMAX, want_deq=False, want_mse=False)
    return x, t, qa, qw


def test_scales_to_mma_matches_layout():
    rng = np.random.default_rng(3)
    for rows, n in ((128, 4), (256, 64), (384, 136)):
        sc = rng.integers(0, 256, size=(rows, n), dtype=np.uint8)
        got = fq.scales_to_mma(dev(sc)).cpu().numpy()
        assert np.array_equal(got, to_mma_layout(sc))


def test_scales_to_mma_rejects_bad_shapes():
    L = fq.lib()
    fake = ctypes.c_void_p(0x10000)
    assert L.fp4_scales_to_mma(fake, 100, 8, fake, None) == 1
    assert L.fp4_scales_to_mma(fake, 128, 6, fake, None) == 1
    assert L.fp4_scales_to_mma(fake, 0, 8, fake, None) == 0


@pytest.mark.parametrize("out_dtype", [fq.BF16, fq.F32])
@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (256, 512, 512), (384, 256, 1024), (512, 768, 768),
                                   (1024, 1024, 2048)])
def test_mx_gemm_packed(O, M, N, K, out_dtype):
    _, _, qa, qw = operands(O, M, N, K, seed=M + N + K)
    out = fq.mxfp4_gemm(dev(qa["codes"]), dev(qw["codes"]), dev(to_mma_layout(qw["scales"])),
                        a_scales=dev(to_mma_layout(qa["scales"])), out_dtype=out_dtype)
    check_gemm(out, O.mx_decode_exact(qa["codes"], qa["scales"]), O.mx_decode_exact(qw["codes"], qw["scales"]),
               1.0, K, "mx packed %dx%dx%d" % (M, N, K))


@pytest.mark.parametrize("M,N,K", [(256, 256, 512), (384, 512, 256)])
def test_mx_gemm_dense_prologue_equals_packed(O, M, N, K):
    x, t, qa, qw = operands(O, M, N, K, seed=11 + M, rule_w=O.RULE_HESSIAN_EXP)
    ws_sc = dev(to_mma_layout(qw["scales"]))
    packed = fq.mxfp4_gemm(dev(qa["codes"]), dev(qw["codes"]), ws_sc, a_scales=dev(to_mma_layout(qa["scales"])))
    ws = torch.empty(fq.workspace_size(fq.OP_MX_GEMM, M, K, N), dtype=torch.uint8, device="cuda")
    dense = fq.mxfp4_gemm(dev(x), dev(qw["codes"]), ws_sc, chan_scale=dev(t), workspace=ws)
    assert fq.gemm_status(ws) == 0
    assert torch.equal(dense.view(torch.int16), packed.view(torch.int16))
    check_gemm(dense, O.mx_decode_exact(qa["codes"], qa["scales"]), O.mx_decode_exact(qw["codes"], qw["scales"]),
               1.0, K, "mx dense prologue %dx%dx%d" % (M, N, K))


def test_mx_gemm_weights_through_flip_and_relayout(O):
    """Weights refined by Flip-Refinement on the device (row-major exponents),
    then moved to the MMA layout by fp4_scales_to_mma."""
    M, N, K = 256, 256, 512
    x, t, qa, qw = operands(O, M, N, K, seed=21, rule_w=O.RULE_HESSIAN_EXP)
    w32 = inputs.as_f32(inputs.generate("mx_weight", N, K, seed=22))
    tinv = (1.0 / t.astype(np.float64)).astype(np.float32)
    hess = O.hessian_blocks(inputs.as_f32(x), t, True).astype(np.float32)
    codes, _ = O.mxfp4_flip_refine(w32, tinv, True, hess, qw["codes"], qw["scales"], 64)
    wc, wsr = dev(codes), dev(qw["scales"])
    out = fq.mxfp4_gemm(dev(qa["codes"]), wc, fq.scales_to_mma(wsr), a_scales=dev(to_mma_layout(qa["scales"])))
    check_gemm(out, O.mx_decode_exact(qa["codes"], qa["scales"]), O.mx_decode_exact(codes, qw["scales"]),
               1.0, K, "mx flip-refined weights")


def test_mx_gemm_full_size_sampled(O):
    """M=8192 x N=16384 x K=4096 (the size the MACaQ review quotes the online
    transform's overhead at): dense bf16 activations through the prologue."""
    M, N, K = 8192, 16384, 4096
    x = inputs.generate("mx_act", M, K, seed=31)
    w32 = inputs.as_f32(inputs.generate("mx_weight", N, K, seed=32))
    t = inputs.positive_vector(K, seed=33)
    tinv = (1.0 / t.astype(np.float64)).astype(np.float32)
    qw = O.mxfp4_quantize(w32, tinv, True, O.RULE_ABSMAX, want_deq=False, want_mse=False)
    ws = torch.empty(fq.workspace_size(fq.OP_MX_GEMM, M, K, N), dtype=torch.uint8, device="cuda")
    out = fq.mxfp4_gemm(dev(x), dev(qw["codes"]), dev(to_mma_layout(qw["scales"])), chan_scale=dev(t),
                        workspace=ws)
    assert fq.gemm_status(ws) == 0
    rows = band_rows(M, salt=9)
    qa = O.mxfp4_quantize(inputs.as_f32(x)[rows], t, True, O.RULE_ABSMAX, want_deq=False, want_mse=False)
    check_gemm(out[torch.from_numpy(rows).cuda()], O.mx_decode_exact(qa["codes"], qa["scales"]),
               O.mx_decode_exact(qw["codes"], qw["scales"]), 1.0, K, "mx full 8192x16384x4096")
