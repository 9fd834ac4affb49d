"""GPU parity of the tcgen05 W4A4 GEMM ("Why Gated DeltaNet Survives 4-Bit
Quantization" review, section 1: NVFP4 W4A4) against the oracle's fp64 product
of the exactly decoded NVFP4 operands.

Every checked element is held to a bound derived from fp32 accumulation (and,
for bf16 output, the bf16 rounding): see tests/gemm_check.py.  The fp32 output
mode is also held to a relative Frobenius error of 1e-5 against the raw fp64
product, the bf16 output to 1e-3 against the bf16-rounded product.  The
full-size case checks one row in every 128-row band over all columns, so every
output tile of both kernels is sampled.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_scaled_fp4_03_b200 import binding as fq
from block_scaled_fp4_03_b200 import inputs
from gemm_check import band_rows, check_gemm

pytestmark = pytest.mark.gpu


def to_mma_layout(sc):
    """Row-major [rows][K/16] scale bytes -> the MMA scale-factor layout (flat)."""
    rows, kb = sc.shape
    out = np.zeros(rows * kb, np.uint8)
    r = np.arange(rows)[:, None]
    c = np.arange(kb)[None, :]
    off = ((r // 128) * (kb // 4) + c // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + c % 4
    out[off] = sc
    return out


def dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def quantized_operand(O, x32, rule):
    g = O.global_scale(O.amax(x32))
    q = O.nvfp4_quantize(x32, 16, rule, g=g, want_deq=False, want_mse=False)
    return q, g


SHAPES = [(128, 256, 256), (256, 512, 512), (384, 768, 2048), (2048, 4096, 512)]


@pytest.mark.parametrize("out_dtype", [fq.BF16, fq.F32])
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_packed_operands(O, M, N, K, out_dtype):
    a32 = inputs.as_f32(inputs.generate("gemm_act", M, K, seed=M + K))
    w32 = inputs.as_f32(inputs.generate("gemm_weight", N, K, seed=N + K))
    qa, ga = quantized_operand(O, a32, O.RULE_FOUR_OVER_SIX)
    qw, gw = quantized_operand(O, w32, O.RULE_ABSMAX)
    out = fq.w4a4_gemm(dev(qa["codes"]), dev(qw["codes"]), dev(to_mma_layout(qw["scales"])),
                       dev(np.array([gw], np.float32)), a_scales=dev(to_mma_layout(qa["scales"])),
                       a_global_scale=dev(np.array([ga], np.float32)), out_dtype=out_dtype)
    torch.cuda.synchronize()
    rows = np.arange(M) if M <= 512 else band_rows(M)
    da = O.nvfp4_decode_exact(qa["codes"][rows], qa["scales"][rows])
    dw = O.nvfp4_decode_exact(qw["codes"], qw["scales"])
    check_gemm(out[torch.from_numpy(rows).cuda()], da, dw, float(ga) * float(gw), K,
               "nvfp4 packed %dx%dx%d" % (M, N, K))


def test_fp32_and_bf16_outputs_agree(O):
    """The bf16 output is the round-to-nearest bf16 of the fp32 output, element for element."""
    M, N, K = 256, 512, 1024
    a32 = inputs.as_f32(inputs.generate("gemm_act", M, K, seed=3))
    w32 = inputs.as_f32(inputs.generate("gemm_weight", N, K, seed=4))
    qa, ga = quantized_operand(O, a32, O.RULE_FOUR_OVER_SIX)
    qw, gw = quantized_operand(O, w32, O.RULE_ABSMAX)
    args = (dev(qa["codes"]), dev(qw["codes"]), dev(to_mma_layout(qw["scales"])), dev(np.array([gw], np.float32)))
    kw = dict(a_scales=dev(to_mma_layout(qa["scales"])), a_global_scale=dev(np.array([ga], np.float32)))
    o16 = fq.w4a4_gemm(*args, **kw)
    o32 = fq.w4a4_gemm(*args, out_dtype=fq.F32, **kw)
    assert o32.dtype == torch.float32 and o16.dtype == torch.bfloat16
    assert torch.equal(o32.to(torch.bfloat16).view(torch.int16), o16.view(torch.int16))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_gemm_fused_activation_quant(O, dtype):
    M, N, K = 256, 512, 1024
    a = inputs.generate("gemm_act", M, K, seed=5)
    a32 = inputs.as_f32(a)
    if dtype == "f32":
        a = a32
    w32 = inputs.as_f32(inputs.generate("gemm_weight", N, K, seed=5))
    qw, gw = quantized_operand(O, w32, O.RULE_ABSMAX)
    ws = torch.empty(fq.workspace_size(fq.OP_GEMM, M, K, N), dtype=torch.uint8, device="cuda")
    out = fq.w4a4_gemm(dev(a), dev(qw["codes"]), dev(to_mma_layout(qw["scales"])),
                       dev(np.array([gw], np.float32)), a_rule=fq.FOUR_OVER_SIX, workspace=ws)
    assert fq.gemm_status(ws) == 0
    qa, ga = quantized_operand(O, a32, O.RULE_FOUR_OVER_SIX)
    check_gemm(out, O.nvfp4_decode_exact(qa["codes"], qa["scales"]), O.nvfp4_decode_exact(qw["codes"], qw["scales"]),
               float(ga) * float(gw), K, "nvfp4 fused act quant " + dtype)
    # the fused quantizer's outputs in the workspace are the oracle's, bit for bit
    wsh = ws.cpu().numpy()
    assert wsh[4096:4100].view(np.float32)[0] == ga
    assert np.array_equal(wsh[8192:8192 + M * K // 2], qa["codes"].reshape(-1))
    assert np.array_equal(wsh[8192 + M * K // 2:8192 + M * K // 2 + M * K // 16], to_mma_layout(qa["scales"]))


def test_gemm_rejects_unsupported_shapes():
    L = fq.lib()
    fake = ctypes.c_void_p(0x10000)
    for M, N, K in ((100, 256, 256), (128, 200, 256), (128, 256, 100), (0, 256, 256)):
        st = L.w4a4_gemm(fake, fq.NVFP4_PACKED, 0, fake, fake, fake, fake, fake, M, N, K, fake, fq.BF16, fake, 1 << 20, None)
        assert st in (1, 3), (M, N, K, st)


@pytest.mark.parametrize("out_dtype", [fq.BF16, fq.F32])
def test_gemm_full_size_sampled(O, out_dtype):
    """M=8192 tokens x K=4096 x N=14336: dynamic 4-over-6 activations, abs-max
    weights; one row of every 128-row band against all 14336 columns."""
    M, N, K = 8192, 14336, 4096
    a = inputs.generate("gemm_act")
    w32 = inputs.as_f32(inputs.generate("gemm_weight"))
    qw, gw = quantized_operand(O, w32, O.RULE_ABSMAX)
    ws = torch.empty(fq.workspace_size(fq.OP_GEMM, M, K, N), dtype=torch.uint8, device="cuda")
    out = fq.w4a4_gemm(dev(a), dev(qw["codes"]), dev(to_mma_layout(qw["scales"])),
                       dev(np.array([gw], np.float32)), a_rule=fq.FOUR_OVER_SIX, workspace=ws,
                       out_dtype=out_dtype)
    assert fq.gemm_status(ws) == 0
    a32 = inputs.as_f32(a)
    ga = O.global_scale(O.amax(a32))
    rows = band_rows(M, salt=out_dtype)
    qa = O.nvfp4_quantize(a32[rows], 16, O.RULE_FOUR_OVER_SIX, g=ga, want_deq=False, want_mse=False)
    check_gemm(out[torch.from_numpy(rows).cuda()], O.nvfp4_decode_exact(qa["codes"], qa["scales"]),
               O.nvfp4_decode_exact(qw["codes"], qw["scales"]), float(ga) * float(gw), K,
               "nvfp4 full 8192x14336x4096")
