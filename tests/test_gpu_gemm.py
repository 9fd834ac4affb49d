"""GPU parity of the tcgen05 W4A4 GEMM against the oracle's fp64 product of
the exactly decoded NVFP4 operands.

Bar: relative Frobenius error against the bf16-rounded fp64 reference
<= 1e-3 (bf16 output rounding alone is ~1.5e-3 against the raw fp64 value,
so the raw-reference error is reported, and bounded at 4e-3).
"""
import ctypes

import numpy as np
import pytest
import torch

from block_scaled_fp4_03_b200 import binding as fq
from block_scaled_fp4_03_b200 import inputs

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


def bf16_round(x64):
    f = x64.astype(np.float32)
    return inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits(f)).astype(np.float64)


def check(gpu_bf16, ref64, tol=1e-3):
    got = gpu_bf16.float().cpu().numpy().astype(np.float64)
    ref_b = bf16_round(ref64)
    den = np.linalg.norm(ref64)
    e_b = np.linalg.norm(got - ref_b) / den
    e_raw = np.linalg.norm(got - ref64) / den
    assert np.isfinite(got).all()
    assert e_b <= tol, (e_b, e_raw)
    assert e_raw <= 4e-3, (e_b, e_raw)
    return e_b, e_raw


def dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def quantized_operand(O, x32, rule):
    g = O.global_scale(O.amax(x32))
    q = O.nvfp4_quantize(x32, 16, rule, g=g, want_deq=False, want_mse=False)
    return q, g


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (256, 512, 512), (384, 768, 2048), (2048, 4096, 512)])
def test_gemm_packed_operands(O, M, N, K):
    a32 = inputs.as_f32(inputs.generate("gemm_act", M, K, seed=M + K))
    w32 = inputs.as_f32(inputs.generate("gemm_weight", N, K, seed=N + K))
    qa, ga = quantized_operand(O, a32, O.RULE_FOUR_OVER_SIX)
    qw, gw = quantized_operand(O, w32, O.RULE_ABSMAX)
    out = fq.w4a4_gemm(dev(qa["codes"]), dev(qw["codes"]), dev(to_mma_layout(qw["scales"])),
                       dev(np.array([gw], np.float32)), a_scales=dev(to_mma_layout(qa["scales"])),
                       a_global_scale=dev(np.array([ga], np.float32)))
    torch.cuda.synchronize()
    rows = np.arange(M) if M <= 512 else np.sort(np.random.default_rng(0).choice(M, 96, replace=False))
    ref = O.gemm_ref(qa["codes"], qa["scales"], ga, qw["codes"], qw["scales"], gw, rows=rows)
    check(out[torch.from_numpy(rows).cuda()], ref)


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
    ref = O.gemm_ref(qa["codes"], qa["scales"], ga, qw["codes"], qw["scales"], gw)
    check(out, ref)
    # the fused quantizer's outputs in the workspace are the oracle's, bit for bit
    wsh = ws.cpu().numpy()
    assert wsh[4096:4100].view(np.float32)[0] == ga
    assert np.array_equal(wsh[8192:8192 + M * K // 2], qa["codes"].reshape(-1))
    assert np.array_equal(wsh[8192 + M * K // 2:8192 + M * K // 2 + M * K // 16], to_mma_layout(qa["scales"]))


def test_gemm_rejects_unsupported_shapes():
    L = fq.lib()
    fake = ctypes.c_void_p(0x10000)
    for M, N, K in ((100, 256, 256), (128, 200, 256), (128, 256, 100), (0, 256, 256)):
        st = L.w4a4_gemm(fake, fq.NVFP4_PACKED, 0, fake, fake, fake, fake, fake, M, N, K, fake, fake, 1 << 20, None)
        assert st in (1, 3), (M, N, K, st)


def test_gemm_full_size_sampled(O):
    """M=8192 tokens x K=4096 x N=14336: dynamic 4-over-6 activations, abs-max weights."""
    M, N, K = 8192, 14336, 4096
    a = inputs.generate("gemm_act")
    w32 = inputs.as_f32(inputs.generate("gemm_weight"))
    qw, gw = quantized_operand(O, w32, O.RULE_ABSMAX)
    ws = torch.empty(fq.workspace_size(fq.OP_GEMM, M, K, N), dtype=torch.uint8, device="cuda")
    out = fq.w4a4_gemm(dev(a), dev(qw["codes"]), dev(to_mma_layout(qw["scales"])),
                       dev(np.array([gw], np.float32)), a_rule=fq.FOUR_OVER_SIX, workspace=ws)
    assert fq.gemm_status(ws) == 0
    a32 = inputs.as_f32(a)
    ga = O.global_scale(O.amax(a32))
    rows = np.sort(np.random.default_rng(1).choice(M, 48, replace=False))
    qa = O.nvfp4_quantize(a32[rows], 16, O.RULE_FOUR_OVER_SIX, g=ga, want_deq=False, want_mse=False)
    ref = O.gemm_ref(qa["codes"], qa["scales"], ga, qw["codes"], qw["scales"], gw)
    check(out[torch.from_numpy(rows).cuda()], ref)
    # one full row tile and one full column tile, to cover every M and N tile position
    cols = np.arange(0, N, 97)
    ref_c = O.gemm_ref(qa["codes"], qa["scales"], ga, qw["codes"], qw["scales"], gw, cols=cols)
    check(out[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()], ref_c)
