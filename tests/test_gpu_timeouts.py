"""Failure detection of the tensor-core kernels, exercised without a GPU fault.

Every wait of the GEMM kernels (single-CTA and CTA-pair) and of the Hessian
kernel on its own barriers is bounded.  With the process-wide debug limit set
to one cycle (fp4q_debug_set_wait_cycles), the first wait that is not
satisfied at once gives up: the kernel raises its abort flag, lets the copies
and MMAs it already issued finish (those waits keep the default limit),
releases its tensor memory and returns.  The host sees FP4Q_ERR_TIMEOUT from
the entry point's status call.  A normal call on the same workspace
afterwards must return FP4Q_OK with output bit-identical to a call made
before: the context stays usable.

The quantizers' fused global amax waits at a grid barrier, also bounded: a
CTA whose wait runs out computes the whole maximum itself, so its results do
not change at all (tested with the same one-cycle limit).
"""
import numpy as np
import pytest
import torch

from block_scaled_fp4_03_b200 import binding as fq
from block_scaled_fp4_03_b200 import inputs
from test_gpu_gemm import dev, quantized_operand, to_mma_layout

pytestmark = pytest.mark.gpu

TIMEOUT = 5


class short_waits:
    """Context manager: every bounded device wait gives up after one cycle."""

    def __enter__(self):
        self.prev = fq.debug_set_wait_cycles(1)

    def __exit__(self, *exc):
        fq.debug_set_wait_cycles(self.prev)


def gemm_operands(O, M, N, K):
    a32 = inputs.as_f32(inputs.generate("gemm_act", M, K, seed=40))
    w32 = inputs.as_f32(inputs.generate("gemm_weight", N, K, seed=41))
    qa, ga = quantized_operand(O, a32, O.RULE_FOUR_OVER_SIX)
    qw, gw = quantized_operand(O, w32, O.RULE_ABSMAX)
    args = (dev(qa["codes"]), dev(qw["codes"]), dev(to_mma_layout(qw["scales"])), dev(np.array([gw], np.float32)))
    kw = dict(a_scales=dev(to_mma_layout(qa["scales"])), a_global_scale=dev(np.array([ga], np.float32)))
    return args, kw


# M = 128: the single-CTA kernel; M = 256: the CTA-pair kernel.  K = 4096 gives
# each tile a 16-step main loop, so the epilogue's wait for the accumulator
# cannot be satisfied at its first test.
@pytest.mark.parametrize("M", [128, 256])
@pytest.mark.parametrize("mx", [False, True])
def test_gemm_wait_gives_up_and_reports_timeout(O, M, mx):
    N, K = 512, 4096
    ws = torch.zeros(8192, dtype=torch.uint8, device="cuda")
    if mx:
        x32 = inputs.as_f32(inputs.generate("mx_act", M, K, seed=42))
        w32 = inputs.as_f32(inputs.generate("mx_weight", N, K, seed=43))
        qa = O.mxfp4_quantize(x32, None, True, O.RULE_ABSMAX, want_deq=False, want_mse=False)
        qw = O.mxfp4_quantize(w32, None, True, O.RULE_ABSMAX, want_deq=False, want_mse=False)
        args = (dev(qa["codes"]), dev(qw["codes"]), dev(to_mma_layout(qw["scales"])))

        def run():
            return fq.mxfp4_gemm(*args, a_scales=dev(to_mma_layout(qa["scales"])), workspace=ws)
    else:
        args, kw = gemm_operands(O, M, N, K)

        def run():
            return fq.w4a4_gemm(*args, workspace=ws, **kw)
    ref = run()
    assert fq.gemm_status(ws) == 0
    with short_waits():
        run()
        st = fq.gemm_status(ws)
    assert st == TIMEOUT, st
    again = run()
    assert fq.gemm_status(ws) == 0
    assert torch.equal(again.view(torch.int16), ref.view(torch.int16))


def test_razer_two_pass_gemm_wait_gives_up(O):
    """The multi-pass K loop (RaZeR weights: two passes) winds down the same way."""
    M, N, K = 256, 512, 2048
    args, kw = gemm_operands(O, M, N, K)
    a_codes, w_codes, w_sc, gw = args
    ws = torch.zeros(8192, dtype=torch.uint8, device="cuda")

    def run():
        return fq.razer_w4a4_gemm(a_codes, kw["a_scales"], kw["a_global_scale"], w_codes, w_sc, gw,
                                  w_extra=w_codes, workspace=ws)
    ref = run()
    assert fq.gemm_status(ws) == 0
    with short_waits():
        run()
        st = fq.gemm_status(ws)
    assert st == TIMEOUT, st
    again = run()
    assert fq.gemm_status(ws) == 0
    assert torch.equal(again.view(torch.int16), ref.view(torch.int16))


def test_hessian_wait_gives_up_and_reports_timeout():
    """H' blocks: the CTAs that gave up leave NaN blocks and the error word set."""
    rows, cols = 2048, 256
    x = dev(inputs.generate("mx_act", rows, cols, seed=44))
    t = dev(inputs.positive_vector(cols, seed=45))
    ws = torch.empty(fq.workspace_size(fq.OP_HESSIAN, rows, cols), dtype=torch.uint8, device="cuda")
    ref = fq.hessian_blocks(x, t, True, workspace=ws)
    assert fq.hessian_status(ws) == 0
    assert torch.isfinite(ref).all()
    with short_waits():
        bad = fq.hessian_blocks(x, t, True, workspace=ws)
        st = fq.hessian_status(ws)
    assert st == TIMEOUT, st
    assert torch.isnan(bad).any()
    again = fq.hessian_blocks(x, t, True, workspace=ws)
    assert fq.hessian_status(ws) == 0
    assert torch.equal(again.view(torch.int32), ref.view(torch.int32))


@pytest.mark.parametrize("kind,rule,B", [("gaussian", fq.PREVENT_ZERO, 16), ("gemm_act", fq.FOUR_OVER_SIX, 16),
                                         ("student_t", fq.BRUTE_FORCE, 8)])
def test_fused_amax_barrier_fallback_keeps_results(O, kind, rule, B):
    """The hierarchical (AMAX) global scale is reduced inside the quantizer
    launch behind a grid barrier.  With the barrier's wait limited to one cycle
    the CTAs that give up take the maximum of the whole tensor themselves: g,
    codes, scales and errors must not change."""
    from test_gpu_parity import make, assert_bits
    x, x32 = make(kind, 1000, 512, seed=7, dtype="bf16" if kind == "gemm_act" else "f32")
    ref = O.nvfp4_quantize(x32, B, rule, g=O.global_scale(O.amax(x32)))
    normal = fq.nvfp4_quantize(x, B, rule, gs_mode=fq.GS_AMAX, mse=True)
    with short_waits():
        alone = fq.nvfp4_quantize(x, B, rule, gs_mode=fq.GS_AMAX, mse=True)
        torch.cuda.synchronize()
    for r in (normal, alone):
        assert_bits(r["global_scale"], np.array([O.global_scale(O.amax(x32))], np.float32), "g")
        assert_bits(r["codes"], ref["codes"], "codes")
        assert_bits(r["scales"], ref["scales"], "scales")
        assert_bits(r["mse"], ref["mse"], "mse")



class separate_amax_pass:
    """Context manager: hierarchical global scales through the separate amax pass."""

    def __enter__(self):
        self.prev = fq.debug_force_amax_pass(True)

    def __exit__(self, *exc):
        fq.debug_force_amax_pass(self.prev)


@pytest.mark.parametrize("kind,rule,B", [("gaussian", fq.PREVENT_ZERO, 16), ("student_t", fq.FOUR_OVER_SIX, 4),
                                         ("student_t", fq.BRUTE_FORCE, 32)])
def test_separate_amax_pass_matches_fused(O, kind, rule, B):
    """The path taken when the quantizer cannot be launched cooperatively: a
    separate amax pass (amax_kernel) writes partial maxima, the quantizer
    reduces them.  g, codes, scales and errors equal the fused path's and the
    oracle's."""
    from test_gpu_parity import make, assert_bits
    x, x32 = make(kind, 777, 512, seed=11, dtype="f32")
    g = np.array([O.global_scale(O.amax(x32))], np.float32)
    ref = O.nvfp4_quantize(x32, B, rule, g=g[0])
    fused = fq.nvfp4_quantize(x, B, rule, gs_mode=fq.GS_AMAX, mse=True)
    with separate_amax_pass():
        alone = fq.nvfp4_quantize(x, B, rule, gs_mode=fq.GS_AMAX, mse=True)
        torch.cuda.synchronize()
    for r in (fused, alone):
        assert_bits(r["global_scale"], g, "g")
        assert_bits(r["codes"], ref["codes"], "codes")
        assert_bits(r["scales"], ref["scales"], "scales")
        assert_bits(r["mse"], ref["mse"], "mse")


def test_separate_amax_pass_razer_and_gemm_activations(O):
    """The same fallback for a RaZeR quantizer and for the W4A4 GEMM's dense
    activations: results equal the fused path's bit for bit."""
    from test_gpu_parity import make
    x, _ = make("razer_act", 512, 256, seed=12, dtype="bf16")
    fused = fq.razer_quantize(x, fq.SF_E4M3, [5.0, -5.0], gs_mode=fq.GS_AMAX, mse=True)
    with separate_amax_pass():
        alone = fq.razer_quantize(x, fq.SF_E4M3, [5.0, -5.0], gs_mode=fq.GS_AMAX, mse=True)
        torch.cuda.synchronize()
    for k in ("codes", "meta", "mse", "global_scale"):
        assert torch.equal(fused[k].view(torch.uint8), alone[k].view(torch.uint8)), k
    M, N, K = 256, 512, 1024
    a = torch.from_numpy(inputs.generate("gemm_act", M, K, seed=13).view(np.int16)).cuda().view(torch.bfloat16)
    w32 = inputs.as_f32(inputs.generate("gemm_weight", N, K, seed=14))
    qw, gw = quantized_operand(O, w32, O.RULE_ABSMAX)
    wargs = (dev(qw["codes"]), dev(to_mma_layout(qw["scales"])), dev(np.array([gw], np.float32)))
    y0 = fq.w4a4_gemm(a, *wargs)
    with separate_amax_pass():
        y1 = fq.w4a4_gemm(a, *wargs)
        torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
