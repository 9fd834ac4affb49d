"""Benchmark of the block-scaled FP4 hot path on B200.

One step = one pass over every hot-path row at its workload size:
  c1  NVFP4 prevent-zero quantize, 4096x4096 fp32 N(0,1), block 16,
      hierarchical scale, with dequant + per-block MSE        (amax, quantize)
  c2  block sizes {4,8,16,32} x rules {abs-max, prevent-zero, 4-over-6,
      brute force} on 8192x8192 fp32 Student-t(3)*1e-3, g = 1, codes +
      scales + per-block MSE                                  (16 quantizations),
      and, as next rows outside the step, per block size the scale-format
      comparison: UE5M3 abs-max and 4-over-6 (g = 1) against E4M3 4-over-6
      with hierarchical scaling
  c3  RaZeR: 8192x8192 bf16 weights (E3M3 + 4 specials) and 16384x4096 bf16
      activations (E4M3 + 2 specials), hierarchical scale
  c4  MXFP4 prep: channel scale t from 8192x4096 bf16 activations and
      4096x4096 bf16 weights, Hessian blocks H', activation quantize (t,
      Hadamard-32, E8M0), weight quantize with the Hessian-weighted exponent;
      as a next row outside the step, Flip-Refinement of the weight codes
      (128 moves per row)
  c5  W4A4 GEMM M=8192 x K=4096 x N=14336 -> bf16: dynamic 4-over-6 NVFP4
      quantize of the bf16 activations into the MMA scale layout, then the
      tcgen05 block-scaled GEMM on weights quantized once beforehand
Inputs are synthetic and seeded (block_scaled_fp4_03_b200.inputs), resident in
HBM when timing starts; L2 is flushed (a 512 MiB write) before every step.

The JSON line's value is elements quantized per second over the whole step
(Gelem/s, all ranks; the GEMM's time is part of the step); per-row times,
bandwidths, TFLOP/s and roofline fractions are in "rows", the GEMM's
TFLOP/s and FP4-peak fraction also under "gemm".  `--impl reference` times the plain CPU oracle on a bounded sample of
the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FP4 quantize Gelem/s & % of HBM roofline; W4A4 GEMM TFLOP/s & % FP4 peak"
WORKLOAD = "hot path: one pass of every row (NVFP4 4096^2 PZ; 8192^2 block-size x rule sweep; RaZeR W 8192^2 + A 16384x4096; MXFP4 prep 8192x4096 + 4096^2; W4A4 GEMM 8192x14336x4096 with 4-over-6 activation quant)"
SM_COUNT = 148
FP32_LANES_PER_SM = 128


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return (float(d["hbm_gbs"]), float(d.get("sm_max_mhz", 1965.0)), float(d["bf16_tflops"]),
                float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured")
    except Exception:
        return 6650.0, 1965.0, 1590.0, 1400.0, "fallback"


# Per-launch DRAM traffic of a row's kernel, from the committed ncu summary of
# that kernel on the same workload (profiles/*.md); rows without one report null.
PROFILE_OF_ROW = {
    "c1_nvfp4_pz_deq_mse": "nvfp4_quant_kernel_B16_pz_deq_mse_gaussian_4096x4096.md",
    "c1_dequant_mse": "dequant_kernel_B16_e4m3_gaussian_4096x4096.md",
    "c2_B4_bf": "nvfp4_bf_kernel_B4_student_t_8192x8192.md",
    "c2_B8_bf": "nvfp4_bf_kernel_B8_student_t_8192x8192.md",
    "c2_B16_bf": "nvfp4_bf_kernel_B16_student_t_8192x8192.md",
    "c2_B32_bf": "nvfp4_bf_kernel_B32_student_t_8192x8192.md",
    "c2_B4_4o6": "nvfp4_quant_kernel_B4_4o6_student_t_8192x8192.md",
    "c2_B16_absmax": "nvfp4_quant_kernel_B16_absmax_student_t_8192x8192.md",
    "c3_razer_weight": "razer_paired_kernel_weights_8192x8192_bf16.md",
    "c3_razer_act": "razer_paired_kernel_acts_16384x4096_bf16.md",
    "c4_channel_scale": "column_stats_kernel_weights_4096x4096_acts_8192x4096_bf16.md",
    "c4_mx_act": "mx_quant_absmax2_kernel_acts_8192x4096_bf16.md",
    "c4_mx_weight_hessian": "mx_quant_hessian_kernel_weights_4096x4096_bf16.md",
    "c4_hessian_blocks": "hessian_partial_tc_kernel_acts_8192x4096_bf16.md",
    "c4_mx_weight_flip": "flip_blocks_kernel_weights_4096x4096_bf16.md",
    "c5_act_quant_4o6_mma": "nvfp4_quant_kernel_B16_4o6_bf16_mma_layout_8192x4096.md",
    "c5_w4a4_gemm": "w4a4_gemm_2sm_kernel_M8192_N14336_K4096.md",
    "f2_razer_prepare_weights": "razer_prepare_kernel_weights_14336x4096.md",
    "f2_razer_gemm_w_2pass": "w4a4_gemm_2sm_kernel_razer_2pass_M8192_N14336_K4096.md",
    "f3_mx_gemm_packed": "w4a4_gemm_2sm_kernel_mxf4_M8192_N16384_K4096.md",
}


def profiled_traffic(row_name):
    """DRAM bytes per launch recorded in the row's ncu summary, or None."""
    import re
    f = PROFILE_OF_ROW.get(row_name)
    if not f:
        return None
    try:
        with open(os.path.join(ROOT, "profiles", f)) as fh:
            m = re.search(r"DRAM traffic \(read \+ write\): ([0-9.]+) MB per launch", fh.read())
        return float(m.group(1)) * 1e6 if m else None
    except OSError:
        return None


# ----------------------------------------------------------------------------- rows
class Row:
    """One hot-path row: how to launch it on device buffers and what it moves."""

    def __init__(self, name, kernel, units, bytes_, launches, fn, out, bound="hbm", flops=0.0, evals=0.0,
                 eval_ws=None, block=0, extra=False, standalone=False):
        self.name, self.kernel, self.units, self.bytes, self.launches = name, kernel, units, bytes_, launches
        self.fn, self.out, self.bound, self.flops, self.evals = fn, out, bound, flops, evals
        # brute force: workspace whose counter at FP4Q_WS_BF_EVALS receives the
        # number of (block, candidate) error evaluations a call performs
        self.eval_ws, self.block = eval_ws, block
        # rows beyond the hot path proper (the next rows built on it, and the
        # standalone form of a step that the hot path runs fused): timed and
        # reported per row, outside the step and its value
        self.extra = extra
        self.standalone = standalone
        # the step's input tensors (keys of X) this row reads; set per workload
        self.inputs = []


def build_rows(torch, fq, inputs, dev, host_copies=None, groups=None):
    """Create the step's device buffers and rows.  host_copies (dict) receives
    the host arrays that an end-to-end run copies in each step; groups (a set
    of "c1".."c5", default all) limits which workloads are built."""
    def to_dev(a, key):
        if host_copies is not None:
            host_copies[key] = a
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    rows = []
    X = {}

    def set_inputs(start, keys):
        for r in rows[start:]:
            r.inputs = list(keys)
    n0 = len(rows)
    if groups is None or "c1" in groups:
        # c1
        a1 = inputs.generate("gaussian")
        X["c1"] = to_dev(a1, "c1")
        n1 = a1.size
        o1 = {}
        ws1 = torch.empty(fq.workspace_size(fq.OP_QUANTIZE, *a1.shape), dtype=torch.uint8, device=dev)

        def c1():
            o1.update(fq.nvfp4_quantize(X["c1"], 16, fq.PREVENT_ZERO, gs_mode=fq.GS_AMAX, dequant=True,
                                        mse=True, out=o1, workspace=ws1))
        rows.append(Row("c1_nvfp4_pz_deq_mse", "nvfp4_quant_kernel<16, float, 1, 0, true>", n1, n1 * (4 + 0.5 + 1 / 16 + 4 + 4 / 16), 2, c1, o1))
        # the standalone dequantizer (fp4_dequant_mse) on that output: codes,
        # scales and g in, the reference x in for the MSE, dequant and MSE out
        od1 = {"dequant": torch.empty(a1.shape, dtype=torch.float32, device=dev),
               "mse": torch.empty((a1.shape[0], a1.shape[1] // 16), dtype=torch.float32, device=dev)}

        def c1d():
            fq.dequant_mse(o1["codes"], o1["scales"], a1.shape[0], a1.shape[1], 16, fq.SF_E4M3,
                           global_scale=o1["global_scale"], ref=X["c1"], out=od1)
        rows.append(Row("c1_dequant_mse", "dequant_kernel<16, 0, false, float>", n1,
                        n1 * (0.5 + 1 / 16 + 4 + 4 + 4 / 16), 1, c1d, od1, extra=True, standalone=True))
    set_inputs(n0, [k for k in ("c1",) if k in X])
    n0 = len(rows)
    if groups is None or "c2" in groups:
        # c2
        a2 = inputs.generate("student_t")
        X["c2"] = to_dev(a2, "c2")
        n2 = a2.size
        names = {fq.ABSMAX: "absmax", fq.PREVENT_ZERO: "pz", fq.FOUR_OVER_SIX: "4o6", fq.BRUTE_FORCE: "bf"}
        for B in (4, 8, 16, 32):
            for rule in (fq.ABSMAX, fq.PREVENT_ZERO, fq.FOUR_OVER_SIX, fq.BRUTE_FORCE):
                o = {}
                bf = rule == fq.BRUTE_FORCE
                wsr = torch.zeros(fq.workspace_size(fq.OP_QUANTIZE, 1, 1), dtype=torch.uint8, device=dev) if bf else None

                def c2(B=B, rule=rule, o=o, wsr=wsr):
                    o.update(fq.nvfp4_quantize(X["c2"], B, rule, gs_mode=fq.GS_NONE, mse=True, out=o, workspace=wsr))
                kern = ("nvfp4_bf_kernel<%d, float, 0, false>" % B) if bf else ("nvfp4_quant_kernel<%d, float, %d, 0, false>" % (B, rule))
                # brute force is held to the HBM roofline like the other rules (the
                # evaluations it performs are reported beside it, not as its bound)
                rows.append(Row("c2_B%d_%s" % (B, names[rule]), kern,
                                n2, n2 * (4 + 0.5 + 1 / B + 4 / B), 1, c2, o,
                                bound="hbm", eval_ws=wsr, block=B))
        # the summary's comparison: UE5M3 block scales without a global scale
        # against E4M3 with 4-over-6 and hierarchical (global) scaling
        wsh2 = torch.empty(fq.workspace_size(fq.OP_QUANTIZE, 1, 1), dtype=torch.uint8, device=dev)
        for B in (4, 8, 16, 32):
            for tag, rule, sfmt, gsm in (("ue5m3_absmax", fq.ABSMAX, fq.SF_UE5M3, fq.GS_NONE),
                                         ("ue5m3_4o6", fq.FOUR_OVER_SIX, fq.SF_UE5M3, fq.GS_NONE),
                                         ("e4m3_4o6_hier", fq.FOUR_OVER_SIX, fq.SF_E4M3, fq.GS_AMAX)):
                o = {}

                def c2x(B=B, rule=rule, sfmt=sfmt, gsm=gsm, o=o):
                    o.update(fq.nvfp4_quantize(X["c2"], B, rule, gs_mode=gsm, mse=True, out=o, scale_fmt=sfmt,
                                               workspace=wsh2 if gsm == fq.GS_AMAX else None))
                rows.append(Row("c2_B%d_%s" % (B, tag),
                                "nvfp4_quant_kernel<%d, float, %d, %d, false>" % (B, rule, 1 if sfmt == fq.SF_UE5M3 else 0),
                                n2, n2 * (4 + 0.5 + 1 / B + 4 / B), 2 if gsm == fq.GS_AMAX else 1, c2x, o, extra=True))
    set_inputs(n0, [k for k in ("c2",) if k in X])
    n0 = len(rows)
    if groups is None or "c3" in groups:
        # c3
        w3 = inputs.generate("razer_weight")
        X["c3w"] = to_dev(w3, "c3w")
        a3 = inputs.generate("razer_act")
        X["c3a"] = to_dev(a3, "c3a")
        ws3 = torch.empty(fq.workspace_size(fq.OP_QUANTIZE, 1, 1), dtype=torch.uint8, device=dev)
        o3w, o3a = {}, {}

        def c3w():
            o3w.update(fq.razer_quantize(X["c3w"], fq.SF_E3M3, [5.0, -5.0, 3.5, -3.5], gs_mode=fq.GS_AMAX, out=o3w, workspace=ws3))

        def c3a():
            o3a.update(fq.razer_quantize(X["c3a"], fq.SF_E4M3, [5.0, -5.0], gs_mode=fq.GS_AMAX, out=o3a, workspace=ws3))
        rows.append(Row("c3_razer_weight", "razer_paired_kernel<__nv_bfloat16, 1, 2>", w3.size, w3.size * (2 + 0.5 + 1 / 16), 2, c3w, o3w))
        rows.append(Row("c3_razer_act", "razer_paired_kernel<__nv_bfloat16, 0, 1>", a3.size, a3.size * (2 + 0.5 + 1 / 16), 2, c3a, o3a))
    for r in rows[n0:]:
        r.inputs = ["c3w"] if "weight" in r.name else ["c3a"]
    n0 = len(rows)
    if groups is None or "c4" in groups:
        # c4
        x4 = inputs.generate("mx_act")
        w4 = inputs.generate("mx_weight")
        X["c4x"] = to_dev(x4, "c4x")
        X["c4w"] = to_dev(w4, "c4w")
        T, C = x4.shape
        N4 = w4.shape[0]
        t4 = torch.empty(C, dtype=torch.float32, device=dev)
        ti4 = torch.empty(C, dtype=torch.float32, device=dev)
        h4 = torch.empty((C // 32, 32, 32), dtype=torch.float32, device=dev)
        wsc = torch.empty(fq.workspace_size(fq.OP_CHANNEL_SCALE, T, C, N4), dtype=torch.uint8, device=dev)
        wsh = torch.empty(fq.workspace_size(fq.OP_HESSIAN, T, C), dtype=torch.uint8, device=dev)
        o4a, o4w = {}, {}

        def c4s():
            fq.channel_scale(X["c4x"], X["c4w"], 0.75, out=(t4, ti4), workspace=wsc)

        def c4h():
            fq.hessian_blocks(X["c4x"], t4, True, out=h4, workspace=wsh)

        def c4a():
            o4a.update(fq.mxfp4_quantize(X["c4x"], t4, True, fq.ABSMAX, out=o4a))

        def c4w():
            o4w.update(fq.mxfp4_quantize(X["c4w"], ti4, True, fq.HESSIAN_EXP, hess=h4, out=o4w))
        rows.append(Row("c4_channel_scale", "column_stats_kernel", 0, x4.size * 2 + w4.size * 2, 2, c4s, {"t": t4, "t_inv": ti4}))
        rows.append(Row("c4_hessian_blocks", "hessian_partial_kernel", 0, x4.size * 2 + C * 32 * 4, 2, c4h,
                        {"hess": h4}, flops=2.0 * T * C * 32))
        rows.append(Row("c4_mx_act", "mx_quant_absmax_kernel", x4.size, x4.size * (2 + 0.5 + 1 / 32), 1, c4a, o4a))
        rows.append(Row("c4_mx_weight_hessian", "mx_quant_hessian_kernel", w4.size, w4.size * (2 + 0.5 + 1 / 32) + C * 32 * 4,
                        1, c4w, o4w, bound="alu", flops=2.0 * 3 * N4 * (C // 32) * 32 * 32))
        # Flip-Refinement of those weight codes, the pages' K = 128 moves per row
        mv4 = torch.empty(N4, dtype=torch.int32, device=dev)
        wsf = torch.empty(fq.workspace_size(fq.OP_FLIP, N4, C), dtype=torch.uint8, device=dev)

        def c4f():
            fq.mxfp4_flip_refine(X["c4w"], o4w["codes"], o4w["scales"], h4, chan_scale=ti4, max_moves=128, moves=mv4,
                                 workspace=wsf)
        rows.append(Row("c4_mx_weight_flip", "flip_refine_kernel", 0, w4.size * (2 + 0.5 + 0.5 + 1 / 32) + C * 32 * 4,
                        1, c4f, {"moves": mv4}, bound="alu", flops=2.0 * N4 * (C // 32) * 32 * 32, extra=True))

        # MXFP4 GEMM (next rows) at the size the MACaQ review quotes the online
        # transform's overhead at: these activations (8192 x 4096) against
        # 16384 x 4096 MXFP4 weights (1/t, rotation, quantized once, offline).
        # (a) packed activations: the GEMM alone; (b) dense bf16 activations:
        # the prologue (x * t, rotation, E8M0, the GEMM's scale layout) + GEMM.
        N3 = 16384
        w3d = torch.from_numpy(inputs.generate("mx_weight", N3, C, seed=3).view(np.int16)).to(dev).view(torch.bfloat16)
        t3 = torch.from_numpy(inputs.positive_vector(C, seed=3)).to(dev)
        ti3 = 1.0 / t3.double()
        ti3 = ti3.float()
        qw3 = fq.mxfp4_quantize(w3d, ti3, True, fq.ABSMAX)
        del w3d
        w3sc = fq.scales_to_mma(qw3["scales"])
        qa3 = fq.mxfp4_quantize(X["c4x"], t3, True, fq.ABSMAX)
        a3sc = fq.scales_to_mma(qa3["scales"])
        y3 = torch.empty((T, N3), dtype=torch.bfloat16, device=dev)
        ws3 = torch.empty(fq.workspace_size(fq.OP_MX_GEMM, T, C, N3), dtype=torch.uint8, device=dev)

        def f3p():
            fq.mxfp4_gemm(qa3["codes"], qw3["codes"], w3sc, a_scales=a3sc, out=y3, workspace=ws3)

        def f3d():
            fq.mxfp4_gemm(X["c4x"], qw3["codes"], w3sc, chan_scale=t3, out=y3, workspace=ws3)
        mxg_bytes = T * C * (0.5 + 1 / 32) + N3 * C * (0.5 + 1 / 32) + T * N3 * 2
        rows.append(Row("f3_mx_gemm_packed", "w4a4_gemm_2sm_kernel<true>", 0, mxg_bytes, 1, f3p, {"out": y3},
                        bound="tensor", flops=2.0 * T * N3 * C, extra=True))
        rows.append(Row("f3_mx_gemm_with_prologue", "mx_quant_absmax_kernel + w4a4_gemm_2sm_kernel<true>", 0,
                        mxg_bytes + T * C * 2, 2, f3d, {"out": y3}, bound="tensor", flops=2.0 * T * N3 * C,
                        extra=True))
    set_inputs(n0, [k for k in ("c4x", "c4w") if k in X])
    n0 = len(rows)
    if groups is None or "c5" in groups:
        # c5: weights pre-quantized once (abs-max NVFP4, hierarchical scale, MMA
        # scale layout) outside the timed step; the step quantizes the activations
        # (4-over-6, MMA layout) and runs the tcgen05 GEMM on the packed operands
        a5 = inputs.generate("gemm_act")
        X["c5"] = to_dev(a5, "c5")
        w5 = inputs.generate("gemm_weight")
        w5d = torch.from_numpy(w5.view(np.int16)).to(dev).view(torch.bfloat16)
        M5, K5 = a5.shape
        N5 = w5.shape[0]
        qw5 = fq.nvfp4_quantize(w5d, 16, fq.ABSMAX, gs_mode=fq.GS_AMAX, sf_layout=fq.SF_MMA)
        del w5d
        ws5 = torch.empty(fq.workspace_size(fq.OP_QUANTIZE, 1, 1), dtype=torch.uint8, device=dev)
        wsg = torch.empty(fq.workspace_size(fq.OP_GEMM, 128, 256, 256), dtype=torch.uint8, device=dev)
        o5 = {}
        y5 = torch.empty((M5, N5), dtype=torch.bfloat16, device=dev)

        def c5():
            o5.update(fq.nvfp4_quantize(X["c5"], 16, fq.FOUR_OVER_SIX, gs_mode=fq.GS_AMAX, sf_layout=fq.SF_MMA,
                                        out=o5, workspace=ws5))

        def c5g():
            fq.w4a4_gemm(o5["codes"], qw5["codes"], qw5["scales"], qw5["global_scale"], a_scales=o5["scales"],
                         a_global_scale=o5["global_scale"], K=K5, out=y5, workspace=wsg)
        rows.append(Row("c5_act_quant_4o6_mma", "nvfp4_quant_kernel<16, __nv_bfloat16, 2, 0, false>", a5.size, a5.size * (2 + 0.5 + 1 / 16), 2, c5, o5))
        rows.append(Row("c5_w4a4_gemm", "w4a4_gemm_2sm_kernel<false>", 0, M5 * K5 * (0.5 + 1 / 16) + N5 * K5 * (0.5 + 1 / 16) + M5 * N5 * 2,
                        1, c5g, {"out": y5}, bound="tensor", flops=2.0 * M5 * N5 * K5))

        # RaZeR-aware GEMM (next rows): the same weights quantized with RaZeR
        # (E3M3 scale, +-5 / +-3.5) and split into two E2M1 tensors once, offline;
        # (a) with the step's 4-over-6 NVFP4 activations: 2 passes over K;
        # (b) with RaZeR activations (E4M3, +-5) quantized and split per call: 4 passes
        spw, spa = [5.0, -5.0, 3.5, -3.5], [5.0, -5.0]
        w5d = torch.from_numpy(w5.view(np.int16)).to(dev).view(torch.bfloat16)
        rw5 = fq.razer_quantize(w5d, fq.SF_E3M3, spw, gs_mode=fq.GS_AMAX)
        del w5d
        pw5 = fq.razer_gemm_prepare(rw5["codes"], rw5["meta"], fq.SF_E3M3, spw)
        pwo = {"main": pw5["main"], "extra": pw5["extra"], "scales": pw5["scales"]}
        wsr = torch.empty(8192, dtype=torch.uint8, device=dev)
        ra5, pa5 = {}, {}

        def f2p():
            fq.razer_gemm_prepare(rw5["codes"], rw5["meta"], fq.SF_E3M3, spw, out=pwo)

        def f2w():
            fq.razer_w4a4_gemm(o5["codes"], o5["scales"], o5["global_scale"], pw5["main"], pw5["scales"],
                               rw5["global_scale"], w_extra=pw5["extra"], out=y5, workspace=wsr)

        def f2aq():
            ra5.update(fq.razer_quantize(X["c5"], fq.SF_E4M3, spa, gs_mode=fq.GS_AMAX, out=ra5, workspace=ws5))
            pa5.update(fq.razer_gemm_prepare(ra5["codes"], ra5["meta"], fq.SF_E4M3, spa, out=pa5))

        def f2wa():
            fq.razer_w4a4_gemm(pa5["main"], pa5["scales"], ra5["global_scale"], pw5["main"], pw5["scales"],
                               rw5["global_scale"], a_extra=pa5["extra"], w_extra=pw5["extra"], out=y5,
                               workspace=wsr)
        rows.append(Row("f2_razer_prepare_weights", "razer_prepare_kernel<1>", N5 * K5,
                        N5 * K5 * (0.5 + 1 / 16) + N5 * K5 * (0.5 + 0.5 + 1 / 16), 1, f2p, pwo, extra=True))
        rows.append(Row("f2_razer_gemm_w_2pass", "w4a4_gemm_2sm_kernel<false>", 0,
                        M5 * K5 * (0.5 + 1 / 16) + N5 * K5 * (1.0 + 1 / 16) + M5 * N5 * 2, 1, f2w, {"out": y5},
                        bound="tensor", flops=2.0 * M5 * N5 * K5, extra=True))
        rows.append(Row("f2_razer_act_quant_prep", "razer_paired_kernel<__nv_bfloat16, 0, 1>", a5.size,
                        a5.size * (2 + 0.5 + 1 / 16) + a5.size * (0.5 + 1 / 16 + 1.0 + 1 / 16), 3, f2aq, pa5,
                        extra=True))
        rows.append(Row("f2_razer_gemm_wa_4pass", "w4a4_gemm_2sm_kernel<false>", 0,
                        M5 * K5 * (1.0 + 1 / 16) + N5 * K5 * (1.0 + 1 / 16) + M5 * N5 * 2, 1, f2wa, {"out": y5},
                        bound="tensor", flops=2.0 * M5 * N5 * K5, extra=True))
    set_inputs(n0, [k for k in ("c5",) if k in X])
    return rows, X


# ------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = "index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap"

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        self.t0 = time.perf_counter()
        try:
            fd, self.path = tempfile.mkstemp(prefix="fp4q_clocks_", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            p = [v.strip() for v in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                smax.append(float(p[2]))
            except ValueError:
                continue
            for nm, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------- reference arm
def oracle_sample_inputs(inputs, frac_rows):
    """Leading rows of every input (a bounded sample of the step's workload), fp32."""
    def sub(kind, frac):
        a = inputs.as_f32(inputs.generate(kind))
        r = max(1, int(round(a.shape[0] * frac)))
        return np.ascontiguousarray(a[:r])

    return {"c1": sub("gaussian", frac_rows["c1"]), "c2": sub("student_t", frac_rows["c2"]),
            "c3w": sub("razer_weight", frac_rows["c3"]), "c3a": sub("razer_act", frac_rows["c3"]),
            "c4x": sub("mx_act", frac_rows["c4"]), "c4w": sub("mx_weight", frac_rows["c4"]),
            "c5": sub("gemm_act", frac_rows["c5"]), "c5w": inputs.as_f32(inputs.generate("gemm_weight"))}


def oracle_prepare(O, S):
    """Weights of the GEMM row quantized once (abs-max, hierarchical), outside the timed step."""
    if "c5q" not in S:
        gw = O.global_scale(O.amax(S["c5w"]))
        S["c5q"] = (O.nvfp4_quantize(S["c5w"], 16, O.RULE_ABSMAX, g=gw, want_deq=False, want_mse=False), gw)
    return S


def oracle_sample_run(O, S):
    """One step of the CPU oracle over the sampled rows; returns (elements, seconds).
    Global scales come from the sample itself (the sample is the workload)."""
    t0 = time.perf_counter()
    O.nvfp4_quantize(S["c1"], 16, O.RULE_PREVENT_ZERO, g=O.global_scale(O.amax(S["c1"])))
    for B in (4, 8, 16, 32):
        for rule in range(4):
            O.nvfp4_quantize(S["c2"], B, rule, g=1.0, want_deq=False)
    O.razer_quantize(S["c3w"], O.SF_E3M3, [5.0, -5.0, 3.5, -3.5], g=O.global_scale(O.amax(S["c3w"]), O.SF_E3M3),
                     want_deq=False)
    O.razer_quantize(S["c3a"], O.SF_E4M3, [5.0, -5.0], g=O.global_scale(O.amax(S["c3a"]), O.SF_E4M3), want_deq=False)
    t, ti = O.channel_scale(S["c4x"], S["c4w"], 0.75)
    hb = O.hessian_blocks(S["c4x"], t, True).astype(np.float32)
    O.mxfp4_quantize(S["c4x"], t, True, O.RULE_ABSMAX, want_deq=False)
    O.mxfp4_quantize(S["c4w"], ti, True, O.RULE_HESSIAN_EXP, hb, want_deq=False)
    ga = O.global_scale(O.amax(S["c5"]))
    qa = O.nvfp4_quantize(S["c5"], 16, O.RULE_FOUR_OVER_SIX, g=ga, want_deq=False, want_mse=False)
    qw, gw = S["c5q"]
    O.gemm_ref(qa["codes"], qa["scales"], ga, qw["codes"], qw["scales"], gw)
    elems = (S["c1"].size + 16 * S["c2"].size + S["c3w"].size + S["c3a"].size + S["c4x"].size + S["c4w"].size
             + S["c5"].size)
    return elems, time.perf_counter() - t0


FULL_ELEMS = 4096 * 4096 + 16 * 8192 * 8192 + 8192 * 8192 + 16384 * 4096 + 8192 * 4096 + 4096 * 4096 + 8192 * 4096
def cpu_model():
    """The host CPU's model name (first entry of /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def max_over_ranks(torch, dist, ms, device):
    """The slowest rank's time: every rank contributes its own device-timed
    milliseconds and all get the maximum (one all-reduce, same order on every
    rank)."""
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, ms):
    """Whole-job throughput in G units/s: every rank processed units_per_rank
    in the (max-over-ranks) time ms."""
    return units_per_rank * world / (ms * 1e-3) / 1e9


SAMPLE_ROWS = {"c1": 1 / 4, "c2": 1 / 4, "c3": 1 / 4, "c4": 1 / 4, "c5": 1 / 4}


def run_reference(args, rank, world):
    """The reference arm: the plain CPU oracle, bounded sample, on host cores."""
    if rank != 0:
        return
    from block_scaled_fp4_03_b200 import inputs
    from oracle import oracle as O
    O.build()
    cores = O.get_threads()
    S = oracle_prepare(O, oracle_sample_inputs(inputs, SAMPLE_ROWS))
    for _ in range(args.warmup):
        oracle_sample_run(O, S)
    times, elems = [], 0
    for _ in range(args.steps):
        elems, dt = oracle_sample_run(O, S)
        times.append(dt)
    sec = float(np.mean(times))
    value = elems / sec / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Gelem/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": "the first quarter of the rows of every input"},
        "cpu_baseline": {"value": value, "unit": "Gelem/s", "cores": cores, "kind": "oracle", "cpu_model": cpu_model(),
                         "sample": "each step quantizes %d of the %d elements of a full step (row prefixes)" % (elems, FULL_ELEMS)},
        "e2e": {"value": value, "unit": "Gelem/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main arm
def fp4_ceiling(torch, fq, mx, iters=16384, reps=3):
    """Measured tensor-pipe ceiling (TFLOP/s) of the GEMMs' MMA stream: the library's probe
    kernel (fp4q_mma_ceiling) issuing back-to-back 256x256x64 block-scaled FP4 MMAs on every SM
    pair, timed with CUDA events on the launching stream (best of `reps`, after one warm-up)."""
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    fq.mma_ceiling(mx, 64, err)
    best = None
    flops = 0.0
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        flops = fq.mma_ceiling(mx, iters, err)
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b)
        best = ms if best is None else min(best, ms)
    if int(err.item()) != 0:
        raise RuntimeError("tensor-pipe ceiling probe: a bounded wait gave up")
    return flops / (best * 1e-3) / 1e12


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch the timed step eagerly, not as a CUDA graph")
    ap.add_argument("--fp4-ceiling", action="store_true",
                    help="measure the tensor-pipe ceiling of the GEMMs' FP4 MMA stream and print it (no JSON)")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="time the hot-path step only (skip the rows built on top of it)")
    ap.add_argument("--profile-row", default=None,
                    help="for profiler captures: build only this row's workload group, run the group once, "
                         "then the row --reps times; prints no JSON")
    ap.add_argument("--reps", type=int, default=2)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    from block_scaled_fp4_03_b200 import binding as fq
    from block_scaled_fp4_03_b200 import inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    fq.lib(build_if_missing=True)
    hbm_peak, sm_max_mhz, bf16_peak, bf16_sust, peak_src = load_peaks()

    if args.fp4_ceiling:
        for mx in (False, True):
            print("fp4 MMA ceiling (%s): %.1f TFLOP/s" % ("kind::mxf4 block32" if mx else "kind::mxf4nvf4 block16",
                                                         fp4_ceiling(torch, fq, mx)))
        return 0

    if args.profile_row:
        # the next rows f2 / f3 are built with the workloads they extend
        grp = {"f2": "c5", "f3": "c4"}.get(args.profile_row[:2], args.profile_row[:2])
        rows, X = build_rows(torch, fq, inputs, dev, None, groups={grp})
        target = [r for r in rows if r.name == args.profile_row]
        if not target:
            raise SystemExit("unknown row %s; rows: %s" % (args.profile_row, [r.name for r in rows]))
        for r in rows:
            r.fn()
        for _ in range(args.reps):
            target[0].fn()
        torch.cuda.synchronize()
        print("profiled row", args.profile_row, "x", args.reps)
        return 0

    host = {}
    rows, X = build_rows(torch, fq, inputs, dev, host)
    flush = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    hot = [r for r in rows if not r.extra]
    extra = [] if args.no_next_rows else [r for r in rows if r.extra]
    if args.no_next_rows:
        rows = hot

    def run_rows(rs, times=None):
        for r in rs:
            if times is not None:
                e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
                e0.record(stream)
                r.fn()
                e1.record(stream)
                times[r.name].append((e0, e1))
            else:
                r.fn()

    def step(times=None):
        run_rows(hot, times)
        run_rows(extra, times)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    # brute force: the exact number of error evaluations one call performs
    # (deterministic for a given input), read from the library's counter
    for r in rows:
        if r.eval_ws is not None:
            r.eval_ws.zero_()
            r.fn()
            torch.cuda.synchronize()
            n_eval = int(r.eval_ws[fq.WS_BF_EVALS:fq.WS_BF_EVALS + 8].cpu().numpy().view(np.uint64)[0])
            r.evals = float(n_eval) * r.block

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # the hot step as one CUDA graph: its launches replay back to back with no
    # host launch overhead between them (every buffer the rows touch already
    # exists after the warm-up, so the capture allocates nothing)
    graph, graph_note = None, "eager launches (--no-graph)"
    if not args.no_graph:
        try:
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                run_rows(hot)
            torch.cuda.synchronize()
            graph, graph_note = g, "one CUDA graph replay of the step's launches"
        except Exception as e:    # report and time the eager step instead
            graph_note = "eager launches (graph capture failed: %s)" % str(e).splitlines()[0][:160]
            torch.cuda.synchronize()

    def hot_step():
        if graph is not None:
            graph.replay()
        else:
            run_rows(hot)

    clocks = ClockSampler(local)
    per_row = {r.name: [] for r in rows}
    step_ev = []
    barrier()
    clocks.start()
    for _ in range(args.steps):
        flush.zero_()
        s0, s1 = torch.cuda.Event(True), torch.cuda.Event(True)
        s0.record(stream)
        hot_step()
        s1.record(stream)
        step_ev.append((s0, s1))
        # per-row times: the same rows launched one by one, each between two
        # events, after another flush; then the next rows, outside the step
        flush.zero_()
        run_rows(hot, per_row)
        flush.zero_()
        run_rows(extra, per_row)
    barrier()
    # nvidia-smi samples every 100 ms; a step takes a few ms, so the sampling
    # window extends past the K timed steps with untimed repeats of the same
    # step until it has lasted at least 1.5 s
    n_repeats = 0
    while time.perf_counter() - clocks.t0 < 1.5:
        hot_step()
        torch.cuda.synchronize()
        n_repeats += 1
    clk = clocks.stop()
    if clk is not None:
        clk["window"] = "the %d timed steps plus %d untimed repeats of the same step" % (args.steps, n_repeats)
    step_ms = float(np.mean([a.elapsed_time(b) for a, b in step_ev]))
    if world > 1:
        step_ms = max_over_ranks(torch, dist, step_ms, dev)
    units = sum(r.units for r in hot)
    value = whole_job_rate(units, world, step_ms)

    row_out = {}
    for r in rows:
        ms = float(np.mean([a.elapsed_time(b) for a, b in per_row[r.name]]))
        d = {"ms": ms, "GB_s": r.bytes / (ms * 1e-3) / 1e9, "hbm_frac": r.bytes / (ms * 1e-3) / 1e9 / hbm_peak,
             "hbm_frac_of_8000": r.bytes / (ms * 1e-3) / 1e9 / 8000.0,
             "launches": r.launches, "bound": r.bound}
        if r.units:
            d["Gelem_s"] = r.units / (ms * 1e-3) / 1e9
        if r.flops:
            d["TFLOP_s"] = r.flops / (ms * 1e-3) / 1e12
        row_out[r.name] = d
    for r in extra:
        row_out[r.name]["standalone_call" if r.standalone else "next_row"] = True
    dom = max(hot, key=lambda r: row_out[r.name]["ms"])
    dms = row_out[dom.name]["ms"]
    # fp32 pipe: 148 SMs x 128 lanes x clock; one element-candidate evaluation of
    # a scale search is 6 issue slots (scale multiply, e2m1 encode and decode,
    # dequant multiply, subtract, fma).  Brute-force rows count the element
    # evaluations the call actually performed (the exact shortcuts skip most of
    # the 126 candidates); the overhead around them (seeds, bounds, the warp's
    # work sharing) is what keeps the fraction below 1.
    eval_peak = SM_COUNT * FP32_LANES_PER_SM * sm_max_mhz * 1e6 / 6.0 / 1e9
    for r in rows:
        if r.evals:
            row_out[r.name]["Geval_s"] = r.evals / (row_out[r.name]["ms"] * 1e-3) / 1e9
            row_out[r.name]["alu_frac"] = row_out[r.name]["Geval_s"] / eval_peak
            row_out[r.name]["evals_per_block"] = r.evals / r.block / (r.units / r.block)
    fp4_peak = bf16_peak * 4.0     # dense FP4 = 4 x dense bf16 (nominal 9 / 2.25 PFLOP/s)
    for r in rows:
        if r.bound == "tensor":
            row_out[r.name]["tensor_frac"] = row_out[r.name]["TFLOP_s"] / fp4_peak
    if dom.bound == "tensor":
        ach = dom.flops / (dms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": fp4_peak, "unit": "TFLOP/s", "frac": ach / fp4_peak,
                "traffic": None, "kernel": dom.kernel, "row": dom.name,
                "note": "FP4 peak = measured bf16 burst x 4 (nominal fp4/bf16 ratio); sustained-based: %.3f"
                        % (ach / (bf16_sust * 4.0))}
    elif dom.bound == "alu" and dom.evals:
        ach = dom.evals / (dms * 1e-3) / 1e9
        roof = {"bound": "alu", "achieved": ach, "peak": eval_peak, "unit": "Geval/s", "frac": ach / eval_peak,
                "traffic": None, "kernel": dom.kernel, "row": dom.name,
                "note": "brute force: element-candidate error evaluations the launch performed (counted by the "
                        "library; %.2f per block of the 126 a naive scan does) / time, against 148 SMs x 128 "
                        "fp32 lanes x clock / 6 issue slots per evaluation"
                        % row_out[dom.name]["evals_per_block"]}
    else:
        ach = dom.bytes / (dms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s", "frac": ach / hbm_peak,
                "traffic": None, "kernel": dom.kernel, "row": dom.name}
    roof["peak_source"] = peak_src
    roof["traffic"] = profiled_traffic(dom.name)

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(torch, hot, X, host, stream, args, barrier, world, dist if world > 1 else None, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import oracle as O
        O.build()
        S = oracle_prepare(O, oracle_sample_inputs(inputs, SAMPLE_ROWS))
        secs = []
        for _ in range(3):
            elems, sec = oracle_sample_run(O, S)
            secs.append(sec)
        sec = float(np.mean(secs))
        cpu = {"value": elems / sec / 1e9, "unit": "Gelem/s", "cores": O.get_threads(), "kind": "oracle",
               "cpu_model": cpu_model(),
               "sample": "the first quarter of the rows of every input (%d of the %d elements of a step), "
                         "3 repeats, %.1f s each" % (elems, FULL_ELEMS, sec)}

    launches = sum(r.launches for r in hot) * args.steps
    gem = next((r for r in rows if r.name == "c5_w4a4_gemm"), None)
    gemm = None
    if gem is not None:
        g = row_out[gem.name]
        ceil = fp4_ceiling(torch, fq, False)
        gemm = {"TFLOP_s": g["TFLOP_s"], "frac_of_fp4_peak": g["tensor_frac"], "fp4_peak_TFLOP_s": fp4_peak,
                "frac_of_9000_spec": g["TFLOP_s"] / 9000.0,
                "fp4_mma_ceiling_TFLOP_s": ceil, "frac_of_mma_ceiling": g["TFLOP_s"] / ceil,
                "ms": g["ms"], "shape": "M=8192 N=14336 K=4096", "traffic": profiled_traffic("c5_w4a4_gemm")}
        for r in rows:
            if r.name.startswith("f3_mx_gemm"):
                row_out[r.name]["frac_of_mma_ceiling"] = row_out[r.name]["TFLOP_s"] / fp4_ceiling(torch, fq, True)
                break
    line = {
        "metric": METRIC, "value": value, "unit": "Gelem/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "elements_per_step_per_gpu": units, "l2": "flushed before every step (512 MiB write)",
                   "step_launch": graph_note,
                   "parallelism": "replicas: every rank runs the full step on its own inputs"},
        "roofline": roof, "gemm": gemm, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clk,
        "rows": row_out,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_e2e(torch, rows, X, host, stream, args, barrier, world, dist, dev):
    """Same step through the public API with host buffers: pinned host -> device
    copies of every input, the step, and device -> host copies of every output.
    The copies run on two copy streams, overlapped with the rows' compute: a row
    starts once its inputs have landed, its outputs go back as soon as it is
    done, and the next step's copies wait only for the buffers they overwrite."""
    pinned = {k: torch.from_numpy(v.view(np.int16) if v.dtype == np.uint16 else v).pin_memory() for k, v in host.items()}
    h2d = sum(p.numel() * p.element_size() for p in pinned.values())

    outs_of = []          # per row: the output tensors it is the first to list
    seen = []
    for r in rows:
        mine = []
        for t in r.out.values():
            if torch.is_tensor(t) and all(t.data_ptr() != u.data_ptr() for u in seen):
                seen.append(t)
                mine.append(t)
        outs_of.append(mine)
    host_of = {t.data_ptr(): torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in seen}
    d2h = sum(t.numel() * t.element_size() for t in seen)
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    last_use = {}         # input key -> event after the last row that read it
    out_done = {}         # output pointer -> event after its copy back
    order = []
    for r in rows:
        for k in r.inputs:
            if k not in order:
                order.append(k)
    order += [k for k in pinned if k not in order]

    def one():
        ev_in = {}
        for k in order:
            if k in last_use:
                s_in.wait_event(last_use[k])
            with torch.cuda.stream(s_in):
                dst = X[k]
                dst.view(torch.int16 if dst.dtype == torch.bfloat16 else dst.dtype).copy_(pinned[k], non_blocking=True)
                ev_in[k] = torch.cuda.Event()
                ev_in[k].record(s_in)
        for r, mine in zip(rows, outs_of):
            for k in r.inputs:
                stream.wait_event(ev_in[k])
            for t in mine:
                if t.data_ptr() in out_done:
                    stream.wait_event(out_done[t.data_ptr()])
            r.fn()
            ev = torch.cuda.Event()
            ev.record(stream)
            for k in r.inputs:
                last_use[k] = ev
            if mine:
                s_out.wait_event(ev)
                with torch.cuda.stream(s_out):
                    for t in mine:
                        host_of[t.data_ptr()].copy_(t, non_blocking=True)
                    done = torch.cuda.Event()
                    done.record(s_out)
                for t in mine:
                    out_done[t.data_ptr()] = done

    for _ in range(2):
        one()
    barrier()
    e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
    e0.record(s_in)
    n = max(1, min(args.steps, 3))
    for _ in range(n):
        one()
    # the last copy back is the end of the step's work
    s_out.wait_event(_record(torch, stream))
    s_out.wait_event(_record(torch, s_in))
    e1.record(s_out)
    barrier()
    ms = e0.elapsed_time(e1) / n
    if dist is not None:
        ms = max_over_ranks(torch, dist, ms, dev)
    units = sum(r.units for r in rows)
    return {"value": whole_job_rate(units, world, ms), "unit": "Gelem/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "overlap": "inputs in and outputs back on two copy streams, overlapped with the rows' compute"}


def _record(torch, s):
    ev = torch.cuda.Event()
    ev.record(s)
    return ev


if __name__ == "__main__":
    main()
