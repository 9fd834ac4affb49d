"""The C-ABI library builds for sm_100a, loads, and exports every symbol the
public headers declare; host-side argument checks reject bad calls before any
CUDA work (so these run without a GPU)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names += re.findall(r"FP4Q_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    from block_scaled_fp4_03_b200 import binding
    return binding.lib()


def test_every_declared_symbol_is_exported(L):
    from block_scaled_fp4_03_b200 import binding
    names = declared_symbols()
    assert len(names) >= 9
    for n in names:
        assert hasattr(L, n), n
        assert n in binding.SIGNATURES, n


def test_header_constants_match_binding():
    from block_scaled_fp4_03_b200 import binding
    src = open(os.path.join(ROOT, "include", "fp4q.h")).read()
    m = re.search(r"#define\s+FP4Q_WS_BF_EVALS\s+(\d+)", src)
    assert m and int(m.group(1)) == binding.WS_BF_EVALS
    assert binding.WS_BF_EVALS % 8 == 0


def test_version_and_status_strings(L):
    assert b"sm_100a" in L.fp4q_version()
    assert L.fp4q_status_str(0) == b"ok"
    assert L.fp4q_status_str(1) == b"invalid argument"
    assert L.fp4q_status_str(99) == b"unknown status"


def test_workspace_sizes(L):
    assert L.fp4q_workspace_size(0, 4096, 4096, 0) >= 592 * 4
    h = L.fp4q_workspace_size(1, 8192, 4096, 0)
    assert h == 256 + (8192 // 256) * (4096 // 32) * 1024 * 4     # error word header + partials
    assert L.fp4q_workspace_size(1, 8192, 100, 0) == 0
    assert L.fp4q_workspace_size(2, 8192, 4096, 4096) > 0


FAKE = ctypes.c_void_p(0x10000)          # aligned, never dereferenced: calls fail before launch
MIS = ctypes.c_void_p(0x10004)


@pytest.mark.parametrize("kw,expect", [
    (dict(block=5), 1), (dict(block=16, cols=24), 1), (dict(rule=7), 1), (dict(dtype=3), 1),
    (dict(gs_mode=9), 1), (dict(rows=-1), 1), (dict(sf_layout=1, rows=100), 1),
    (dict(x=MIS), 2), (dict(codes=MIS), 2), (dict(gs_mode=1, ws=None), 6),
    (dict(gs_mode=2, gs=None), 1),
])
def test_nvfp4_argument_errors(L, kw, expect):
    a = dict(x=FAKE, dtype=0, rows=128, cols=64, block=16, rule=0, gs_mode=0, gs=FAKE, codes=FAKE,
             scales=FAKE, sf_layout=0, deq=None, mse=None, ws=FAKE, wsb=4096)
    a.update(kw)
    st = L.nvfp4_quantize(a["x"], a["dtype"], a["rows"], a["cols"], a["block"], a["rule"], a["gs_mode"],
                          a["gs"], a["codes"], a["scales"], a["sf_layout"], a["deq"], a["mse"], a["ws"],
                          a["wsb"], None)
    assert st == expect


def test_block_quantize_scale_formats(L):
    args = lambda sf, layout: (FAKE, 0, 128, 64, 16, 0, sf, 0, None, FAKE, FAKE, layout, None, None, None, 0, None)
    assert L.fp4_block_quantize(*args(1, 0)) == 1          # E3M3 is RaZeR's, not a block-quantizer format
    assert L.fp4_block_quantize(*args(2, 0)) == 1
    assert L.fp4_block_quantize(*args(9, 0)) == 1
    assert L.fp4_block_quantize(*args(3, 1)) == 1          # UE5M3 scales are row-major only
    # UE5M3 dequant takes no specials
    sp = (ctypes.c_float * 2)(5.0, -5.0)
    assert L.fp4_dequant_mse(FAKE, FAKE, 4, 64, 16, 3, ctypes.cast(sp, ctypes.c_void_p), 2, None, None, 0,
                             FAKE, None, None) == 1


def test_razer_rejects_bad_specials(L):
    for sp, n, sf in (([5.3], 1, 0), ([0.0], 1, 0), ([5, -5, 3.5], 3, 0), ([5, -5, 3.5, -3.5, 1], 5, 1),
                      ([100.0], 1, 1)):
        arr = (ctypes.c_float * len(sp))(*sp)
        st = L.razer_quantize(FAKE, 0, 16, 32, sf, ctypes.cast(arr, ctypes.c_void_p), n, 0, None,
                              FAKE, FAKE, None, None, None, 0, None)
        assert st == 1, sp


def test_mx_and_dequant_argument_errors(L):
    assert L.mxfp4_quantize(FAKE, 0, 4, 48, None, 1, 0, None, FAKE, FAKE, None, None, None) == 1
    assert L.mxfp4_quantize(FAKE, 0, 4, 64, None, 1, 4, None, FAKE, FAKE, None, None, None) == 1
    assert L.mxfp4_quantize(FAKE, 0, 4, 64, None, 1, 2, None, FAKE, FAKE, None, None, None) == 1
    assert L.fp4_dequant_mse(FAKE, FAKE, 4, 64, 16, 2, None, 0, None, None, 0, FAKE, None, None) == 1
    assert L.fp4_dequant_mse(FAKE, FAKE, 4, 64, 16, 0, None, 0, None, None, 0, FAKE, FAKE, None) == 1
    assert L.fp4_hessian_blocks(FAKE, 0, 64, 64, None, 1, FAKE, None, 0, None) == 6
    need = L.fp4q_workspace_size(1, 64, 64, 0)
    assert L.fp4_hessian_blocks(FAKE, 0, 64, 64, None, 1, FAKE, FAKE, need - 1, None) == 6
    assert L.fp4_hessian_blocks(FAKE, 0, 64, 64, None, 1, FAKE, MIS, need, None) == 2
    assert L.mxfp4_channel_scale(FAKE, 0, 64, FAKE, 0, 64, 12, 0.75, FAKE, None, FAKE, 1 << 20, None) == 1
    # Flip-Refinement: bad width, budget, missing Hessian, misalignment, too wide,
    # missing workspace, empty
    big = 1 << 30
    assert L.mxfp4_flip_refine(FAKE, 0, 4, 48, None, 1, FAKE, 8, FAKE, FAKE, None, FAKE, big, None) == 1
    assert L.mxfp4_flip_refine(FAKE, 0, 4, 64, None, 1, FAKE, -1, FAKE, FAKE, None, FAKE, big, None) == 1
    assert L.mxfp4_flip_refine(FAKE, 0, 4, 64, None, 1, FAKE, (1 << 20) + 1, FAKE, FAKE, None, FAKE, big, None) == 1
    assert L.mxfp4_flip_refine(FAKE, 0, 4, 64, None, 1, None, 8, FAKE, FAKE, None, FAKE, big, None) == 1
    assert L.mxfp4_flip_refine(MIS, 0, 4, 64, None, 1, FAKE, 8, FAKE, FAKE, None, FAKE, big, None) == 2
    assert L.mxfp4_flip_refine(FAKE, 0, 4, 8224, None, 1, FAKE, 8, FAKE, FAKE, None, FAKE, big, None) == 3
    need = L.fp4q_workspace_size(4, 4, 64, 0)
    assert need > 0
    assert L.mxfp4_flip_refine(FAKE, 0, 4, 64, None, 1, FAKE, 8, FAKE, FAKE, None, FAKE, need - 1, None) == 6
    assert L.mxfp4_flip_refine(FAKE, 0, 4, 64, None, 1, FAKE, 8, FAKE, FAKE, None, None, 0, None) == 6
    assert L.mxfp4_flip_refine(None, 0, 0, 64, None, 1, None, 8, None, None, None, None, 0, None) == 0


def test_gemm_family_argument_errors(L):
    """RaZeR split, RaZeR / MXFP4 GEMMs and the scale relayout reject bad calls on the host."""
    def table(*v):
        arr = (ctypes.c_float * len(v))(*v)
        return ctypes.cast(arr, ctypes.c_void_p), arr
    sp, keep = table(5.0, -5.0, 3.5, -3.5)
    bad, keep2 = table(11.0)
    # razer_gemm_prepare: shapes, format, table, alignment, empty
    assert L.razer_gemm_prepare(FAKE, FAKE, 120, 64, 1, sp, 4, FAKE, FAKE, FAKE, None) == 1
    assert L.razer_gemm_prepare(FAKE, FAKE, 128, 96, 1, sp, 4, FAKE, FAKE, FAKE, None) == 1
    assert L.razer_gemm_prepare(FAKE, FAKE, 128, 64, 0, sp, 4, FAKE, FAKE, FAKE, None) == 1
    assert L.razer_gemm_prepare(FAKE, FAKE, 128, 64, 1, bad, 1, FAKE, FAKE, FAKE, None) == 3
    assert L.razer_gemm_prepare(MIS, FAKE, 128, 64, 1, sp, 4, FAKE, FAKE, FAKE, None) == 2
    assert L.razer_gemm_prepare(None, None, 0, 64, 1, sp, 4, None, None, None, None) == 0
    # razer_w4a4_gemm: missing operands, shapes, alignment, workspace
    assert L.razer_w4a4_gemm(None, None, FAKE, FAKE, FAKE, None, FAKE, FAKE, 128, 256, 256, FAKE, 1, FAKE, 8192, None) == 1
    assert L.razer_w4a4_gemm(FAKE, None, FAKE, FAKE, FAKE, None, FAKE, FAKE, 100, 256, 256, FAKE, 1, FAKE, 8192, None) == 3
    assert L.razer_w4a4_gemm(FAKE, MIS, FAKE, FAKE, FAKE, None, FAKE, FAKE, 128, 256, 256, FAKE, 1, FAKE, 8192, None) == 2
    assert L.razer_w4a4_gemm(FAKE, None, FAKE, FAKE, FAKE, None, FAKE, FAKE, 128, 256, 256, FAKE, 1, FAKE, 100, None) == 6
    # mxfp4_gemm: format, packed A without scales or with a channel scale, shapes, workspace
    assert L.mxfp4_gemm(FAKE, 2, FAKE, None, 1, FAKE, FAKE, 128, 256, 256, FAKE, 1, FAKE, 1 << 20, None) == 1
    assert L.mxfp4_gemm(FAKE, 3, None, None, 1, FAKE, FAKE, 128, 256, 256, FAKE, 1, FAKE, 1 << 20, None) == 1
    assert L.mxfp4_gemm(FAKE, 3, FAKE, FAKE, 1, FAKE, FAKE, 128, 256, 256, FAKE, 1, FAKE, 1 << 20, None) == 1
    assert L.mxfp4_gemm(FAKE, 1, None, None, 1, FAKE, FAKE, 128, 256, 100, FAKE, 1, FAKE, 1 << 20, None) == 3
    assert L.mxfp4_gemm(FAKE, 1, None, None, 1, FAKE, FAKE, 0, 256, 256, FAKE, 1, FAKE, 1 << 20, None) == 1
    need = L.fp4q_workspace_size(5, 128, 256, 256)
    assert need == 8192 + 128 * 256 // 2 + 128 * 256 // 32
    assert L.mxfp4_gemm(FAKE, 1, None, None, 1, FAKE, FAKE, 128, 256, 256, FAKE, 1, FAKE, need - 1, None) == 6
    assert L.mxfp4_gemm(FAKE, 3, FAKE, None, 1, FAKE, FAKE, 128, 256, 256, FAKE, 1, FAKE, 8191, None) == 6
    # fp4_scales_to_mma
    # every GEMM rejects an output type other than bf16 / fp32
    assert L.razer_w4a4_gemm(FAKE, None, FAKE, FAKE, FAKE, None, FAKE, FAKE, 128, 256, 256, FAKE, 2, FAKE, 8192, None) == 1
    assert L.mxfp4_gemm(FAKE, 1, None, None, 1, FAKE, FAKE, 128, 256, 256, FAKE, 3, FAKE, 1 << 20, None) == 1
    assert L.w4a4_gemm(FAKE, 2, 0, FAKE, FAKE, FAKE, FAKE, FAKE, 128, 256, 256, FAKE, 2, FAKE, 1 << 20, None) == 1
    # fp4_scales_to_mma
    assert L.fp4_scales_to_mma(FAKE, 100, 8, FAKE, None) == 1
    assert L.fp4_scales_to_mma(FAKE, 128, 6, FAKE, None) == 1
    assert L.fp4_scales_to_mma(MIS, 128, 8, FAKE, None) == 2
    assert L.fp4_scales_to_mma(None, 0, 8, None, None) == 0


def test_header_is_plain_c(tmp_path):
    """include/fp4q.h compiles as C99 on its own (a C-ABI header, no C++ or CUDA types)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use.c"
    src.write_text('#include "fp4q.h"\n'
                   'int main(void) {\n'
                   '    size_t n = fp4q_workspace_size(FP4Q_OP_GEMM, 128, 256, 256);\n'
                   '    const char* s = fp4q_status_str(FP4Q_ERR_ARG);\n'
                   '    return (int)(n == 0) + (s == 0);\n'
                   '}\n')
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-fsyntax-only",
                        "-I", os.path.join(ROOT, "include"), str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_status_calls_reject_a_missing_workspace(L):
    assert L.fp4q_gemm_status(None, None) == 1


def test_mma_ceiling_probe_argument_errors(L):
    assert L.fp4q_mma_ceiling(0, 0, FAKE, None) == 1            # no iterations
    assert L.fp4q_mma_ceiling(0, (1 << 20) + 1, FAKE, None) == 1
    assert L.fp4q_mma_ceiling(2, 16, FAKE, None) == 1            # mx is 0 or 1
    assert L.fp4q_mma_ceiling(0, 16, None, None) == 1
    assert L.fp4q_mma_ceiling(0, 16, ctypes.c_void_p(0x10002), None) == 2
    assert L.fp4q_mma_ceiling_flops(0) == 0.0


def test_debug_wait_limit_setter_round_trips(L):
    """The wait-limit knob is host state only: it stores and returns settings, 0 = default."""
    prev = L.fp4q_debug_set_wait_cycles(1)
    try:
        assert L.fp4q_debug_set_wait_cycles(12345) == 1
        assert L.fp4q_debug_set_wait_cycles(-5) == 12345
        assert L.fp4q_debug_set_wait_cycles(0) == 0          # a negative value stored as the default
    finally:
        L.fp4q_debug_set_wait_cycles(prev)


def test_debug_force_amax_pass_setter_round_trips(L):
    """The forced-amax-pass knob is host state only: any nonzero value reads back as 1."""
    prev = L.fp4q_debug_force_amax_pass(1)
    try:
        assert L.fp4q_debug_force_amax_pass(7) == 1
        assert L.fp4q_debug_force_amax_pass(0) == 1
        assert L.fp4q_debug_force_amax_pass(0) == 0
    finally:
        L.fp4q_debug_force_amax_pass(prev)
