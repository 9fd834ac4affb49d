"""Plain CPU oracle for block-scaled FP4 quantization (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It wraps ``fp4_oracle.c`` (compiled here
with gcc, ``-ffp-contract=off``, no fast-math) and adds the fp64 pieces that
are plain library calls:

* ``hessian_blocks``  -- H'_k = X'_k^T X'_k for every 32-column block of the
  transformed activations ("MACaQ" review, section 1: Hessian-weighted
  exponent selection uses H = X^T X);
* ``mxfp4_flip_refine`` -- greedy adjacent-level code moves by closed-form
  Hessian-weighted gain ("MACaQ" review, sections 1 and 3: Flip-Refinement);
* ``channel_scale``   -- t_j = (sigma_j^W / rms_j^X)^alpha ("MACaQ" review,
  section 3: online scaling, alpha = 0.75, rms from the Hessian diagonal);
* ``gemm_ref``        -- the W4A4 product of the dequantized operands in fp64
  ("Why Gated DeltaNet Survives 4-Bit Quantization" review, section 1: NVFP4
  W4A4 inference).

Parity status: all functions pinned by tests/test_oracle_*.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-std=gnu99", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-shared", "-fPIC"]

SF_E4M3, SF_E3M3, SF_E8M0, SF_UE5M3 = 0, 1, 2, 3
RULE_ABSMAX, RULE_PREVENT_ZERO, RULE_FOUR_OVER_SIX, RULE_BRUTE_FORCE, RULE_HESSIAN_EXP = range(5)

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into oracle/liboracle.so (if stale or forced)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            f32p = ctypes.POINTER(ctypes.c_float)
            u8p = ctypes.POINTER(ctypes.c_uint8)
            i64 = ctypes.c_int64
            L.oracle_e2m1_value.restype = ctypes.c_float
            L.oracle_e2m1_value.argtypes = [ctypes.c_int]
            L.oracle_e2m1_encode.restype = ctypes.c_int
            L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
            for name in ("oracle_e4m3_value", "oracle_e3m3_value", "oracle_ue5m3_value"):
                getattr(L, name).restype = ctypes.c_float
                getattr(L, name).argtypes = [ctypes.c_int]
            for name in ("oracle_e4m3_encode", "oracle_e3m3_encode", "oracle_ue5m3_encode"):
                getattr(L, name).restype = ctypes.c_int
                getattr(L, name).argtypes = [ctypes.c_float]
            L.oracle_e8m0_value.restype = ctypes.c_double
            L.oracle_e8m0_value.argtypes = [ctypes.c_int]
            L.oracle_global_scale.restype = ctypes.c_float
            L.oracle_global_scale.argtypes = [ctypes.c_float, ctypes.c_int]
            L.oracle_amax.restype = ctypes.c_float
            L.oracle_amax.argtypes = [f32p, i64]
            L.oracle_nvfp4_quantize.restype = ctypes.c_int
            L.oracle_nvfp4_quantize.argtypes = [f32p, i64, i64, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_float, u8p, u8p, f32p, f32p]
            L.oracle_block_fp4_quantize.restype = ctypes.c_int
            L.oracle_block_fp4_quantize.argtypes = [f32p, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                    ctypes.c_float, u8p, u8p, f32p, f32p]
            L.oracle_razer_quantize.restype = ctypes.c_int
            L.oracle_razer_quantize.argtypes = [f32p, i64, i64, ctypes.c_int, f32p, ctypes.c_int,
                                                ctypes.c_float, u8p, u8p, f32p, f32p]
            L.oracle_mx_transform.restype = ctypes.c_int
            L.oracle_mx_transform.argtypes = [f32p, i64, i64, f32p, ctypes.c_int, f32p]
            L.oracle_mxfp4_quantize.restype = ctypes.c_int
            L.oracle_mxfp4_quantize.argtypes = [f32p, i64, i64, f32p, ctypes.c_int, ctypes.c_int,
                                                f32p, u8p, u8p, f32p, f32p]
            L.oracle_mxfp4_flip_refine.restype = ctypes.c_int
            L.oracle_mxfp4_flip_refine.argtypes = [f32p, i64, i64, f32p, ctypes.c_int, f32p, ctypes.c_int,
                                                   u8p, u8p, ctypes.POINTER(ctypes.c_int32)]
            L.oracle_dequant_mse.restype = ctypes.c_int
            L.oracle_dequant_mse.argtypes = [u8p, u8p, i64, i64, ctypes.c_int, ctypes.c_int,
                                             f32p, ctypes.c_int, ctypes.c_float, f32p, f32p, f32p]
            L.oracle_set_threads.restype = None
            L.oracle_set_threads.argtypes = [ctypes.c_int]
            L.oracle_get_threads.restype = ctypes.c_int
            L.oracle_get_threads.argtypes = []
            _lib = L
    return _lib


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _p(a, ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())


# ---------------------------------------------------------------- formats
def e2m1_value(code: int) -> float:
    return float(lib().oracle_e2m1_value(int(code)))


def ue5m3_value(code: int) -> float:
    return float(lib().oracle_ue5m3_value(int(code)))


def ue5m3_encode(r: float) -> int:
    return int(lib().oracle_ue5m3_encode(float(np.float32(r))))


def e2m1_encode(y: float) -> int:
    return int(lib().oracle_e2m1_encode(float(np.float32(y))))


def e4m3_value(code: int) -> float:
    return float(lib().oracle_e4m3_value(int(code)))


def e4m3_encode(r: float) -> int:
    return int(lib().oracle_e4m3_encode(float(np.float32(r))))


def e3m3_value(code: int) -> float:
    return float(lib().oracle_e3m3_value(int(code)))


def e3m3_encode(r: float) -> int:
    return int(lib().oracle_e3m3_encode(float(np.float32(r))))


def e8m0_value(byte: int) -> float:
    return float(lib().oracle_e8m0_value(int(byte)))


def global_scale(amax: float, sf: int = SF_E4M3) -> np.float32:
    return np.float32(lib().oracle_global_scale(float(np.float32(amax)), int(sf)))


def amax(x) -> np.float32:
    x = _f32(x)
    return np.float32(lib().oracle_amax(_p(x, ctypes.c_float), x.size))


# ------------------------------------------------------------- quantizers
def nvfp4_quantize(x, block: int, rule: int, g: float = 1.0, want_deq=True, want_mse=True):
    """Returns dict(codes [rows, cols/2] u8, scales [rows, cols/block] u8, deq, mse)."""
    x = _f32(x)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // block), np.uint8)
    deq = np.zeros((rows, cols), np.float32) if want_deq else None
    mse = np.zeros((rows, cols // block), np.float32) if want_mse else None
    rc = lib().oracle_nvfp4_quantize(_p(x, ctypes.c_float), rows, cols, block, rule,
                                     float(np.float32(g)), _p(codes, ctypes.c_uint8),
                                     _p(scales, ctypes.c_uint8), _p(deq, ctypes.c_float),
                                     _p(mse, ctypes.c_float))
    if rc != 0:
        raise ValueError("oracle_nvfp4_quantize rejected its arguments")
    return dict(codes=codes, scales=scales, deq=deq, mse=mse)


def block_fp4_quantize(x, block: int, rule: int, sf: int = SF_E4M3, g: float = 1.0, want_deq=True,
                       want_mse=True):
    """nvfp4_quantize with the block-scale format as a parameter (SF_E4M3 or
    SF_UE5M3, the wide-exponent scale of the "Finer is Better" summary)."""
    x = _f32(x)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // block), np.uint8)
    deq = np.zeros((rows, cols), np.float32) if want_deq else None
    mse = np.zeros((rows, cols // block), np.float32) if want_mse else None
    rc = lib().oracle_block_fp4_quantize(_p(x, ctypes.c_float), rows, cols, block, rule, sf,
                                         float(np.float32(g)), _p(codes, ctypes.c_uint8),
                                         _p(scales, ctypes.c_uint8), _p(deq, ctypes.c_float),
                                         _p(mse, ctypes.c_float))
    if rc != 0:
        raise ValueError("oracle_block_fp4_quantize rejected its arguments")
    return dict(codes=codes, scales=scales, deq=deq, mse=mse)


def razer_quantize(x, sf: int, specials, g: float = 1.0, want_deq=True, want_mse=True):
    """Returns dict(codes, meta [rows, cols/16] u8, deq, mse)."""
    x = _f32(x)
    rows, cols = x.shape
    sp = _f32(specials)
    codes = np.zeros((rows, cols // 2), np.uint8)
    meta = np.zeros((rows, cols // 16), np.uint8)
    deq = np.zeros((rows, cols), np.float32) if want_deq else None
    mse = np.zeros((rows, cols // 16), np.float32) if want_mse else None
    rc = lib().oracle_razer_quantize(_p(x, ctypes.c_float), rows, cols, sf, _p(sp, ctypes.c_float),
                                     sp.size, float(np.float32(g)), _p(codes, ctypes.c_uint8),
                                     _p(meta, ctypes.c_uint8), _p(deq, ctypes.c_float),
                                     _p(mse, ctypes.c_float))
    if rc != 0:
        raise ValueError("oracle_razer_quantize rejected its arguments")
    return dict(codes=codes, meta=meta, deq=deq, mse=mse)


def mx_transform(x, t=None, hadamard: bool = True):
    x = _f32(x)
    rows, cols = x.shape
    tt = None if t is None else _f32(t)
    out = np.zeros((rows, cols), np.float32)
    rc = lib().oracle_mx_transform(_p(x, ctypes.c_float), rows, cols, _p(tt, ctypes.c_float),
                                   int(bool(hadamard)), _p(out, ctypes.c_float))
    if rc != 0:
        raise ValueError("oracle_mx_transform rejected its arguments")
    return out


def mxfp4_quantize(x, t=None, hadamard: bool = True, rule: int = RULE_ABSMAX, hess=None,
                   want_deq=True, want_mse=True):
    """Returns dict(codes, scales (E8M0 bytes), deq, mse) -- deq/mse in the transformed domain."""
    x = _f32(x)
    rows, cols = x.shape
    tt = None if t is None else _f32(t)
    hh = None if hess is None else _f32(hess)
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 32), np.uint8)
    deq = np.zeros((rows, cols), np.float32) if want_deq else None
    mse = np.zeros((rows, cols // 32), np.float32) if want_mse else None
    rc = lib().oracle_mxfp4_quantize(_p(x, ctypes.c_float), rows, cols, _p(tt, ctypes.c_float),
                                     int(bool(hadamard)), rule, _p(hh, ctypes.c_float),
                                     _p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8),
                                     _p(deq, ctypes.c_float), _p(mse, ctypes.c_float))
    if rc != 0:
        raise ValueError("oracle_mxfp4_quantize rejected its arguments")
    return dict(codes=codes, scales=scales, deq=deq, mse=mse)


def mxfp4_flip_refine(x, t, hadamard: bool, hess, codes, scales, max_moves: int = 128):
    """Flip-Refinement of MXFP4 codes ("MACaQ" review, section 1 Key Terms and
    section 3 Method): per output row, greedy moves of single codes to a
    neighbouring E2M1 level by the largest closed-form decrease of
    sum_k d_k^T H'_k d_k, at most max_moves per row.  x: weights [rows, cols]
    (the transform with t and the Hadamard flag is applied as in
    mxfp4_quantize); codes / scales: the MX quantization to refine (exponents
    stay fixed).  Returns (refined codes, accepted moves per row)."""
    x = _f32(x)
    rows, cols = x.shape
    tt = None if t is None else _f32(t)
    hh = _f32(hess)
    out = np.array(codes, np.uint8, copy=True, order="C")
    sc = np.ascontiguousarray(scales, np.uint8)
    moves = np.zeros(rows, np.int32)
    rc = lib().oracle_mxfp4_flip_refine(_p(x, ctypes.c_float), rows, cols, _p(tt, ctypes.c_float),
                                        int(bool(hadamard)), _p(hh, ctypes.c_float), int(max_moves),
                                        _p(out, ctypes.c_uint8), _p(sc, ctypes.c_uint8),
                                        moves.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    if rc != 0:
        raise ValueError("oracle_mxfp4_flip_refine rejected its arguments")
    return out, moves


def dequant_mse(codes, scales, rows: int, cols: int, block: int, sf: int, specials=None,
                g: float = 1.0, ref=None, want_deq=True):
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    sp = None if specials is None else _f32(specials)
    rf = None if ref is None else _f32(ref)
    deq = np.zeros((rows, cols), np.float32) if want_deq else None
    mse = np.zeros((rows, cols // block), np.float32) if rf is not None else None
    rc = lib().oracle_dequant_mse(_p(codes, ctypes.c_uint8), _p(scales, ctypes.c_uint8), rows, cols,
                                  block, sf, _p(sp, ctypes.c_float), 0 if sp is None else sp.size,
                                  float(np.float32(g)), _p(rf, ctypes.c_float),
                                  _p(deq, ctypes.c_float), _p(mse, ctypes.c_float))
    if rc != 0:
        raise ValueError("oracle_dequant_mse rejected its arguments")
    return dict(deq=deq, mse=mse)


# ------------------------------------------------------- fp64 library steps
def hessian_blocks(x, t=None, hadamard: bool = True):
    """H'_k = X'_k^T X'_k in fp64 for each 32-column block k of X' = transform(X).

    Returns an array [cols/32, 32, 32] (fp64)."""
    xt = mx_transform(x, t, hadamard).astype(np.float64)
    rows, cols = xt.shape
    out = np.empty((cols // 32, 32, 32), np.float64)
    for k in range(cols // 32):
        blk = xt[:, 32 * k:32 * (k + 1)]
        out[k] = blk.T @ blk
    return out


def channel_scale(x, w, alpha: float = 0.75):
    """Per-input-channel online scale t_j = (sigma_j^W / rms_j^X)^alpha in fp64.

    x: [tokens, cols] activations; w: [n_out, cols] weights.  sigma_j^W is the
    population standard deviation of weight column j, rms_j^X = sqrt(H_jj / tokens)
    with H = X^T X.  A zero factor gives t_j = 1.  Returns (t, 1/t) as fp32, the
    reciprocal taken in fp32 of the rounded t."""
    x = np.asarray(x, np.float64)
    w = np.asarray(w, np.float64)
    sigma = w.std(axis=0)
    hdiag = np.einsum("ij,ij->j", x, x)
    rms = np.sqrt(hdiag / x.shape[0])
    t = np.ones(x.shape[1], np.float64)
    ok = (sigma > 0) & (rms > 0)
    t[ok] = (sigma[ok] / rms[ok]) ** alpha
    t32 = t.astype(np.float32)
    return t32, (np.float32(1.0) / t32).astype(np.float32)


def decode_tables():
    """(e2m1 values for 16 codes, e4m3 values for 256 bytes) in fp64, from the C oracle."""
    e2 = np.array([e2m1_value(c) for c in range(16)], np.float64)
    e4 = np.array([e4m3_value(c) if (c & 0x7F) != 0x7F else np.nan for c in range(256)], np.float64)
    return e2, e4


def nvfp4_decode_exact(codes, scales, block: int = 16):
    """v * sc for every element in fp64 (exact), from packed codes and row-major E4M3 scales."""
    e2, e4 = decode_tables()
    codes = np.asarray(codes, np.uint8)
    rows = codes.shape[0]
    cols = codes.shape[1] * 2
    v = np.empty((rows, cols), np.float64)
    v[:, 0::2] = e2[codes & 0xF]
    v[:, 1::2] = e2[codes >> 4]
    sc = e4[np.asarray(scales, np.uint8)]
    return v * np.repeat(sc, block, axis=1)


def razer_decode_exact(codes, meta, sf: int, specials):
    """RaZeR values in fp64 (exact), "RaZeR: Redundant Zero Remapping" section
    2.2: every code decodes to its E2M1 value except -0 (code 8), which takes the
    block's special value specials[sel]; times the block scale (E3M3 for
    weights, meta = sel<<6 | code; E4M3 for activations, meta = sel<<7 | code)."""
    codes = np.asarray(codes, np.uint8)
    meta = np.asarray(meta, np.uint8)
    rows, cols = codes.shape[0], codes.shape[1] * 2
    e2 = np.array([e2m1_value(c) for c in range(16)], np.float64)
    c = np.empty((rows, cols), np.int64)
    c[:, 0::2] = codes & 0xF
    c[:, 1::2] = codes >> 4
    if sf == SF_E3M3:
        sel, sc_code = meta >> 6, meta & 0x3F
        sc = np.array([e3m3_value(int(k)) for k in range(64)], np.float64)[sc_code]
    elif sf == SF_E4M3:
        sel, sc_code = meta >> 7, meta & 0x7F
        sc = np.array([e4m3_value(int(k)) for k in range(128)], np.float64)[sc_code]
    else:
        raise ValueError("RaZeR scales are E3M3 or E4M3")
    sp = np.asarray(specials, np.float64)
    v = e2[c]
    special = np.repeat(sp[sel], 16, axis=1)
    v = np.where(c == 8, special, v)
    return v * np.repeat(sc, 16, axis=1)


def mx_decode_exact(codes, scales):
    """MXFP4 values in fp64 (exact), "MACaQ" review section 1: each E2M1 code
    times 2^(byte - 127) of its 32-element block."""
    codes = np.asarray(codes, np.uint8)
    rows, cols = codes.shape[0], codes.shape[1] * 2
    e2 = np.array([e2m1_value(c) for c in range(16)], np.float64)
    v = np.empty((rows, cols), np.float64)
    v[:, 0::2] = e2[codes & 0xF]
    v[:, 1::2] = e2[codes >> 4]
    p2 = np.ldexp(1.0, np.asarray(scales, np.int64) - 127)
    return v * np.repeat(p2, 32, axis=1)


def gemm_values(da, dw, g_a, g_w):
    """out = g_a * g_w * (da @ dw^T) in fp64 for exactly decoded operands."""
    return (float(g_a) * float(g_w)) * (np.asarray(da, np.float64) @ np.asarray(dw, np.float64).T)


def gemm_ref(a_codes, a_scales, g_a, w_codes, w_scales, g_w, rows=None, cols=None):
    """out = g_a * g_w * (deqA @ deqW^T) in fp64, optionally for a subset of rows / cols."""
    if rows is not None:
        a_codes, a_scales = a_codes[rows], a_scales[rows]
    if cols is not None:
        w_codes, w_scales = w_codes[cols], w_scales[cols]
    da = nvfp4_decode_exact(a_codes, a_scales)
    dw = nvfp4_decode_exact(w_codes, w_scales)
    return (float(g_a) * float(g_w)) * (da @ dw.T)
