"""Thin Python binding of the fp4q C ABI (include/fp4q.h).

Argument marshalling only: torch tensors provide device memory and the
current CUDA stream; every step of the computation runs in the CUDA library
``libfp4q.so``.  There is no CPU fallback -- if the library is missing or the
tensors are not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

F32, BF16, NVFP4_PACKED, MXFP4_PACKED = 0, 1, 2, 3
SF_E4M3, SF_E3M3, SF_E8M0, SF_UE5M3 = 0, 1, 2, 3
ABSMAX, PREVENT_ZERO, FOUR_OVER_SIX, BRUTE_FORCE, HESSIAN_EXP = range(5)
GS_NONE, GS_AMAX, GS_GIVEN = 0, 1, 2
SF_ROWMAJOR, SF_MMA = 0, 1
OP_QUANTIZE, OP_HESSIAN, OP_CHANNEL_SCALE, OP_GEMM, OP_FLIP, OP_MX_GEMM = range(6)
# byte offset, in a quantize workspace, of the uint64 that brute force adds its
# evaluation count to (FP4Q_WS_BF_EVALS)
WS_BF_EVALS = 3072

# name -> (restype, argtypes) of every exported entry point
_vp, _i, _i64, _sz, _fp = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
SIGNATURES = {
    "fp4q_workspace_size": (_sz, [_i, _i64, _i64, _i64]),
    "fp4q_status_str": (ctypes.c_char_p, [_i]),
    "fp4q_version": (ctypes.c_char_p, []),
    "nvfp4_quantize": (_i, [_vp, _i, _i64, _i64, _i, _i, _i, _vp, _vp, _vp, _i, _vp, _vp, _vp, _sz, _vp]),
    "fp4_block_quantize": (_i, [_vp, _i, _i64, _i64, _i, _i, _i, _i, _vp, _vp, _vp, _i, _vp, _vp, _vp, _sz, _vp]),
    "razer_quantize": (_i, [_vp, _i, _i64, _i64, _i, _vp, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "mxfp4_quantize": (_i, [_vp, _i, _i64, _i64, _vp, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "mxfp4_flip_refine": (_i, [_vp, _i, _i64, _i64, _vp, _i, _vp, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "fp4_hessian_blocks": (_i, [_vp, _i, _i64, _i64, _vp, _i, _vp, _vp, _sz, _vp]),
    "fp4_hessian_blocks_noalloc": (_i, [_vp, _i, _i64, _i64, _vp, _i, _vp, _vp]),
    "mxfp4_channel_scale": (_i, [_vp, _i, _i64, _vp, _i, _i64, _i64, _fp, _vp, _vp, _vp, _sz, _vp]),
    "fp4_dequant_mse": (_i, [_vp, _vp, _i64, _i64, _i, _i, _vp, _i, _vp, _vp, _i, _vp, _vp, _vp]),
    "w4a4_gemm": (_i, [_vp, _i, _i, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _i, _vp, _sz, _vp]),
    "fp4q_gemm_status": (_i, [_vp, _vp]),
    "fp4q_hessian_status": (_i, [_vp, _vp]),
    "fp4q_debug_set_wait_cycles": (_i64, [_i64]),
    "fp4q_debug_force_amax_pass": (_i, [_i]),
    "fp4q_mma_ceiling": (_i, [_i, _i, _vp, _vp]),
    "fp4q_mma_ceiling_flops": (ctypes.c_double, [_i]),
    "razer_gemm_prepare": (_i, [_vp, _vp, _i64, _i64, _i, _vp, _i, _vp, _vp, _vp, _vp]),
    "razer_w4a4_gemm": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _i, _vp, _sz, _vp]),
    "fp4_scales_to_mma": (_i, [_vp, _i64, _i64, _vp, _vp]),
    "mxfp4_gemm": (_i, [_vp, _i, _vp, _vp, _i, _vp, _vp, _i64, _i64, _i64, _vp, _i, _vp, _sz, _vp]),
}

_lock = threading.Lock()
_lib = None


def library_path() -> str:
    return _build.LIB


def lib(build_if_missing: bool = True):
    """Load libfp4q.so (compiling it in-tree first if it is missing or stale)."""
    global _lib
    with _lock:
        if _lib is None:
            if build_if_missing:
                _build.build()
            if not os.path.exists(_build.LIB):
                raise RuntimeError("fp4q CUDA library not built: %s" % _build.LIB)
            L = ctypes.CDLL(_build.LIB)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


class Fp4qError(RuntimeError):
    pass


def _check(status: int, what: str):
    if status != 0:
        msg = lib().fp4q_status_str(status).decode()
        raise Fp4qError("%s failed: %s (%d)" % (what, msg, status))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError("fp4q takes float32 or bfloat16 tensors, got %s" % t.dtype)


def _out_tensor(out, M, N, out_dtype, device):
    """The GEMM output tensor and its fp4q dtype code (bf16 unless fp32 is asked for)."""
    if out is not None:
        return out, _dtype_code(out)
    dt = torch.float32 if out_dtype == F32 else torch.bfloat16
    return torch.empty((M, N), dtype=dt, device=device), (F32 if out_dtype == F32 else BF16)


def _need_cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("fp4q needs CUDA tensors (no CPU path)")
            if not t.is_contiguous():
                raise ValueError("fp4q needs contiguous tensors")


def workspace_size(op: int, rows: int, cols: int, n: int = 0) -> int:
    return int(lib().fp4q_workspace_size(op, rows, cols, n))


def _workspace(op, rows, cols, n, device, ws):
    need = workspace_size(op, rows, cols, n)
    if ws is None and need:
        ws = torch.empty(need, dtype=torch.uint8, device=device)
    return ws, (0 if ws is None else ws.numel())


def nvfp4_quantize(x: torch.Tensor, block: int = 16, rule: int = ABSMAX, gs_mode: int = GS_AMAX,
                   global_scale: torch.Tensor | None = None, sf_layout: int = SF_ROWMAJOR,
                   dequant: bool = False, mse: bool = False, out: dict | None = None,
                   workspace: torch.Tensor | None = None, stream=None, scale_fmt: int = SF_E4M3) -> dict:
    """NVFP4 block quantization; returns dict(codes, scales, global_scale, dequant, mse).
    scale_fmt=SF_UE5M3 runs the same rules with UE5M3 block scales
    (fp4_block_quantize)."""
    _need_cuda(x)
    rows, cols = x.shape
    dev = x.device
    o = out or {}
    codes = o.get("codes") if o.get("codes") is not None else torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    scales = o.get("scales") if o.get("scales") is not None else torch.empty((rows, cols // block), dtype=torch.uint8, device=dev)
    if global_scale is None and gs_mode != GS_NONE:
        global_scale = o.get("global_scale") if o.get("global_scale") is not None else torch.empty(1, dtype=torch.float32, device=dev)
    dq = (o.get("dequant") if o.get("dequant") is not None else torch.empty((rows, cols), dtype=torch.float32, device=dev)) if dequant else None
    ms = (o.get("mse") if o.get("mse") is not None else torch.empty((rows, cols // block), dtype=torch.float32, device=dev)) if mse else None
    ws, wsb = (workspace, workspace.numel()) if workspace is not None else (
        _workspace(OP_QUANTIZE, rows, cols, 0, dev, None) if gs_mode == GS_AMAX else (None, 0))
    _need_cuda(codes, scales, global_scale, dq, ms, ws)
    if scale_fmt == SF_E4M3:
        st = lib().nvfp4_quantize(_ptr(x), _dtype_code(x), rows, cols, block, rule, gs_mode,
                                  _ptr(global_scale), _ptr(codes), _ptr(scales), sf_layout, _ptr(dq),
                                  _ptr(ms), _ptr(ws), wsb, _stream(stream))
        _check(st, "nvfp4_quantize")
    else:
        st = lib().fp4_block_quantize(_ptr(x), _dtype_code(x), rows, cols, block, rule, scale_fmt, gs_mode,
                                      _ptr(global_scale), _ptr(codes), _ptr(scales), sf_layout, _ptr(dq),
                                      _ptr(ms), _ptr(ws), wsb, _stream(stream))
        _check(st, "fp4_block_quantize")
    return dict(codes=codes, scales=scales, global_scale=global_scale, dequant=dq, mse=ms)


def razer_quantize(x: torch.Tensor, scale_fmt: int, specials, gs_mode: int = GS_AMAX,
                   global_scale: torch.Tensor | None = None, dequant: bool = False,
                   mse: bool = False, out: dict | None = None,
                   workspace: torch.Tensor | None = None, stream=None) -> dict:
    """RaZeR quantization (blocks of 16); returns dict(codes, meta, global_scale, dequant, mse)."""
    _need_cuda(x)
    rows, cols = x.shape
    dev = x.device
    o = out or {}
    codes = o.get("codes") if o.get("codes") is not None else torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    meta = o.get("meta") if o.get("meta") is not None else torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)
    if global_scale is None and gs_mode != GS_NONE:
        global_scale = o.get("global_scale") if o.get("global_scale") is not None else torch.empty(1, dtype=torch.float32, device=dev)
    dq = (o.get("dequant") if o.get("dequant") is not None else torch.empty((rows, cols), dtype=torch.float32, device=dev)) if dequant else None
    ms = (o.get("mse") if o.get("mse") is not None else torch.empty((rows, cols // 16), dtype=torch.float32, device=dev)) if mse else None
    ws, wsb = (workspace, workspace.numel()) if workspace is not None else (
        _workspace(OP_QUANTIZE, rows, cols, 0, dev, None) if gs_mode == GS_AMAX else (None, 0))
    sp = (ctypes.c_float * len(specials))(*[float(v) for v in specials])
    st = lib().razer_quantize(_ptr(x), _dtype_code(x), rows, cols, scale_fmt, ctypes.cast(sp, ctypes.c_void_p),
                              len(specials), gs_mode, _ptr(global_scale), _ptr(codes), _ptr(meta),
                              _ptr(dq), _ptr(ms), _ptr(ws), wsb, _stream(stream))
    _check(st, "razer_quantize")
    return dict(codes=codes, meta=meta, global_scale=global_scale, dequant=dq, mse=ms)


def mxfp4_quantize(x: torch.Tensor, chan_scale: torch.Tensor | None = None, hadamard: bool = True,
                   rule: int = ABSMAX, hess: torch.Tensor | None = None, dequant: bool = False,
                   mse: bool = False, out: dict | None = None, stream=None) -> dict:
    """MXFP4 quantization with the online transform; returns dict(codes, scales, dequant, mse)."""
    _need_cuda(x, chan_scale, hess)
    rows, cols = x.shape
    dev = x.device
    o = out or {}
    codes = o.get("codes") if o.get("codes") is not None else torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    scales = o.get("scales") if o.get("scales") is not None else torch.empty((rows, cols // 32), dtype=torch.uint8, device=dev)
    dq = (o.get("dequant") if o.get("dequant") is not None else torch.empty((rows, cols), dtype=torch.float32, device=dev)) if dequant else None
    ms = (o.get("mse") if o.get("mse") is not None else torch.empty((rows, cols // 32), dtype=torch.float32, device=dev)) if mse else None
    st = lib().mxfp4_quantize(_ptr(x), _dtype_code(x), rows, cols, _ptr(chan_scale), int(bool(hadamard)),
                              rule, _ptr(hess), _ptr(codes), _ptr(scales), _ptr(dq), _ptr(ms),
                              _stream(stream))
    _check(st, "mxfp4_quantize")
    return dict(codes=codes, scales=scales, dequant=dq, mse=ms)


def mxfp4_flip_refine(w: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, hess: torch.Tensor,
                      chan_scale: torch.Tensor | None = None, hadamard: bool = True, max_moves: int = 128,
                      moves: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """Flip-Refinement of MXFP4 codes in place (exponents fixed); returns the
    int32 [rows] count of moves each row took."""
    _need_cuda(w, codes, scales, hess, chan_scale, workspace)
    rows, cols = w.shape
    mv = moves if moves is not None else torch.empty(rows, dtype=torch.int32, device=w.device)
    ws, wsb = (workspace, workspace.numel()) if workspace is not None else _workspace(OP_FLIP, rows, cols, 0, w.device, None)
    st = lib().mxfp4_flip_refine(_ptr(w), _dtype_code(w), rows, cols, _ptr(chan_scale), int(bool(hadamard)),
                                 _ptr(hess), int(max_moves), _ptr(codes), _ptr(scales), _ptr(mv), _ptr(ws), wsb,
                                 _stream(stream))
    _check(st, "mxfp4_flip_refine")
    return mv


def hessian_blocks(x: torch.Tensor, chan_scale: torch.Tensor | None = None, hadamard: bool = True,
                   out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """H'_k = X'_k^T X'_k for every 32-column block; returns [cols/32, 32, 32] fp32."""
    _need_cuda(x, chan_scale)
    rows, cols = x.shape
    dev = x.device
    h = out if out is not None else torch.empty((cols // 32, 32, 32), dtype=torch.float32, device=dev)
    ws, wsb = (workspace, workspace.numel()) if workspace is not None else _workspace(OP_HESSIAN, rows, cols, 0, dev, None)
    st = lib().fp4_hessian_blocks(_ptr(x), _dtype_code(x), rows, cols, _ptr(chan_scale),
                                  int(bool(hadamard)), _ptr(h), _ptr(ws), wsb, _stream(stream))
    _check(st, "fp4_hessian_blocks")
    return h


def channel_scale(x: torch.Tensor, w: torch.Tensor, alpha: float = 0.75, out=None,
                  workspace: torch.Tensor | None = None, stream=None):
    """Online per-channel scale t and 1/t ([tokens, cols] activations, [n_out, cols] weights)."""
    _need_cuda(x, w)
    tokens, cols = x.shape
    n_out = w.shape[0]
    dev = x.device
    t = out[0] if out is not None else torch.empty(cols, dtype=torch.float32, device=dev)
    ti = out[1] if out is not None else torch.empty(cols, dtype=torch.float32, device=dev)
    ws, wsb = (workspace, workspace.numel()) if workspace is not None else _workspace(OP_CHANNEL_SCALE, tokens, cols, n_out, dev, None)
    st = lib().mxfp4_channel_scale(_ptr(x), _dtype_code(x), tokens, _ptr(w), _dtype_code(w), n_out,
                                   cols, float(alpha), _ptr(t), _ptr(ti), _ptr(ws), wsb,
                                   _stream(stream))
    _check(st, "mxfp4_channel_scale")
    return t, ti


def dequant_mse(codes: torch.Tensor, scales: torch.Tensor, rows: int, cols: int, block: int,
                scale_fmt: int, specials=None, global_scale: torch.Tensor | None = None,
                ref: torch.Tensor | None = None, want_dequant: bool = True, stream=None,
                out: dict | None = None) -> dict:
    """Dequantized values (and, given the reference, per-block MSE) of packed codes;
    returns dict(dequant, mse).  `out` may supply the output tensors."""
    _need_cuda(codes, scales, global_scale, ref)
    dev = codes.device
    o = out or {}
    dq = (o.get("dequant") if o.get("dequant") is not None else
          torch.empty((rows, cols), dtype=torch.float32, device=dev)) if want_dequant else None
    ms = (o.get("mse") if o.get("mse") is not None else
          torch.empty((rows, cols // block), dtype=torch.float32, device=dev)) if ref is not None else None
    sp = None
    n_sp = 0
    if specials is not None:
        n_sp = len(specials)
        sp = (ctypes.c_float * n_sp)(*[float(v) for v in specials])
    st = lib().fp4_dequant_mse(_ptr(codes), _ptr(scales), rows, cols, block, scale_fmt,
                               None if sp is None else ctypes.cast(sp, ctypes.c_void_p), n_sp,
                               _ptr(global_scale), _ptr(ref), 0 if ref is None else _dtype_code(ref),
                               _ptr(dq), _ptr(ms), _stream(stream))
    _check(st, "fp4_dequant_mse")
    return dict(dequant=dq, mse=ms)


def w4a4_gemm(a: torch.Tensor, w_codes: torch.Tensor, w_scales: torch.Tensor, w_global_scale: torch.Tensor,
              a_scales: torch.Tensor | None = None, a_global_scale: torch.Tensor | None = None,
              a_rule: int = FOUR_OVER_SIX, K: int | None = None, out: torch.Tensor | None = None,
              workspace: torch.Tensor | None = None, stream=None, out_dtype: int = BF16) -> torch.Tensor:
    """out = A . W^T in bf16 (or fp32 with out_dtype=F32, or an fp32 `out`).  `a` is either a
    dense fp32/bf16 [M, K] tensor (quantized on the fly with `a_rule`) or packed NVFP4 codes
    [M, K/2] uint8 with `a_scales` (MMA layout) and `a_global_scale`.  W is packed codes
    [N, K/2] with MMA-layout scales."""
    _need_cuda(a, w_codes, w_scales, w_global_scale, a_scales, a_global_scale)
    if a.dtype == torch.uint8:
        fmt = NVFP4_PACKED
        M = a.shape[0]
        K = a.shape[1] * 2 if K is None else K
    else:
        fmt = _dtype_code(a)
        M, K = a.shape
    N = w_codes.shape[0]
    dev = a.device
    o, odt = _out_tensor(out, M, N, out_dtype, dev)
    ws, wsb = (workspace, workspace.numel()) if workspace is not None else _workspace(OP_GEMM, M, K, N, dev, None)
    st = lib().w4a4_gemm(_ptr(a), fmt, a_rule, _ptr(a_scales), _ptr(a_global_scale), _ptr(w_codes),
                         _ptr(w_scales), _ptr(w_global_scale), M, N, K, _ptr(o), odt, _ptr(ws), wsb,
                         _stream(stream))
    _check(st, "w4a4_gemm")
    return o


def razer_gemm_prepare(codes: torch.Tensor, meta: torch.Tensor, scale_fmt: int, specials,
                       out: dict | None = None, stream=None) -> dict:
    """Split RaZeR codes into (main, extra) E2M1 tensors sharing E4M3 scales in the MMA layout;
    returns dict(main, extra, scales)."""
    _need_cuda(codes, meta)
    rows, half = codes.shape
    cols = half * 2
    dev = codes.device
    o = out or {}
    main = o.get("main") if o.get("main") is not None else torch.empty((rows, half), dtype=torch.uint8, device=dev)
    extra = o.get("extra") if o.get("extra") is not None else torch.empty((rows, half), dtype=torch.uint8, device=dev)
    scales = o.get("scales") if o.get("scales") is not None else torch.empty((rows * cols // 16,), dtype=torch.uint8, device=dev)
    sp = (ctypes.c_float * len(specials))(*[float(v) for v in specials])
    st = lib().razer_gemm_prepare(_ptr(codes), _ptr(meta), rows, cols, scale_fmt, ctypes.cast(sp, ctypes.c_void_p),
                                  len(specials), _ptr(main), _ptr(extra), _ptr(scales), _stream(stream))
    _check(st, "razer_gemm_prepare")
    return dict(main=main, extra=extra, scales=scales)


def razer_w4a4_gemm(a_codes: torch.Tensor, a_scales: torch.Tensor, a_global_scale: torch.Tensor,
                    w_codes: torch.Tensor, w_scales: torch.Tensor, w_global_scale: torch.Tensor,
                    a_extra: torch.Tensor | None = None, w_extra: torch.Tensor | None = None,
                    out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                    stream=None, out_dtype: int = BF16) -> torch.Tensor:
    """out = bf16(g_a g_w (A + A_extra) . (W + W_extra)^T): each operand a packed code tensor
    plus an optional extra code tensor sharing its MMA-layout E4M3 scales."""
    _need_cuda(a_codes, a_scales, a_global_scale, w_codes, w_scales, w_global_scale, a_extra, w_extra)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = w_codes.shape[0]
    dev = a_codes.device
    o, odt = _out_tensor(out, M, N, out_dtype, dev)
    ws = workspace if workspace is not None else torch.empty(8192, dtype=torch.uint8, device=dev)
    st = lib().razer_w4a4_gemm(_ptr(a_codes), _ptr(a_extra), _ptr(a_scales), _ptr(a_global_scale),
                               _ptr(w_codes), _ptr(w_extra), _ptr(w_scales), _ptr(w_global_scale),
                               M, N, K, _ptr(o), odt, _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "razer_w4a4_gemm")
    return o


def scales_to_mma(scales: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Row-major scale bytes [rows, nscales] -> the MMA scale layout (flat uint8)."""
    _need_cuda(scales, out)
    rows, n = scales.shape
    o = out if out is not None else torch.empty((rows * n,), dtype=torch.uint8, device=scales.device)
    _check(lib().fp4_scales_to_mma(_ptr(scales), rows, n, _ptr(o), _stream(stream)), "fp4_scales_to_mma")
    return o


def mxfp4_gemm(a: torch.Tensor, w_codes: torch.Tensor, w_scales: torch.Tensor,
               a_scales: torch.Tensor | None = None, chan_scale: torch.Tensor | None = None,
               hadamard: bool = True, K: int | None = None, out: torch.Tensor | None = None,
               workspace: torch.Tensor | None = None, stream=None, out_dtype: int = BF16) -> torch.Tensor:
    """out = A' . W'^T in bf16 with MXFP4 operands.  `a` is a dense fp32/bf16 [M, K] tensor
    (transformed with chan_scale and the 32-block rotation and quantized in the call) or packed
    MXFP4 codes [M, K/2] uint8 with `a_scales` (E8M0, MMA layout).  W: codes [N, K/2] with
    E8M0 scales in the MMA layout."""
    _need_cuda(a, w_codes, w_scales, a_scales, chan_scale)
    if a.dtype == torch.uint8:
        fmt = MXFP4_PACKED
        M = a.shape[0]
        K = a.shape[1] * 2 if K is None else K
    else:
        fmt = _dtype_code(a)
        M, K = a.shape
    N = w_codes.shape[0]
    dev = a.device
    o, odt = _out_tensor(out, M, N, out_dtype, dev)
    ws, wsb = (workspace, workspace.numel()) if workspace is not None else _workspace(OP_MX_GEMM, M, K, N, dev, None)
    if fmt == MXFP4_PACKED and ws is None:
        ws = torch.empty(8192, dtype=torch.uint8, device=dev)
        wsb = ws.numel()
    st = lib().mxfp4_gemm(_ptr(a), fmt, _ptr(a_scales), _ptr(chan_scale), int(bool(hadamard)), _ptr(w_codes),
                          _ptr(w_scales), M, N, K, _ptr(o), odt, _ptr(ws), wsb, _stream(stream))
    _check(st, "mxfp4_gemm")
    return o


def gemm_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronize and return the device-side status word of the last GEMM on `workspace`."""
    return int(lib().fp4q_gemm_status(_ptr(workspace), _stream(stream)))


def hessian_status(workspace: torch.Tensor | None, stream=None) -> int:
    """Synchronize and return the status of the last fp4_hessian_blocks call on `workspace`
    (None: the last fp4_hessian_blocks_noalloc call on the current device)."""
    return int(lib().fp4q_hessian_status(_ptr(workspace), _stream(stream)))


def debug_set_wait_cycles(cycles: int) -> int:
    """Process-wide limit of the tensor-core kernels' bounded waits (0: the default);
    returns the previous setting.  For tests of the timeout path."""
    return int(lib().fp4q_debug_set_wait_cycles(int(cycles)))


def debug_force_amax_pass(on: bool) -> int:
    """Process-wide: hierarchical global scales through the separate amax pass (the
    non-cooperative fallback) instead of the fused one; returns the previous setting."""
    return int(lib().fp4q_debug_force_amax_pass(int(bool(on))))


def mma_ceiling(mx: bool, iters: int, err: torch.Tensor, stream=None) -> float:
    """Enqueue the tensor-pipe ceiling probe (fp4q_mma_ceiling); returns the flops the launch
    performs.  err: a device int32 tensor the kernel sets to 1 if its final wait gave up."""
    _need_cuda(err)
    _check(lib().fp4q_mma_ceiling(int(bool(mx)), int(iters), _ptr(err), _stream(stream)), "fp4q_mma_ceiling")
    return float(lib().fp4q_mma_ceiling_flops(int(iters)))

