"""fp4_hessian_blocks_noalloc -- the Hessian-block accumulation for callers
that cannot allocate device memory (code living in another framework's fixed
memory plan, or paths that must not call cudaMalloc because it can
synchronize the device).  Its partial sums live in the library's fixed 16 MiB
device array instead of a caller workspace; everything else is the
computation of fp4_hessian_blocks, which adds the same partials in the same
order, so the two must agree bit for bit -- and both must agree with the
oracle's fp64 blocks within the tolerance of the other H' tests.

Collected last on purpose (file name), so that a run stopping at the first
failure has already run every other test.  Each test stands alone (no state
from earlier tests is needed).
"""
import ctypes

import numpy as np
import pytest
import torch

from block_scaled_fp4_03_b200 import binding as fq
from block_scaled_fp4_03_b200 import inputs

pytestmark = pytest.mark.gpu

TOO_LARGE = 7
TIMEOUT = 5


def _bf16_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(x, t, out, rows, cols):
    L = fq.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = L.fp4_hessian_blocks_noalloc(_p(x), fq.BF16, rows, cols, _p(t), 1, _p(out), stream)
    assert st == 0, L.fp4q_status_str(st)
    return out


def _same_bits(a, b):
    return torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.mark.parametrize("seed,rows,cols", [(1, 1000, 256), (2, 777, 128)])
def test_noalloc_equals_workspace_entry_point_and_oracle_on_two_calls(O, seed, rows, cols):
    xa = inputs.generate("mx_act", rows, cols, seed=seed)
    x = _bf16_dev(xa)
    tn = inputs.positive_vector(cols, seed=seed)
    t = torch.from_numpy(tn).cuda()
    ref = fq.hessian_blocks(x, t, True)
    for _ in range(2):          # the second call reuses the scratch the first one left behind
        out = _noalloc(x, t, torch.full_like(ref, float("nan")), rows, cols)
        assert fq.hessian_status(None) == 0
        assert _same_bits(out, ref)
    exp = O.hessian_blocks(inputs.as_f32(xa), tn, True)
    got = out.cpu().numpy().astype(np.float64)
    for k in range(exp.shape[0]):
        assert np.linalg.norm(got[k] - exp[k]) / np.linalg.norm(exp[k]) <= 1e-5, k


def test_noalloc_at_its_exact_limit():
    """8192 tokens x 4096 columns needs 32 x 128 partial blocks: all 16 MiB of the array."""
    rows, cols = 8192, 4096
    x = _bf16_dev(inputs.generate("mx_act", rows, cols, seed=3))
    t = torch.from_numpy(inputs.positive_vector(cols, seed=3)).cuda()
    ref = fq.hessian_blocks(x, t, True)
    out = _noalloc(x, t, torch.full_like(ref, float("nan")), rows, cols)
    assert fq.hessian_status(None) == 0
    assert _same_bits(out, ref)


def test_noalloc_empty_token_set_gives_zero_blocks():
    cols = 128
    x = _bf16_dev(np.zeros((1, cols), np.uint16))        # a valid pointer; no row is read
    out = _noalloc(x, None, torch.full((cols // 32, 32, 32), float("nan"), device="cuda"), 0, cols)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0


def test_noalloc_rejects_problems_beyond_its_scratch():
    L = fq.lib()
    fake = ctypes.c_void_p(0x10000)   # never touched: the size check comes first
    # 8193 rows x 4096 columns needs 33 x 128 partial blocks (> 4096 = 16 MiB)
    assert L.fp4_hessian_blocks_noalloc(fake, fq.BF16, 8193, 4096, None, 1, fake, None) == TOO_LARGE
    assert L.fp4q_status_str(TOO_LARGE) == b"problem exceeds the library's built-in scratch"


def test_noalloc_reports_a_wait_that_gave_up():
    """With every device wait limited to one cycle the call's blocks come out
    NaN and fp4q_hessian_status(NULL) reports the timeout; the next normal call
    clears it and matches the workspace entry point again."""
    rows, cols = 2048, 256
    x = _bf16_dev(inputs.generate("mx_act", rows, cols, seed=4))
    t = torch.from_numpy(inputs.positive_vector(cols, seed=4)).cuda()
    ref = fq.hessian_blocks(x, t, True)
    prev = fq.debug_set_wait_cycles(1)
    try:
        bad = _noalloc(x, t, torch.empty_like(ref), rows, cols)
        st = fq.hessian_status(None)
    finally:
        fq.debug_set_wait_cycles(prev)
    assert st == TIMEOUT, st
    assert torch.isnan(bad).any()
    out = _noalloc(x, t, torch.empty_like(ref), rows, cols)
    assert fq.hessian_status(None) == 0
    assert _same_bits(out, ref)
