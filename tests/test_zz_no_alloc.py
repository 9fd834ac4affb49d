"""fp4_hessian_blocks_noalloc -- the Hessian-block accumulation for callers
that cannot allocate device memory (code living in another framework's fixed
memory plan, or paths that must not call cudaMalloc because it can
synchronize the device).  It must give the same blocks as
fp4_hessian_blocks, which takes a caller-provided workspace instead.

Collected last on purpose (file name), so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_scaled_fp4_03_b200 import binding as fq
from block_scaled_fp4_03_b200 import inputs

pytestmark = pytest.mark.gpu


def _bf16_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    L = fq.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for seed, (rows, cols) in ((1, (1000, 256)), (2, (777, 128))):
        x = _bf16_dev(inputs.generate("mx_act", rows, cols, seed=seed))
        t = torch.from_numpy(inputs.positive_vector(cols, seed=seed)).cuda()
        ref = fq.hessian_blocks(x, t, True)
        out = torch.full_like(ref, float("nan"))
        st = L.fp4_hessian_blocks_noalloc(_p(x), fq.BF16, rows, cols, _p(t), 1, _p(out), stream)
        assert st == 0, L.fp4q_status_str(st)
        torch.cuda.synchronize()
        got, exp = out.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64)
        for k in range(exp.shape[0]):
            err = np.linalg.norm(got[k] - exp[k]) / np.linalg.norm(exp[k])
            assert err <= 1e-5, (seed, k, err)


def test_noalloc_rejects_problems_beyond_its_scratch():
    L = fq.lib()
    fake = ctypes.c_void_p(0x10000)   # never touched: the size check comes first
    # 8193 rows x 4096 columns needs 33 x 128 partial blocks (> 4096 = 16 MiB)
    assert L.fp4_hessian_blocks_noalloc(fake, fq.BF16, 8193, 4096, None, 1, fake, None) == 7
    assert L.fp4q_status_str(7) == b"problem exceeds the library's built-in scratch"
