"""The no-allocation entry point, called through the C ABI, against the
ordinary entry point on the same inputs, twice in a row.

Some callers cannot allocate device memory (a runtime that owns every
allocation through its own pool, a latency-critical path where an allocation
would synchronise the device, a plugin that is only handed its input and
output buffers); am_compact_heads_noalloc serves them from a fixed scratch
array inside the library.  This file is collected last so that a run that
stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from attention_matching_b200 import workloads as W

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")

SCRATCH_BYTES = 16 << 20


def _noalloc():
    import attention_matching_b200 as am
    L = am.lib()
    f = L.am_compact_heads_noalloc
    c_int, c_void_p = ctypes.c_int32, ctypes.c_void_p
    f.argtypes = [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, ctypes.POINTER(ctypes.c_int32),
                  ctypes.POINTER(am.AmOpts), ctypes.POINTER(ctypes.c_int64), c_void_p, c_void_p, c_void_p,
                  c_void_p, c_void_p, c_void_p]
    f.restype = c_int
    return f


def _call_noalloc(heads, budgets, topk, refit):
    import attention_matching_b200 as am
    Q = torch.stack([h.Q for h in heads]).contiguous().cuda()
    K = torch.stack([h.K for h in heads]).contiguous().cuda()
    V = torch.stack([h.V for h in heads]).contiguous().cuda()
    H, n, d = Q.shape
    T = K.shape[1]
    opts = am.make_opts(am.BF16 if Q.dtype == torch.bfloat16 else am.FP32, topk, refit)
    cu = np.concatenate([[0], np.cumsum(budgets)]).astype(np.int64)
    tot = int(cu[-1])
    out = {
        "C_k": torch.empty((tot, d), dtype=Q.dtype, device="cuda"),
        "beta": torch.empty((tot,), dtype=torch.float32, device="cuda"),
        "C_v": torch.empty((tot, d), dtype=torch.float32, device="cuda"),
        "indices": torch.empty((tot,), dtype=torch.int32, device="cuda"),
        "status": torch.full((H,), -1, dtype=torch.int32, device="cuda"),
    }
    b = (ctypes.c_int32 * H)(*budgets)
    offs = (ctypes.c_int64 * (H + 1))(*cu.tolist())
    rc = _noalloc()(Q.data_ptr(), K.data_ptr(), V.data_ptr(), n, T, d, H, b, ctypes.byref(opts), offs,
                    out["C_k"].data_ptr(), out["beta"].data_ptr(), out["C_v"].data_ptr(),
                    out["indices"].data_ptr(), out["status"].data_ptr(),
                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return rc, out, (Q, K, V)


CASES = [
    ("bf16 two heads", lambda: [W.structured_head(500 + h, n=640, T=640) for h in range(2)], [12, 20], 4, 2),
    ("fp32 single head", lambda: W.single_head_fp32().heads, [16], 1, 1),
]


@needs_cuda
@pytest.mark.parametrize("label,make,budgets,topk,refit", CASES)
def test_noalloc_matches_ordinary_entry_point_twice(label, make, budgets, topk, refit):
    import attention_matching_b200 as am
    heads = make()
    for call in range(2):
        rc, out, (Q, K, V) = _call_noalloc(heads, budgets, topk, refit)
        assert rc == 0, f"{label} call {call}: {am.STATUS.get(rc, rc)}"
        assert out["status"].tolist() == [0] * len(budgets), out["status"]
        ref = am.compact_heads(Q, K, V, budgets, topk=topk, refit_every=refit)
        assert torch.equal(out["indices"], ref["indices"]), label
        assert torch.equal(out["C_k"], ref["C_k"]), label
        assert torch.equal(out["beta"], ref["beta"]), label
        torch.testing.assert_close(out["C_v"], ref["C_v"], rtol=1e-5, atol=1e-6)


@needs_cuda
def test_noalloc_rejects_problems_beyond_the_scratch():
    import attention_matching_b200 as am
    opts = am.make_opts(am.BF16, 4, 2)
    assert am.workspace_size(2048, 2048, 128, [40], opts) > SCRATCH_BYTES
    H, n, T, d = 1, 2048, 2048, 128
    b = (ctypes.c_int32 * 1)(40)
    offs = (ctypes.c_int64 * 2)(0, 40)
    # every device pointer is null: the size check answers first, and were it
    # ever skipped the null-argument check would stop the call before any launch
    rc = _noalloc()(None, None, None, n, T, d, H, b, ctypes.byref(opts), offs,
                    None, None, None, None, None, None)
    assert rc == 3   # AM_ERR_WORKSPACE, returned before any GPU work
