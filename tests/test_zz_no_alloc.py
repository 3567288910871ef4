"""ba_attention_fwd_noalloc against ba_attention_fwd, through the C ABI.

The no-allocation entry point serves callers that cannot allocate device memory (a plugin
given only its input and output buffers, a runtime whose device memory is fixed at start-up):
it takes its workspace from a fixed array inside the library. Its output must match the
workspace-taking entry point on the same inputs, on two calls in a row (the array keeps the
previous call's contents, which must not leak into the next result). This file is collected
last so that a stop-at-first-failure run has already run every other test.
"""
import ctypes

import numpy as np
import pytest

from util import O_MAX_ABS, O_MEAN_ABS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ba():
    import torch
    assert torch.cuda.is_available(), "needs a CUDA device"
    from bit_qk_attention_b200 import build
    build.build()
    import bit_qk_attention_b200 as mod
    mod.lib()
    mod.set_attention_impl(0)
    return mod


def _call_noalloc(ba, q, k, v, bias, out):
    import torch
    cb = (bias or ba.Bias()).c()
    st = ba.lib().ba_attention_fwd_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()), ba._dt(q),
        q.shape[0], q.shape[1], q.shape[2], q.shape[3], ctypes.byref(cb), 0.0, ctypes.c_void_p(out.data_ptr()),
        ba._dt(out), None, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


@pytest.mark.parametrize("name", ["tiny", "dit256", "deit_b"])
def test_noalloc_matches_workspace_entry_point(ba, name):
    import torch
    from bit_qk_attention_b200 import inputs
    w = inputs.by_name(name)
    assert ba.workspace_bytes(w.B, w.H, w.N, w.d) <= 32 * 1024 * 1024  # fits the library's array
    q, k, v = w.q.cuda(), w.k.cuda(), w.v.cuda()
    bias = ba.bias_from_workload(w, q.device)
    ref = ba.attention_fwd(q, k, v, bias, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref_np = ref.cpu().numpy()
    for _ in range(2):  # two calls in a row share (and reuse) the library's scratch array
        out = torch.full_like(ref, float("nan"))
        assert _call_noalloc(ba, q, k, v, bias, out) == 0
        torch.cuda.synchronize()
        diff = np.abs(out.cpu().numpy().astype(np.float64) - ref_np)
        assert diff.max() <= O_MAX_ABS and diff.mean() <= O_MEAN_ABS
    ba.check_device_status()


def test_noalloc_refuses_oversized_problems(ba):
    import torch
    limit = 32 * 1024 * 1024
    B, H, N, d = 64, 16, 1024, 64
    assert ba.workspace_bytes(B, H, N, d) > limit
    small = torch.zeros((1, 1, 16, 64), dtype=torch.float16, device="cuda")
    out = torch.zeros((1, 1, 16, 64), dtype=torch.float32, device="cuda")
    cb = ba.Bias().c()
    st = ba.lib().ba_attention_fwd_noalloc(small.data_ptr(), small.data_ptr(), small.data_ptr(), 0, B, H, N, d,
                                           ctypes.byref(cb), 0.0, out.data_ptr(), 2, None, None)
    assert st == 4  # BA_ERR_WORKSPACE, refused before any launch
    torch.cuda.synchronize()
