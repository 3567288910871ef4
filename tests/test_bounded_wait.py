"""The kernels' bounded waits, made to run out on purpose, without faulting or hanging the GPU.

A test-only build of the library (-DBA_TEST_SKIP_ARRIVE, never part of the product library)
withholds one producer arrival on the first key block of every CTA. Every wait on that block
then reaches its one-second limit: the kernel records BA_ERR_TIMEOUT in its device status word,
each role leaves its loop, the CTA releases its tensor memory and the kernel returns. The host
reads the status through ba_check_device_status, and the device stays usable: the product
library's next call on it matches the oracle.
"""
import ctypes

import numpy as np
import pytest

from util import assert_o_close, oracle_forward

pytestmark = pytest.mark.gpu


def test_expired_wait_reports_timeout_and_device_stays_usable():
    import torch
    import bit_qk_attention_b200 as ba
    from bit_qk_attention_b200 import build, inputs
    assert torch.cuda.is_available(), "needs a CUDA device"
    build.build()
    path = build.build_variant("skiparrive", ["BA_TEST_SKIP_ARRIVE"])
    test_lib = ba.lib(path)
    assert test_lib.ba_set_attention_impl(2) == 0
    w = inputs.random_case(1, 2, 256, 64, torch.float16, 0, seed=3)
    q, k, v = w.q.cuda(), w.k.cuda(), w.v.cuda()
    out = torch.zeros(q.shape, dtype=torch.float32, device="cuda")
    ws = torch.empty(ba.workspace_bytes(1, 2, 256, 64), dtype=torch.uint8, device="cuda")
    nb = ba.CBias()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = test_lib.ba_attention_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), 0, 1, 2, 256, 64, ctypes.byref(nb),
                                   0.0, out.data_ptr(), 2, ws.data_ptr(), ws.numel(), None, stream)
    assert st == 0, "the launch itself succeeds"
    assert test_lib.ba_check_device_status(stream) == 6, "BA_ERR_TIMEOUT expected"
    assert test_lib.ba_check_device_status(stream) == 0, "the status word is cleared once read"
    torch.cuda.synchronize()  # no CUDA error: the context survived

    # The product library on the same device and stream: correct, no timeout.
    ba.set_attention_impl(2)
    got = ba.attention_fwd(q, k, v, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ba.check_device_status()
    ba.set_attention_impl(0)
    assert_o_close(got.cpu().numpy(), oracle_forward(w), "after a timed-out call")
