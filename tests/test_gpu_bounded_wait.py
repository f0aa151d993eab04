"""The bounded waits' failure path, exercised without a fault: a wait that
nothing completes gives up after its limit, raises GQA_DEV_TIMEOUT, and the
context still runs work afterwards."""
import ctypes

import pytest
import torch

import rope_gqa_kv_b200 as gqa

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_wait_that_nothing_completes_times_out(cuda_lib):
    lib = gqa.load()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.gqa_selftest_bounded_wait(ctypes.c_void_p(status.data_ptr()), 50, stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert status.item() & gqa.GQA_DEV_TIMEOUT
    # the context is intact: a decode runs and reports nothing
    q = torch.randn(2, 4, 64, dtype=torch.bfloat16, device=DEV)
    kc = torch.randn(2, 2, 128, 64, dtype=torch.bfloat16, device=DEV)
    st2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = gqa.gqa_decode(q, kc, kc.clone(), torch.tensor([5, 100], dtype=torch.int32, device=DEV),
                         100, status=st2)
    torch.cuda.synchronize()
    assert st2.item() == 0 and torch.isfinite(out.float()).all()
