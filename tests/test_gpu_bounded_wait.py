"""The bounded waits' failure path, exercised without a fault: a wait that
nothing completes gives up after its limit, raises GQA_DEV_TIMEOUT, and the
context still runs work afterwards.  The self-test kernel waits through the
very function every kernel of the library waits with (ptx::mbar_wait), only
with a shorter limit, so the time it takes shows that the limit is honoured."""
import ctypes

import pytest
import torch

import rope_gqa_kv_b200 as gqa

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _selftest(lib, limit_ms):
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    rc = lib.gqa_selftest_bounded_wait(ctypes.c_void_p(status.data_ptr()), limit_ms, stream)
    e1.record()
    assert rc == 0
    torch.cuda.synchronize()
    return int(status.item()), e0.elapsed_time(e1)


def test_wait_that_nothing_completes_times_out(cuda_lib):
    lib = gqa.load()
    for limit_ms in (20, 150):
        st, ms = _selftest(lib, limit_ms)
        # the completed barrier passed (no BAD_LEN); the other one timed out
        assert st == gqa.GQA_DEV_TIMEOUT, (limit_ms, st)
        # the wait lasted its limit, not the kernels' default of one second
        assert limit_ms * 0.9 <= ms <= limit_ms + 200, (limit_ms, ms)
    # the context is intact: a decode runs and reports nothing
    q = torch.randn(2, 4, 64, dtype=torch.bfloat16, device=DEV)
    kc = torch.randn(2, 2, 128, 64, dtype=torch.bfloat16, device=DEV)
    st2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = gqa.gqa_decode(q, kc, kc.clone(), torch.tensor([5, 100], dtype=torch.int32, device=DEV),
                         100, status=st2)
    torch.cuda.synchronize()
    assert st2.item() == 0 and torch.isfinite(out.float()).all()


def test_selftest_rejects_bad_limits(cuda_lib):
    lib = gqa.load()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    assert lib.gqa_selftest_bounded_wait(ctypes.c_void_p(status.data_ptr()), 0, None) != 0
    assert lib.gqa_selftest_bounded_wait(ctypes.c_void_p(status.data_ptr()), 10001, None) != 0
    assert lib.gqa_selftest_bounded_wait(None, 10, None) != 0
