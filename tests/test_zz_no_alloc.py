"""The no-allocation decode against the workspace decode, through the C ABI.

gqa_decode_noalloc exists for callers that cannot give the library device
scratch memory: code hosted by a framework that owns all device memory and
offers its plugins no allocator, or a loop that must not call cudaMalloc once
it runs (the call synchronises the device and can fail when memory is short).
It keeps its scratch in a fixed array inside the library instead.  Its answers
must agree with gqa_decode's, call after call, since every call reuses that
array.  This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import rope_gqa_kv_b200 as gqa
from rope_gqa_kv_b200 import inputs

from helpers import DECODE_MAX_ABS, MEAN_ABS, bf16_ulp

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(lib, q, kc, vc, lens, max_len, B, Hq, Hkv, D):
    out = torch.full_like(q, float("nan"))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.gqa_decode_noalloc(_p(q), _p(kc), _p(vc), _p(lens), max_len, _p(out), B, Hq, Hkv,
                                D, kc.shape[2], 0.0, _p(status), stream)
    assert rc == 0, lib.gqa_status_string(rc)
    torch.cuda.synchronize()
    assert status.item() == 0
    return out


def _same(got, want, what):
    """The two entry points run the same kernels on the same inputs: the answers
    agree bit for bit, and so within the decode bound (1e-2 plus half a bf16
    ulp of the reference value, mean 1e-3) as well."""
    g = got.double().cpu().numpy()
    w = want.double().cpu().numpy()
    assert np.isfinite(g).all(), what
    d = np.abs(g - w)
    assert (d <= DECODE_MAX_ABS + 0.5 * bf16_ulp(w)).all() and d.mean() <= MEAN_ABS, \
        "%s: max|d| %.3g mean|d| %.3g" % (what, d.max(), d.mean())
    assert torch.equal(got.view(torch.int16), want.view(torch.int16)), what


def test_noalloc_decode_matches_workspace_decode_on_two_calls(cuda_lib):
    lib = gqa.load()
    w = inputs.BY_NAME["batched_decode"]          # B=64, 24/8 heads, D=128, lens U[256, 2048]
    x = inputs.make_inputs(w)
    q = x["steps"][0][0].to(DEV)
    kc, vc = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
    lens = x["lens"].to(DEV)                     # slots past each length hold NaN
    max_len = int(x["lens"].max())
    want = gqa.gqa_decode(q, kc, vc, lens, max_len)          # the existing entry point
    torch.cuda.synchronize()
    for call in range(2):
        got = _noalloc(lib, q, kc, vc, lens, max_len, w.B, w.Hq, w.Hkv, w.D)
        _same(got, want, "batched decode, call %d" % call)

    # A smaller problem after the large ones: the array now holds the large
    # calls' partials in another layout, and none of them may leak into this
    # answer.
    t = inputs.BY_NAME["tiny_gqa"]                # B=1, 4/2 heads, D=64
    xt = inputs.make_inputs(t)
    g = torch.Generator().manual_seed(5)
    qt = torch.randn(t.B, t.Hq, t.D, generator=g).to(torch.bfloat16).to(DEV)
    kct, vct = xt["k_cache"].clone(), xt["v_cache"].clone()
    kct[:, :, :t.T] = torch.randn(t.B, t.Hkv, t.T, t.D, generator=g).to(torch.bfloat16)
    vct[:, :, :t.T] = torch.randn(t.B, t.Hkv, t.T, t.D, generator=g).to(torch.bfloat16)
    kct, vct = kct.to(DEV), vct.to(DEV)
    lt = torch.full((t.B,), t.T, dtype=torch.int32, device=DEV)
    want_t = gqa.gqa_decode(qt, kct, vct, lt, t.T)
    torch.cuda.synchronize()
    got_t = _noalloc(lib, qt, kct, vct, lt, t.T, t.B, t.Hq, t.Hkv, t.D)
    _same(got_t, want_t, "small decode after the batched ones")


def test_noalloc_decode_rejects_sizes_beyond_its_array(cuda_lib):
    lib = gqa.load()
    # 64 sequences x 64 heads x 8192 slots x D=128 need ~272 MB of scratch (> 32 MiB)
    assert lib.gqa_decode_workspace_bytes(64, 64, 128, 8192) > (32 << 20)
    fake = ctypes.c_void_p(0x10000)
    rc = lib.gqa_decode_noalloc(fake, fake, fake, fake, 8192, fake, 64, 64, 8, 128, 8192, 0.0,
                                None, None)
    assert rc == 6      # GQA_ERR_WORKSPACE
