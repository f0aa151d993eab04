"""C-ABI checks that need no GPU: exported symbols and host-side validation.

The argument checks below all fail before the library touches the CUDA
runtime, so they run on a machine without a GPU.
"""
import ctypes
import re
import os

import pytest

import rope_gqa_kv_b200 as gqa
from rope_gqa_kv_b200 import _lib
from rope_gqa_kv_b200 import build as gqa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa.h")


@pytest.fixture(scope="module")
def lib():
    gqa_build.build()
    return gqa.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:gqa_status|size_t|const char \*|int)\s*\**\s*(\w+)\s*\(",
                                 text, flags=re.M)))


def test_header_declares_the_four_entry_points():
    names = declared_functions()
    for n in ("gqa_rope_apply", "kv_cache_append", "gqa_prefill", "gqa_decode",
              "gqa_prefill_chunk"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert names, "no declarations parsed from gqa.h"
    raw = ctypes.CDLL(_lib.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), "libgqa.so does not export %s" % n
    # the binding covers exactly the declared surface
    assert sorted(_lib.SIGNATURES) == names


def test_status_strings_and_version(lib):
    for s in range(7):
        assert lib.gqa_status_string(s)
    assert lib.gqa_status_string(99) == b"unknown status"
    assert lib.gqa_version() >= 100


def test_workspace_size(lib):
    # B * Hq * ceil(max_len / 64) rows of (D + 2) floats
    assert lib.gqa_decode_workspace_bytes(64, 24, 128, 2049) == 64 * 24 * 33 * (128 + 2) * 4
    assert lib.gqa_decode_workspace_bytes(1, 3, 64, 64) == 3 * (64 + 2) * 4
    assert lib.gqa_decode_workspace_bytes(0, 24, 128, 100) == 0
    assert lib.gqa_decode_workspace_bytes(1, 24, 80, 100) == 0


P = _lib.RopeParams(0, 1e-6, 10000.0)
FAKE = ctypes.c_void_p(0x10000)          # 16-byte aligned, never dereferenced
ODD = ctypes.c_void_p(0x10008)           # misaligned


def test_rope_apply_validation(lib):
    assert lib.gqa_rope_apply(None, None, 1, 1, 1, 64, P, None) == 1
    assert lib.gqa_rope_apply(FAKE, None, 1, 1, 1, 80, P, None) == 2
    assert lib.gqa_rope_apply(ODD, None, 1, 1, 1, 64, P, None) == 1
    assert lib.gqa_rope_apply(FAKE, None, 0, 1, 1, 64, P, None) == 1
    bad = _lib.RopeParams(0, 1e-6, 0.5)
    assert lib.gqa_rope_apply(FAKE, None, 1, 1, 1, 64, bad, None) == 1


def test_rope_scaling_validation(lib):
    f = FAKE
    def params(kind, factor=2.0, L=2048, alpha=1.0, beta=32.0):
        return _lib.RopeParams(0, 1e-6, 10000.0, kind, factor, L, alpha, beta)
    assert lib.gqa_rope_apply(f, None, 1, 1, 1, 64, params(9), None) == 1          # unknown kind
    assert lib.gqa_rope_apply(f, None, 1, 1, 1, 64, params(1, 0.5), None) == 1     # factor < 1
    assert lib.gqa_rope_apply(f, None, 1, 1, 1, 64, params(2, 0.9), None) == 1
    assert lib.gqa_rope_apply(f, None, 1, 1, 1, 64, params(3, L=0), None) == 1     # no trained length
    assert lib.gqa_rope_apply(f, None, 1, 1, 1, 64, params(3, alpha=32.0, beta=1.0), None) == 1
    assert lib.kv_cache_append(f, f, f, f, None, 0, None, 1, 16, 2, 64, 128, params(3, 0.5),
                               None, None) == 1


def test_append_validation(lib):
    f = FAKE
    # capacity known on the host: max_pos0 + T > Lmax
    assert lib.kv_cache_append(f, f, f, f, None, 120, None, 1, 16, 2, 64, 128, P, None, None) == 3
    # Lmax not a multiple of 128
    assert lib.kv_cache_append(f, f, f, f, None, 0, None, 1, 16, 2, 64, 100, P, None, None) == 1
    assert lib.kv_cache_append(f, f, f, f, None, 0, None, 1, 16, 2, 72, 128, P, None, None) == 2
    # fused call: Hq not a multiple of Hkv
    assert lib.gqa_rope_append(f, f, f, f, f, None, 0, None, 1, 1, 6, 4, 64, 128, P, None,
                               None) == 1


def test_prefill_validation(lib):
    f = FAKE
    assert lib.gqa_prefill(f, f, f, f, 1, 10, 6, 4, 64, 128, 0.0, None, None) == 1
    assert lib.gqa_prefill(f, f, f, f, 1, 10, 4, 2, 48, 128, 0.0, None, None) == 2
    assert lib.gqa_prefill(f, f, f, f, 1, 300, 4, 2, 64, 256, 0.0, None, None) == 3
    assert lib.gqa_prefill(f, f, f, ODD, 1, 10, 4, 2, 64, 128, 0.0, None, None) == 1
    assert lib.gqa_prefill(f, f, f, f, 1, 0, 4, 2, 64, 128, 0.0, None, None) == 1


def test_prefill_chunk_validation(lib):
    f = FAKE
    odd4 = ctypes.c_void_p(0x10002)      # not 4-byte aligned
    # pos0 is required
    assert lib.gqa_prefill_chunk(f, f, f, f, None, None, 0, 1, 10, 4, 2, 64, 128, 0.0,
                                 None, None) == 1
    # max_pos0 + T beyond the cache
    assert lib.gqa_prefill_chunk(f, f, f, f, f, None, 100, 1, 29, 4, 2, 64, 128, 0.0,
                                 None, None) == 3
    assert lib.gqa_prefill_chunk(f, f, f, f, f, None, -1, 1, 10, 4, 2, 64, 128, 0.0,
                                 None, None) == 1
    assert lib.gqa_prefill_chunk(f, f, f, f, odd4, None, 0, 1, 10, 4, 2, 64, 128, 0.0,
                                 None, None) == 1
    assert lib.gqa_prefill_chunk(f, f, f, f, f, odd4, 0, 1, 10, 4, 2, 64, 128, 0.0,
                                 None, None) == 1
    assert lib.gqa_prefill_chunk(f, f, f, f, f, None, 0, 1, 10, 4, 2, 48, 128, 0.0,
                                 None, None) == 2
    assert lib.gqa_prefill_chunk(f, f, f, f, f, None, 0, 1, 10, 6, 4, 64, 128, 0.0,
                                 None, None) == 1


def test_docs_validation(lib):
    f = FAKE
    odd4 = ctypes.c_void_p(0x10002)
    assert lib.gqa_prefill_docs(f, f, f, f, None, 1, 10, 4, 2, 64, 128, 0.0, None, None) == 1
    assert lib.gqa_prefill_docs(f, f, f, f, odd4, 1, 10, 4, 2, 64, 128, 0.0, None, None) == 1
    assert lib.gqa_prefill_docs(f, f, f, f, f, 1, 10, 4, 2, 80, 128, 0.0, None, None) == 2
    assert lib.gqa_prefill_docs(f, f, f, f, f, 1, 300, 4, 2, 64, 256, 0.0, None, None) == 3
    assert lib.gqa_doc_start(None, f, 1, 10, None, None) == 1
    assert lib.gqa_doc_start(f, odd4, 1, 10, None, None) == 1
    assert lib.gqa_doc_start(f, f, 0, 10, None, None) == 1


def test_backward_validation(lib):
    f = FAKE
    ws = ctypes.c_size_t(1 << 20)
    args = lambda D=64, T=100, L=128, Hq=4, wsb=ws, w=f: (f, f, f, f, f, f, f, f, f, 1, T, Hq, 2, D,
                                                          L, 0.0, w, wsb, None, None)
    assert lib.gqa_attention_backward(None, *args()[1:]) == 1
    assert lib.gqa_attention_backward(*args(D=80)) == 2
    assert lib.gqa_attention_backward(*args(T=300, L=256)) == 3
    assert lib.gqa_attention_backward(*args(Hq=5)) == 1
    assert lib.gqa_attention_backward(*args(wsb=ctypes.c_size_t(16))) == 6
    assert lib.gqa_attention_backward(*args(w=None)) == 6
    # Delta and the scaled log-sum-exp, float32 [B, Hq, round_up(T, 4)] each
    assert lib.gqa_backward_workspace_bytes(2, 1001, 24) == 2 * (2 * 24 * 1004 * 4)
    assert lib.gqa_backward_workspace_bytes(0, 10, 1) == 0
    assert lib.gqa_prefill_lse(f, f, f, f, None, 1, 10, 4, 2, 64, 128, 0.0, None, None) == 1


def test_selftest_validation(lib):
    assert lib.gqa_selftest_bounded_wait(None, 10, None) == 1
    assert lib.gqa_selftest_bounded_wait(FAKE, 0, None) == 1
    assert lib.gqa_selftest_bounded_wait(FAKE, 20000, None) == 1


def test_decode_validation(lib):
    f = FAKE
    ws = ctypes.c_size_t(1 << 20)
    assert lib.gqa_decode(f, f, f, f, 100, f, 1, 4, 2, 64, 128, 0.0, None, 0, None, None) == 6
    assert lib.gqa_decode(f, f, f, f, 100, f, 1, 4, 2, 64, 128, 0.0, f, 16, None, None) == 6
    assert lib.gqa_decode(f, f, f, f, 200, f, 1, 4, 2, 64, 128, 0.0, f, ws, None, None) == 3
    assert lib.gqa_decode(f, f, f, f, 0, f, 1, 4, 2, 64, 128, 0.0, f, ws, None, None) == 1
    assert lib.gqa_decode(f, f, f, f, 100, f, 1, 5, 2, 64, 128, 0.0, f, ws, None, None) == 1
    assert lib.gqa_decode(f, f, f, f, 100, f, 1, 4, 2, 32, 128, 0.0, f, ws, None, None) == 2
    assert lib.gqa_decode(None, f, f, f, 100, f, 1, 4, 2, 64, 128, 0.0, f, ws, None, None) == 1


def test_binding_refuses_cpu_tensors(lib):
    import torch
    q = torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        gqa.gqa_rope_apply(q)


def test_decode_graph_refuses_host_tensors():
    """DecodeGraph captures device work only: host tensors are refused up front."""
    import torch
    kc = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        gqa.DecodeGraph(kc, kc.clone(), torch.zeros(1, dtype=torch.int32), 1)


def _ptxas_registers(src):
    """{kernel name: registers per thread} from ptxas's report for one source,
    compiled exactly as the library build compiles it."""
    import subprocess
    import tempfile
    with tempfile.TemporaryDirectory() as d:
        cmd = ([gqa_build.nvcc()] + gqa_build.NVCC_FLAGS + ["-Xptxas", "-v", "-c", src, "-o",
                                                         os.path.join(d, "x.o")])
        r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    regs, name = {}, None
    for ln in r.stderr.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", ln)
        if m:
            name = m.group(1)
        m = re.search(r"Used (\d+) registers", ln)
        if m and name:
            regs[name] = int(m.group(1))
            name = None
    return regs


@pytest.mark.parametrize("src,pattern,launch_regs", [
    ("prefill.cu", "prefill_kernel", 168),
    ("backward.cu", "bwd_kv_kernel", 168),
    ("backward.cu", "bwd_q_kernel", 168),
])
def test_tensor_core_kernels_keep_their_launch_registers(src, pattern, launch_regs):
    """The tcgen05 kernels split their registers between warpgroups with
    setmaxnreg (2 x 208 + 88 = 3 x 168), which only balances when ptxas gives
    each thread exactly 168 at launch; the host refuses to launch them
    otherwise (GQA_ERR_UNSUPPORTED).  A compiler that allocates differently is
    caught here, on the CPU, instead of by a GPU run."""
    regs = _ptxas_registers(os.path.join(gqa_build.CSRC, src))
    found = {k: v for k, v in regs.items() if pattern in k}
    assert found, "no %s instantiation in ptxas output" % pattern
    wrong = {k: v for k, v in found.items() if v != launch_regs}
    assert not wrong, "registers per thread differ from %d: %s" % (launch_regs, wrong)
