"""ctypes binding of libgqa.so: argument marshalling only.

Every function here takes torch CUDA tensors, checks dtype / shape / device /
contiguity on the host, and passes raw device pointers, sizes and the current
CUDA stream to the C ABI declared in include/gqa.h.  All arithmetic happens in
the library's CUDA kernels; there is no CPU or PyTorch fallback, and a missing
library or a CPU tensor raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgqa.so")
_lib = None

GQA_OK = 0
GQA_DEV_CAPACITY = 0x1
GQA_DEV_TIMEOUT = 0x2
GQA_DEV_BAD_LEN = 0x4

# Every symbol include/gqa.h declares, with (restype, argtypes).
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


class RopeParams(ctypes.Structure):
    _fields_ = [("qk_norm", ctypes.c_int), ("eps", ctypes.c_float),
                ("rope_base", ctypes.c_float), ("scaling", ctypes.c_int),
                ("factor", ctypes.c_float), ("original_max_pos", ctypes.c_int),
                ("yarn_alpha", ctypes.c_float), ("yarn_beta", ctypes.c_float)]


ROPE_KINDS = {"plain": 0, "linear": 1, "ntk": 2, "yarn": 3}


class RopeScaling:
    """A RoPE context-extension variant (see gqa.h): kind 'linear', 'ntk' or
    'yarn', the extension factor s >= 1 and, for YaRN, the trained context
    length and the ramp bounds alpha < beta."""

    def __init__(self, kind: str, factor: float, original_max_pos: int = 0,
                 alpha: float = 1.0, beta: float = 32.0):
        if kind not in ROPE_KINDS:
            raise ValueError("unknown RoPE scaling %r" % kind)
        self.kind, self.factor = kind, float(factor)
        self.original_max_pos, self.alpha, self.beta = int(original_max_pos), float(alpha), float(beta)


SIGNATURES = {
    "gqa_rope_apply": (_i, [_vp, _vp, _i, _i, _i, _i, RopeParams, _vp]),
    "kv_cache_append": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i,
                             RopeParams, _vp, _vp]),
    "gqa_rope_append": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i,
                             RopeParams, _vp, _vp]),
    "gqa_prefill": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp]),
    "gqa_prefill_chunk": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f,
                               _vp, _vp]),
    "gqa_doc_start": (_i, [_vp, _vp, _i, _i, _vp, _vp]),
    "gqa_prefill_lse": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp]),
    "gqa_attention_backward": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                    _i, _i, _f, _vp, _sz, _vp, _vp]),
    "gqa_backward_workspace_bytes": (_sz, [_i, _i, _i]),
    "gqa_prefill_docs": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _vp]),
    "gqa_decode": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _f, _vp, _sz,
                        _vp, _vp]),
    "gqa_decode_workspace_bytes": (_sz, [_i, _i, _i, _i]),
    "gqa_decode_noalloc": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _f, _vp, _vp]),
    "gqa_selftest_bounded_wait": (_i, [_vp, _i, _vp]),
    "gqa_status_string": (ctypes.c_char_p, [_i]),
    "gqa_version": (_i, []),
}


class GqaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (fn, status_string(status), status))


def load(path: str | None = None):
    """Load libgqa.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(
                "libgqa.so not found at %s; build it with `python -m rope_gqa_kv_b200.build`" % p)
        lib = ctypes.CDLL(p)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().gqa_status_string(status).decode()


def _check(fn: str, st: int):
    if st != GQA_OK:
        raise GqaError(fn, st)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor (no CPU path exists)" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if ndim is not None and t.dim() != ndim:
        raise ValueError("%s must have %d dims, got %s" % (name, ndim, tuple(t.shape)))


def _params(qk_norm, eps, rope_base, scaling=None):
    if scaling is None:
        return RopeParams(1 if qk_norm else 0, float(eps), float(rope_base))
    return RopeParams(1 if qk_norm else 0, float(eps), float(rope_base), ROPE_KINDS[scaling.kind],
                      scaling.factor, scaling.original_max_pos, scaling.alpha, scaling.beta)


# ---------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ---------------------------------------------------------------------------
def gqa_rope_apply(q, pos0=None, qk_norm=False, eps=1e-6, rope_base=10000.0, stream=None,
                   scaling=None):
    """In place: q [B, T, H, D] <- RoPE(RMSNorm?(q)) at positions pos0[b] + t."""
    _need(q, "q", torch.bfloat16, 4)
    if pos0 is not None:
        _need(pos0, "pos0", torch.int32, 1)
    B, T, H, D = q.shape
    _check("gqa_rope_apply", load().gqa_rope_apply(
        _ptr(q), _ptr(pos0), B, T, H, D, _params(qk_norm, eps, rope_base, scaling),
        _stream(stream)))
    return q


def kv_cache_append(k, v, k_cache, v_cache, pos0=None, max_pos0=-1, new_len=None,
                    qk_norm=False, eps=1e-6, rope_base=10000.0, status=None, stream=None,
                    scaling=None):
    """Write RoPE(RMSNorm?(k)) and v of the new tokens [B, T, Hkv, D] into the caches."""
    _need(k, "k", torch.bfloat16, 4)
    _need(v, "v", torch.bfloat16, 4)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    B, T, Hkv, D = k.shape
    if v.shape != k.shape or k_cache.shape != v_cache.shape or k_cache.shape[0] != B or \
            k_cache.shape[1] != Hkv or k_cache.shape[3] != D:
        raise ValueError("k/v/cache shapes disagree")
    for name, t in (("pos0", pos0), ("new_len", new_len), ("status", status)):
        if t is not None:
            _need(t, name, torch.int32)
    _check("kv_cache_append", load().kv_cache_append(
        _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(pos0), int(max_pos0),
        _ptr(new_len), B, T, Hkv, D, k_cache.shape[2], _params(qk_norm, eps, rope_base, scaling),
        _ptr(status), _stream(stream)))


def gqa_rope_append(q, k, v, k_cache, v_cache, pos0=None, max_pos0=-1, new_len=None,
                    qk_norm=False, eps=1e-6, rope_base=10000.0, status=None, stream=None,
                    scaling=None):
    """gqa_rope_apply on q and kv_cache_append of k, v in one launch."""
    _need(q, "q", torch.bfloat16)
    _need(k, "k", torch.bfloat16)
    _need(v, "v", torch.bfloat16)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    if q.dim() == 3:            # decode layout [B, H, D] == [B, 1, H, D]
        q4, k4 = q.unsqueeze(1), k.unsqueeze(1)
    else:
        q4, k4 = q, k
    B, T, Hq, D = q4.shape
    Hkv = k4.shape[2]
    if k4.shape != (B, T, Hkv, D) or v.numel() != k.numel() or k_cache.shape[0] != B or \
            k_cache.shape[1] != Hkv or k_cache.shape[3] != D or v_cache.shape != k_cache.shape:
        raise ValueError("q/k/v/cache shapes disagree")
    for name, t in (("pos0", pos0), ("new_len", new_len), ("status", status)):
        if t is not None:
            _need(t, name, torch.int32)
    _check("gqa_rope_append", load().gqa_rope_append(
        _ptr(q), _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(pos0), int(max_pos0),
        _ptr(new_len), B, T, Hq, Hkv, D, k_cache.shape[2], _params(qk_norm, eps, rope_base, scaling),
        _ptr(status), _stream(stream)))


def gqa_prefill(q, k_cache, v_cache, out=None, scale=0.0, status=None, stream=None):
    """Causal GQA attention of a prompt from position 0: q [B, T, Hq, D] -> out."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    B, T, Hq, D = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape != (B, Hkv, Lmax, D) or v_cache.shape != k_cache.shape:
        raise ValueError("cache shape disagrees with q")
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, 4)
    if status is not None:
        _need(status, "status", torch.int32)
    _check("gqa_prefill", load().gqa_prefill(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), B, T, Hq, Hkv, D, Lmax,
        float(scale), _ptr(status), _stream(stream)))
    return out


def gqa_prefill_chunk(q, k_cache, v_cache, pos0, max_pos0, n_tok=None, out=None, scale=0.0,
                      status=None, stream=None):
    """Causal attention of T new tokens per sequence continuing a cached prefix:
    query t of sequence b sits at position pos0[b] + t.  q [B, T, Hq, D] -> out;
    rows t >= n_tok[b] of out are left as they were."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(pos0, "pos0", torch.int32, 1)
    B, T, Hq, D = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape != (B, Hkv, Lmax, D) or v_cache.shape != k_cache.shape:
        raise ValueError("cache shape disagrees with q")
    if pos0.shape != (B,):
        raise ValueError("pos0 must be [B]")
    if n_tok is not None:
        _need(n_tok, "n_tok", torch.int32, 1)
        if n_tok.shape != (B,):
            raise ValueError("n_tok must be [B]")
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, 4)
    if status is not None:
        _need(status, "status", torch.int32)
    _check("gqa_prefill_chunk", load().gqa_prefill_chunk(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(pos0), _ptr(n_tok),
        int(max_pos0), B, T, Hq, Hkv, D, Lmax, float(scale), _ptr(status), _stream(stream)))
    return out


def gqa_prefill_lse(q, k_cache, v_cache, out=None, lse=None, scale=0.0, status=None,
                    stream=None):
    """gqa_prefill that also returns each row's log-sum-exp: (out, lse) with
    lse float32 [B, Hq, round_up(T, 4)] (the padding columns are not written)."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    B, T, Hq, D = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape != (B, Hkv, Lmax, D) or v_cache.shape != k_cache.shape:
        raise ValueError("cache shape disagrees with q")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, (T + 3) // 4 * 4, dtype=torch.float32, device=q.device)
    _need(out, "out", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    if lse.shape != (B, Hq, (T + 3) // 4 * 4):
        raise ValueError("lse must be [B, Hq, round_up(T, 4)]")
    if status is not None:
        _need(status, "status", torch.int32)
    _check("gqa_prefill_lse", load().gqa_prefill_lse(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse), B, T, Hq, Hkv, D, Lmax,
        float(scale), _ptr(status), _stream(stream)))
    return out, lse


def gqa_backward_workspace_bytes(B, T, Hq):
    return int(load().gqa_backward_workspace_bytes(B, T, Hq))


def gqa_attention_backward(q, k, v, out, dout, lse, dq=None, dk=None, dv=None, scale=0.0,
                           workspace=None, status=None, stream=None):
    """Gradients (dq, dk, dv) of causal GQA attention.  q, out, dout [B, T, Hq, D];
    k, v [B, Hkv, Lmax, D] (cache layout, slots < T used); lse from gqa_prefill_lse."""
    for name, t in (("q", q), ("out", out), ("dout", dout)):
        _need(t, name, torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    _need(v, "v", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    B, T, Hq, D = q.shape
    Hkv, Lmax = k.shape[1], k.shape[2]
    if k.shape != (B, Hkv, Lmax, D) or v.shape != k.shape or out.shape != q.shape or \
            dout.shape != q.shape:
        raise ValueError("q/k/v/out/dout shapes disagree")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.zeros_like(k) if dk is None else dk
    dv = torch.zeros_like(v) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _need(t, name, torch.bfloat16, 4)
    if workspace is None:
        workspace = torch.empty(max(gqa_backward_workspace_bytes(B, T, Hq), 16), dtype=torch.uint8,
                                device=q.device)
    if status is not None:
        _need(status, "status", torch.int32)
    _check("gqa_attention_backward", load().gqa_attention_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
        B, T, Hq, Hkv, D, Lmax, float(scale), _ptr(workspace), workspace.numel(), _ptr(status),
        _stream(stream)))
    return dq, dk, dv


def gqa_doc_start(doc_id, out=None, status=None, stream=None):
    """First position of each token's document, from non-decreasing per-token
    document ids doc_id [B, T] (int32)."""
    _need(doc_id, "doc_id", torch.int32, 2)
    B, T = doc_id.shape
    if out is None:
        out = torch.empty_like(doc_id)
    _need(out, "out", torch.int32, 2)
    if status is not None:
        _need(status, "status", torch.int32)
    _check("gqa_doc_start", load().gqa_doc_start(_ptr(doc_id), _ptr(out), B, T, _ptr(status),
                                                 _stream(stream)))
    return out


def gqa_prefill_docs(q, k_cache, v_cache, doc_start, out=None, scale=0.0, status=None,
                     stream=None):
    """Causal attention of a prompt of packed documents: query t sees keys
    doc_start[b, t] .. t.  q [B, T, Hq, D] -> out."""
    _need(q, "q", torch.bfloat16, 4)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(doc_start, "doc_start", torch.int32, 2)
    B, T, Hq, D = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape != (B, Hkv, Lmax, D) or v_cache.shape != k_cache.shape:
        raise ValueError("cache shape disagrees with q")
    if doc_start.shape != (B, T):
        raise ValueError("doc_start must be [B, T]")
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, 4)
    if status is not None:
        _need(status, "status", torch.int32)
    _check("gqa_prefill_docs", load().gqa_prefill_docs(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(doc_start), B, T, Hq, Hkv, D, Lmax,
        float(scale), _ptr(status), _stream(stream)))
    return out


def gqa_decode_workspace_bytes(B, Hq, D, max_len):
    return int(load().gqa_decode_workspace_bytes(B, Hq, D, max_len))


def decode_workspace(B, Hq, D, max_len, device):
    """Scratch for gqa_decode; one workspace serves any number of calls that do
    not run at the same time."""
    need = gqa_decode_workspace_bytes(B, Hq, D, max_len)
    return torch.empty(max(need, 16), dtype=torch.uint8, device=device)


def gqa_decode(q, k_cache, v_cache, lens, max_len, out=None, workspace=None, scale=0.0,
               status=None, stream=None):
    """One query token per sequence: q [B, Hq, D] against lens[b] cached keys."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(lens, "lens", torch.int32, 1)
    B, Hq, D = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape != (B, Hkv, Lmax, D) or v_cache.shape != k_cache.shape:
        raise ValueError("cache shape disagrees with q")
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, 3)
    need = gqa_decode_workspace_bytes(B, Hq, D, max_len)
    if workspace is None:
        workspace = decode_workspace(B, Hq, D, max_len, q.device)
    _need(workspace, "workspace", torch.uint8)
    if status is not None:
        _need(status, "status", torch.int32)
    _check("gqa_decode", load().gqa_decode(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(lens), int(max_len), _ptr(out), B, Hq, Hkv,
        D, Lmax, float(scale), _ptr(workspace), workspace.numel(), _ptr(status),
        _stream(stream)))
    return out


def gqa_decode_noalloc(q, k_cache, v_cache, lens, max_len, out=None, scale=0.0, status=None,
                       stream=None):
    """gqa_decode with its scratch in the library's fixed device array (no
    workspace argument); for callers that cannot allocate device memory."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(lens, "lens", torch.int32, 1)
    B, Hq, D = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape != (B, Hkv, Lmax, D) or v_cache.shape != k_cache.shape:
        raise ValueError("cache shape disagrees with q")
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, 3)
    if status is not None:
        _need(status, "status", torch.int32)
    _check("gqa_decode_noalloc", load().gqa_decode_noalloc(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(lens), int(max_len), _ptr(out), B, Hq, Hkv,
        D, Lmax, float(scale), _ptr(status), _stream(stream)))
    return out
