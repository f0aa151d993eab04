"""float64 CPU oracle for causal GQA + RoPE (+ QK-RMSNorm) and the KV-cache step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library never
imports it and it never imports the CUDA library; the two share no code.

The arithmetic lives in ``oracle.c`` (plain loops, float64, OpenMP over output
rows).  This module only marshals numpy arrays into it and strings the plain
steps together in the order the pages give them:

* QK-norm, then RoPE, on q and k (never on v) -- page "训练3.8B LLM至0.384 CORE，
  成本998美元 – Hugo Vergnes", section "设置"; page "750美元从零训练3个LLM：一位开发者
  的实战复盘", section "V1：现代架构基线".
* causal softmax(q k^T / sqrt(D)) v with query head h reading K/V head h // g --
  same pages, sections "无效的方法" and "V2：引入前沿技术".
* a decode step appends the new token's rotated k and raw v at position
  ``lens[b]`` and attends over ``lens[b] + 1`` keys -- page "750美元从零训练3个LLM",
  section "V3：扩容与推理优化"; a continuation chunk does the same for T tokens
  at once, token t at position ``pos0[b] + t`` seeing the cache and the chunk's
  earlier tokens (the same section, taken a chunk at a time).
* packed documents (``doc_id``): a query sees only the earlier keys of its own
  document -- page "训练3.8B LLM…", section "无效的方法" (document-boundary
  masking with flex attention).
* the backward of causal GQA attention (the pages' models train through the
  causal scaled_dot_product_attention -- page "训练3.8B LLM…", section
  "提高吞吐量"; page "Build a Large Language Model from Scratch", section 3.1):
  the chain rule through softmax written out with numpy matrix products.

Inputs are bfloat16 bit patterns (``numpy.uint16``), widened exactly to float64.

Parity unpinned (conventions no page fixes, declared rather than pinned):
the interior of YaRN's ramp between alpha and beta (``RopeScaling``: taken
continuous in r; its limits, temperature and the other methods are pinned),
the RoPE pairing (halves; the oracle implements both pairings, each pinned to
the complex-number form), and the contiguous head grouping h -> h // g
(pinned against torch's SDPA with ``repeat_interleave``).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
# A prebuilt library elsewhere (the mutation tests load deliberately broken
# builds of oracle.c this way, to show that the pins catch each mistake).
_LIB_OVERRIDE = os.environ.get("GQA_ORACLE_LIB")
_lib = None

_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_u16p = ctypes.POINTER(ctypes.c_uint16)


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared",
                               "-Wall", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        if _LIB_OVERRIDE:
            lib = ctypes.CDLL(_LIB_OVERRIDE)
        else:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
        lib.oracle_bf16_to_f64.argtypes = [_u16p, _f64p, ctypes.c_int64]
        lib.oracle_rmsnorm.argtypes = [_f64p, _f64p, ctypes.c_int64, ctypes.c_int,
                                       ctypes.c_double]
        lib.oracle_rope.argtypes = [_f64p, _f64p, _i64p, ctypes.c_int64, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_double, ctypes.c_int]
        lib.oracle_rope_theta.argtypes = [_f64p, _f64p, _i64p, ctypes.c_int64, ctypes.c_int,
                                          ctypes.c_int, _f64p, ctypes.c_int]
        lib.oracle_attention.argtypes = [_f64p, _f64p, _f64p, _i64p, _f64p,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_double, _i64p, ctypes.c_int64,
                                         ctypes.c_int]
        lib.oracle_attention.restype = ctypes.c_int
        lib.oracle_attention_docs.argtypes = [_f64p, _f64p, _f64p, _i64p, _i64p, _i64p, _f64p,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_double, _i64p, ctypes.c_int64,
                                              ctypes.c_int]
        lib.oracle_attention_docs.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a, t):
    return a.ctypes.data_as(t)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


# --------------------------------------------------------------------------
# elementary steps
# --------------------------------------------------------------------------
def bf16_to_f64(bits) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16 array of any shape) to float64."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    _load().oracle_bf16_to_f64(_ptr(bits, _u16p), _ptr(out, _f64p), bits.size)
    return out


def widen(x) -> np.ndarray:
    """bfloat16 bit patterns (uint16) are widened; float arrays pass as float64."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return bf16_to_f64(x)
    return _f64(x)


def rmsnorm(x, eps: float = 1e-6) -> np.ndarray:
    """Unit-gain RMSNorm over the last axis: x / sqrt(mean(x^2) + eps)."""
    x = _f64(x)
    y = np.empty_like(x)
    D = x.shape[-1]
    _load().oracle_rmsnorm(_ptr(x, _f64p), _ptr(y, _f64p), x.size // D, D, eps)
    return y


class RopeScaling:
    """A RoPE context-extension method.  Page "750美元从零训练3个LLM", section
    "V1：现代架构基线", names NTK-aware scaling and YaRN as the methods RoPE works
    with; the pages give no formulas, so these follow the published methods:

    * ``linear`` (position interpolation): every frequency divided by s;
    * ``ntk`` (NTK-aware): the base raised to base * s^(D/(D-2)), so the fastest
      pair keeps its frequency and the slowest one is divided by s;
    * ``yarn``: pair i makes r_i = L theta_i / (2 pi) turns over the trained
      length L; with the ramp g = 0 below r = alpha, 1 above r = beta and linear
      between, theta_i' = (1 - g) theta_i / s + g theta_i (long wavelengths
      interpolated, short ones kept), and the rotated vectors are multiplied by
      0.1 ln(s) + 1 (the attention temperature).
    """

    def __init__(self, kind: str, factor: float, original_max_pos: int = 0,
                 alpha: float = 1.0, beta: float = 32.0):
        assert kind in ("linear", "ntk", "yarn")
        self.kind, self.factor = kind, float(factor)
        self.original_max_pos, self.alpha, self.beta = int(original_max_pos), float(alpha), float(beta)

    def theta(self, D: int, base: float) -> np.ndarray:
        """The D/2 frequencies theta_i' of the method."""
        i = np.arange(D // 2, dtype=np.float64)
        s = self.factor
        if self.kind == "ntk":
            base = base * s ** (D / (D - 2.0))
        theta = base ** (-2.0 * i / D)
        if self.kind == "linear":
            return theta / s
        if self.kind == "yarn":
            turns = self.original_max_pos * theta / (2.0 * math.pi)
            ramp = np.clip((turns - self.alpha) / (self.beta - self.alpha), 0.0, 1.0)
            return (1.0 - ramp) * theta / s + ramp * theta
        return theta

    def mscale(self) -> float:
        """Factor on the rotated q and k (YaRN only)."""
        return 0.1 * math.log(self.factor) + 1.0 if self.kind == "yarn" else 1.0


def rope(x, pos, base: float = 10000.0, interleaved: bool = False,
         scaling: RopeScaling | None = None) -> np.ndarray:
    """Rotate x [..., N, H, D] (leading axes flattened into N) at positions pos [N]."""
    x = _f64(x)
    H, D = x.shape[-2], x.shape[-1]
    N = x.size // (H * D)
    pos = np.ascontiguousarray(np.broadcast_to(pos, x.shape[:-2]), dtype=np.int64)
    assert pos.size == N
    y = np.empty_like(x)
    if scaling is None:
        _load().oracle_rope(_ptr(x, _f64p), _ptr(y, _f64p), _ptr(pos, _i64p), N, H, D,
                            base, 1 if interleaved else 0)
        return y
    theta = np.ascontiguousarray(scaling.theta(D, base))
    _load().oracle_rope_theta(_ptr(x, _f64p), _ptr(y, _f64p), _ptr(pos, _i64p), N, H, D,
                              _ptr(theta, _f64p), 1 if interleaved else 0)
    return y * scaling.mscale()


def attention(q, k, v, qpos, scale: float | None = None, rows=None,
              nthreads: int = 0, qdoc=None, kdoc=None) -> np.ndarray:
    """Causal GQA attention.

    q [B, Tq, Hq, D]; k, v [B, Tk, Hkv, D]; qpos [B, Tq] = absolute position of
    each query (keys 0..qpos are visible).  ``rows`` optionally lists flat
    (b, t, h) row indices, r = (b*Tq + t)*Hq + h; other output rows stay NaN.
    qdoc [B, Tq] / kdoc [B, Tk]: document ids; a key is then visible only inside
    the query's own document.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Tq, Hq, D = q.shape
    Tk, Hkv = k.shape[1], k.shape[2]
    assert k.shape == (B, Tk, Hkv, D) and v.shape == k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    qpos = np.ascontiguousarray(np.broadcast_to(qpos, (B, Tq)), dtype=np.int64)
    o = np.full(q.shape, np.nan)
    if rows is None:
        rp, nr = None, 0
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        rp, nr = _ptr(rows, _i64p), rows.size
    if qdoc is None:
        rc = _load().oracle_attention(_ptr(q, _f64p), _ptr(k, _f64p), _ptr(v, _f64p),
                                      _ptr(qpos, _i64p), _ptr(o, _f64p), B, Tq, Tk, Hq,
                                      Hkv, D, scale, rp, nr, nthreads)
    else:
        qdoc = np.ascontiguousarray(np.broadcast_to(qdoc, (B, Tq)), dtype=np.int64)
        kdoc = np.ascontiguousarray(np.broadcast_to(kdoc, (B, Tk)), dtype=np.int64)
        rc = _load().oracle_attention_docs(_ptr(q, _f64p), _ptr(k, _f64p), _ptr(v, _f64p),
                                           _ptr(qpos, _i64p), _ptr(qdoc, _i64p),
                                           _ptr(kdoc, _i64p), _ptr(o, _f64p), B, Tq, Tk, Hq,
                                           Hkv, D, scale, rp, nr, nthreads)
    if rc != 0:
        raise ValueError("oracle_attention rejected its arguments (Hq %% Hkv != 0?)")
    return o


# --------------------------------------------------------------------------
# the path, step by step
# --------------------------------------------------------------------------
def prep(x_bits, pos, qk_norm: bool, eps: float = 1e-6, base: float = 10000.0,
         interleaved: bool = False, scaling: RopeScaling | None = None) -> np.ndarray:
    """RoPE(RMSNorm?(x)) for x [B, T, H, D] bf16 bits at positions pos [B, T]."""
    x = widen(x_bits)
    if qk_norm:
        x = rmsnorm(x, eps)
    return rope(x, pos, base, interleaved, scaling)


def positions(pos0, B: int, T: int) -> np.ndarray:
    """Absolute positions pos0[b] + t as an int64 [B, T] array."""
    pos0 = np.broadcast_to(np.asarray(pos0, dtype=np.int64), (B,))
    return pos0[:, None] + np.arange(T, dtype=np.int64)[None, :]


def rope_apply(q_bits, pos0, qk_norm: bool, eps: float = 1e-6,
               base: float = 10000.0, scaling: RopeScaling | None = None) -> np.ndarray:
    """What gqa_rope_apply computes: q [B, T, H, D] rotated at pos0[b] + t."""
    B, T = q_bits.shape[:2]
    return prep(q_bits, positions(pos0, B, T), qk_norm, eps, base, scaling=scaling)


def prefill(q_bits, k_bits, v_bits, qk_norm: bool, eps: float = 1e-6,
            base: float = 10000.0, scale: float | None = None, rows=None,
            nthreads: int = 0, scaling: RopeScaling | None = None, doc_id=None):
    """Prompt prefill from position 0.

    Returns (o [B, T, Hq, D], k_rot [B, T, Hkv, D], v [B, T, Hkv, D]) in float64:
    the attention output and the K/V that the cache holds afterwards.
    """
    B, T = q_bits.shape[:2]
    pos = positions(0, B, T)
    q = prep(q_bits, pos, qk_norm, eps, base, scaling=scaling)
    k = prep(k_bits, pos, qk_norm, eps, base, scaling=scaling)
    v = widen(v_bits)
    o = attention(q, k, v, pos, scale, rows, nthreads, qdoc=doc_id, kdoc=doc_id)
    return o, k, v


def prefill_chunk(q_bits, k_bits, v_bits, k_cache_bits, v_cache_bits, pos0,
                  qk_norm: bool, n_tok=None, eps: float = 1e-6, base: float = 10000.0,
                  scale: float | None = None, rows=None, nthreads: int = 0):
    """A continuation chunk of T new tokens per sequence.

    q [B, T, Hq, D], k/v [B, T, Hkv, D] are raw projections; k_cache/v_cache
    [B, Hkv, Lmax, D] hold rotated K and raw V in slots 0 .. pos0[b]-1 (bf16 bits,
    or float64).  Token t < n_tok[b] of sequence b is normed and rotated at
    position pos0[b] + t, joins the cache at that slot, and attends to slots
    0 .. pos0[b] + t.  Returns (o [B, T, Hq, D], k_rot [B, T, Hkv, D]) in
    float64; rows t >= n_tok[b] of o are NaN.
    """
    B, T = q_bits.shape[:2]
    Hkv = k_bits.shape[2]
    D = q_bits.shape[3]
    pos0 = np.broadcast_to(np.asarray(pos0, dtype=np.int64), (B,))
    n_tok = np.full(B, T, dtype=np.int64) if n_tok is None else np.asarray(n_tok, np.int64)
    pos = positions(pos0, B, T)
    q = prep(q_bits, pos, qk_norm, eps, base)
    k = prep(k_bits, pos, qk_norm, eps, base)
    v = widen(v_bits)
    kc = widen(k_cache_bits)
    vc = widen(v_cache_bits)
    Tk = max(1, int((pos0 + n_tok).max()))
    keys = np.zeros((B, Tk, Hkv, D))
    vals = np.zeros((B, Tk, Hkv, D))
    for b in range(B):
        P, n = int(pos0[b]), int(n_tok[b])
        keys[b, :P] = kc[b, :, :P].transpose(1, 0, 2)
        vals[b, :P] = vc[b, :, :P].transpose(1, 0, 2)
        keys[b, P:P + n] = k[b, :n]
        vals[b, P:P + n] = v[b, :n]
    o = attention(q, keys, vals, pos, scale, rows, nthreads)
    for b in range(B):
        o[b, int(n_tok[b]):] = np.nan
    return o, k


def decode_step(q_bits, k_bits, v_bits, k_cache_bits, v_cache_bits, lens,
                qk_norm: bool, eps: float = 1e-6, base: float = 10000.0,
                scale: float | None = None, nthreads: int = 0, rows=None):
    """One decode step against a KV cache.

    q [B, Hq, D], k/v [B, Hkv, D] are the new token's raw projections;
    k_cache/v_cache [B, Hkv, Lmax, D] hold already-rotated K and raw V in slots
    0 .. lens[b]-1 (bf16 bits, or float64 for exact cached-vs-uncached checks).  The new token sits at position lens[b].  Returns
    (o [B, Hq, D], k_rot [B, Hkv, D]) in float64.
    """
    lens = np.asarray(lens, dtype=np.int64)
    B, Hq, D = q_bits.shape
    Hkv = k_bits.shape[1]
    kc = widen(k_cache_bits)
    vc = widen(v_cache_bits)
    Lmax = kc.shape[2]
    pos = lens[:, None]
    q = prep(q_bits[:, None], pos, qk_norm, eps, base)            # [B, 1, Hq, D]
    k = prep(k_bits[:, None], pos, qk_norm, eps, base)            # [B, 1, Hkv, D]
    v = widen(v_bits)[:, None]
    Tk = int(lens.max()) + 1
    keys = np.zeros((B, Tk, Hkv, D))
    vals = np.zeros((B, Tk, Hkv, D))
    for b in range(B):
        n = int(lens[b])
        assert n < Lmax + 1
        keys[b, :n] = kc[b, :, :n].transpose(1, 0, 2)
        vals[b, :n] = vc[b, :, :n].transpose(1, 0, 2)
        keys[b, n] = k[b, 0]
        vals[b, n] = v[b, 0]
    o = attention(q, keys, vals, pos, scale, rows, nthreads)
    return o[:, 0], k[:, 0]


# --------------------------------------------------------------------------
# backward of causal GQA attention
# --------------------------------------------------------------------------
def attention_backward(q, k, v, dout, scale: float | None = None, heads=None):
    """Gradients of L = sum(dout * o) for o = causal GQA attention(q, k, v).

    q, dout [B, T, Hq, D]; k, v [B, T, Hkv, D] (float64 or bf16 bits); every
    query t sees keys 0..t.  With P = softmax(q k^T * scale) (causal) per query
    head:  dV = P^T dO,  dP = dO V^T,  dS = P * (dP - rowsum(P * dP)),
    dQ = scale dS K,  dK = scale dS^T Q, and the K/V gradients of a KV head are
    the sums over the query heads of its group.  ``heads`` optionally restricts
    the work to some (b, query head) pairs (the other gradients stay NaN for dq
    and hold only those heads' contributions for dk / dv).
    Returns (dq, dk, dv) in float64, plus the forward output o and the row
    log-sum-exp lse [B, Hq, T] (natural log of sum_s exp(q.k_s * scale)).
    """
    q, k, v, do = widen(q), widen(k), widen(v), widen(dout)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = np.full(q.shape, np.nan)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    o = np.full(q.shape, np.nan)
    lse = np.full((B, Hq, T), np.nan)
    future = np.triu(np.ones((T, T), dtype=bool), 1)        # key after query
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in pairs:
        kvh = h // g
        Q, K, V, dO = q[b, :, h], k[b, :, kvh], v[b, :, kvh], do[b, :, h]
        S = (Q @ K.T) * scale
        S[future] = -np.inf
        m = S.max(axis=1, keepdims=True)
        E = np.exp(S - m)
        l = E.sum(axis=1, keepdims=True)
        P = E / l
        o[b, :, h] = P @ V
        lse[b, h] = (m + np.log(l))[:, 0]
        dV = P.T @ dO
        dP = dO @ V.T
        dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
        dq[b, :, h] = scale * (dS @ K)
        dk[b, :, kvh] += scale * (dS.T @ Q)
        dv[b, :, kvh] += dV
    return dq, dk, dv, o, lse
