"""Shared helpers for the GPU parity tests (no attention arithmetic here: the
references come from the oracle and the bf16 floor built from it)."""
import numpy as np
import torch

import oracle
from rope_gqa_kv_b200 import inputs

from ideal_pipeline import assert_floor_close, ideal_attention  # noqa: F401

# Tolerance of the paths that keep fp32 probabilities (decode; RoPE and the
# append, whose outputs are also checked to one ulp): max |d| <= 1e-2 plus half
# an ulp of the exact value in bf16 (the rounding of the answer itself to the
# output format: for |o| > 2.56 it alone exceeds 1e-2), and mean |d| <= 1e-3 --
# the stated bound.  The tensor-core prefill paths (prompt, chunk, documents)
# round the probabilities to bf16 for the P.V product, and no such pipeline
# meets 1e-2 on every element; they are held to the bf16 floor instead,
# element by element (ideal_pipeline.py).
MAX_ABS = 1e-2
DECODE_MAX_ABS = MAX_ABS
MEAN_ABS = 1e-3
# Gradients of the attention backward: the kernels round P and dS to bf16 for
# the tensor cores (as flash-style backwards do) and sum many such products;
# an ideal pipeline with exact arithmetic and only those roundings (plus the
# bf16 outputs) reaches 1.07 x (1e-2 + one ulp) on the 2 x 1000-token case, so
# gradients are held to 2e-2 plus one bf16 ulp of the exact value, mean 1e-3.
GRAD_MAX_ABS = 2e-2
GRAD_MEAN_ABS = 1e-3
# Absolute floor of the one-ulp check: fp32 rotation of O(1) inputs can lose a
# few fp32 ulps (~1e-6) when the result cancels to nearly zero.
ULP_ABS_FLOOR = 2.0 ** -18


def bf16_ulp(x):
    mag = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(mag)) - 7)


def bits(t: torch.Tensor) -> np.ndarray:
    return inputs.bits(t.detach().cpu())


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def assert_close(got: torch.Tensor, want: np.ndarray, what: str, max_abs=MAX_ABS,
                 mean_abs=MEAN_ABS):
    g = f64(got)
    assert g.shape == want.shape, (what, g.shape, want.shape)
    assert np.isfinite(g).all(), "%s: non-finite output" % what
    d = np.abs(g - want)
    allow = max_abs + 0.5 * bf16_ulp(want)
    if not ((d <= allow).all() and d.mean() <= mean_abs):
        i = np.unravel_index(np.argmax(d), d.shape)
        w = want[i]
        rne = float(torch.tensor(w, dtype=torch.float64).to(torch.bfloat16).double())
        raise AssertionError(
            "%s: max|d| %.4g (<= %.3g + half ulp) mean|d| %.3g (<= %.3g); worst at %s: got %.6g "
            "want %.6g (bf16 rounding of want alone: %.3g); elements over: %d of %d"
            % (what, d.max(), max_abs, d.mean(), mean_abs, i, g[i], w, abs(rne - w),
               int((d > allow).sum()), d.size))
    return d.max(), d.mean()


def assert_within_one_ulp(got: torch.Tensor, want: np.ndarray, what: str):
    """Every bf16 element within one bf16 ulp (plus ULP_ABS_FLOOR) of the exact value."""
    g = f64(got)
    w = np.asarray(want, dtype=np.float64)
    ulp = bf16_ulp(w)
    bad = np.abs(g - w) > ulp + ULP_ABS_FLOOR
    assert not bad.any(), "%s: %d elements off by more than one bf16 ulp (worst %.3g ulp)" % (
        what, bad.sum(), (np.abs(g - w) / ulp).max())


def oracle_cache_after(k_rot_f64, v_f64, B, Hkv, Lmax, D):
    """Float64 caches [B, Hkv, Lmax, D] holding prompt slots 0..T-1 (rest zero)."""
    T = k_rot_f64.shape[1]
    kc = np.zeros((B, Hkv, Lmax, D))
    vc = np.zeros((B, Hkv, Lmax, D))
    kc[:, :, :T] = k_rot_f64.transpose(0, 2, 1, 3)
    vc[:, :, :T] = v_f64.transpose(0, 2, 1, 3)
    return kc, vc


def assert_grad_close(got: torch.Tensor, want: np.ndarray, what: str):
    """Gradient check: |d| <= GRAD_MAX_ABS + one bf16 ulp of the exact value,
    mean |d| <= GRAD_MEAN_ABS."""
    g = f64(got)
    assert g.shape == want.shape, (what, g.shape, want.shape)
    assert np.isfinite(g).all(), "%s: non-finite gradient" % what
    d = np.abs(g - want)
    allow = GRAD_MAX_ABS + bf16_ulp(want)
    worst = float((d / allow).max())
    assert (d <= allow).all() and d.mean() <= GRAD_MEAN_ABS, \
        "%s: max |d| %.4g (worst %.3f of the bound), mean |d| %.3g" % (what, d.max(), worst, d.mean())
    return float(d.max()), float(d.mean())


def prompt_refs(q_bits, k_bits, v_bits, qk_norm, doc_id=None, scaling=None):
    """For a prompt prefill from position 0 on these bf16 inputs: the exact
    result (the float64 oracle) and the bf16 floor (ideal, W) built from the
    oracle's rotated q and K."""
    B, T = q_bits.shape[:2]
    exact, k_rot, v = oracle.prefill(q_bits, k_bits, v_bits, qk_norm, scaling=scaling,
                                     doc_id=doc_id)
    pos = oracle.positions(0, B, T)
    q_rot = oracle.prep(q_bits, pos, qk_norm, scaling=scaling)
    ideal, W = ideal_attention(q_rot, k_rot, v, pos, qdoc=doc_id, kdoc=doc_id)
    return exact, ideal, W


def chunk_refs(q_bits, k_bits, v_bits, kc, vc, pos0, qk_norm, n_tok=None):
    """For a continuation chunk: the exact result and the bf16 floor.  kc / vc
    [B, Hkv, Lmax, D] hold the cached prefix (bf16 bits or float64); the floor
    sees the keys the oracle assembles -- the prefix, then the chunk's own
    rotated keys -- with query t of sequence b at position pos0[b] + t.  Rows
    t >= n_tok[b] are NaN in all three."""
    B, T, Hkv = q_bits.shape[0], q_bits.shape[1], k_bits.shape[2]
    D = q_bits.shape[3]
    exact, k_rot = oracle.prefill_chunk(q_bits, k_bits, v_bits, kc, vc, pos0, qk_norm,
                                        n_tok=n_tok)
    pos0 = np.broadcast_to(np.asarray(pos0, dtype=np.int64), (B,))
    n_tok = np.full(B, T, dtype=np.int64) if n_tok is None else np.asarray(n_tok, np.int64)
    qpos = oracle.positions(pos0, B, T)
    q_rot = oracle.prep(q_bits, qpos, qk_norm)
    kw, vw, v_new = oracle.widen(kc), oracle.widen(vc), oracle.widen(v_bits)
    Tk = max(1, int((pos0 + n_tok).max()))
    keys = np.zeros((B, Tk, Hkv, D))
    vals = np.zeros((B, Tk, Hkv, D))
    for b in range(B):
        P, n = int(pos0[b]), int(n_tok[b])
        keys[b, :P] = kw[b, :, :P].transpose(1, 0, 2)
        vals[b, :P] = vw[b, :, :P].transpose(1, 0, 2)
        keys[b, P:P + n] = k_rot[b, :n]
        vals[b, P:P + n] = v_new[b, :n]
    ideal, W = ideal_attention(q_rot, keys, vals, qpos)
    for b in range(B):
        ideal[b, int(n_tok[b]):] = np.nan
        W[b, int(n_tok[b]):] = np.nan
    return exact, ideal, W
