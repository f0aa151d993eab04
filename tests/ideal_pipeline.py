"""The bf16 floor of a tensor-core attention pipeline, built from the oracle.

Test infrastructure: it uses the float64 oracle's values (rotated q and k,
values) and explicit roundings only -- no kernel output.

A kernel that keeps its tensors in bf16 rounds three things the float64 oracle
does not:
  * the rotated q and K it stores (bf16: q in place, K in the cache);
  * the probabilities P it hands to the tensor core for the P.V product (bf16);
  * its output (bf16).
`ideal_attention` computes causal GQA attention with exactly those roundings
and every other step exact (float64), normalising by the sum of the unrounded
probabilities as the kernels do: the smallest error a kernel of that design can
have on given inputs -- the floor -- element by element.

It also returns, per output element (row, coordinate d), W = sum_j p_j |v_jd| /
sum_j p_j.  Rounding
one probability to nearest with bf16's 8 significant bits moves it by at most
2^-8 of itself, so rounding all of them moves the normalised sum by at most
2^-8 W.  A kernel rounds P at other points of its range than the ideal
pipeline does (it scales P by the running maximum of a key tile, not the
row's final maximum), so before the outputs are rounded the two differ by at
most 2 * 2^-8 W = 2^-7 W, and after both round their outputs by at most that
plus one bf16 ulp.  `assert_floor_close` holds the kernel to this bound plus a
small stated slack, element by element.

`ideal_attention_backward` is the same construction for the gradients: the
roundings of P and dS where a bf16 backward hands them to the tensor core, and
of dq, dk, dv, with W the sum of the absolute terms of each output.
"""
from __future__ import annotations

import math

import numpy as np
import torch

MEAN_ABS = 1e-3          # the stated mean bound against the exact result
P_ROUND = 2.0 ** -7      # 2 x (bf16 relative rounding bound 2^-8) per unit of W
# Slack of the per-element bound: fp32 accumulation and the exp2 instruction
# (~1e-6 relative), and the kernel's own rounding of the rotated q and K: it
# rotates in fp32 and may land one bf16 ulp away from the rounding of the exact
# rotation used here (a few elements in 10^5), which moves a score by at most
# scale * |q_i| * ulp(k_i) -- about 5e-3 for the largest normalised elements --
# and the output by that times the weight of the key.
SLACK = 3e-3
# The backward's inputs are bf16 already (nothing is rotated): its slack covers
# fp32 accumulation of dP = dO V^T, Delta and the three gradient sums, the
# float32 log-sum-exp and the exp2 instruction.
BW_SLACK = 1e-3


def round_bf16(x: torch.Tensor) -> torch.Tensor:
    """float64 -> the nearest value with 8 significant bits, ties to even (the
    bf16 significand; bf16's exponent range holds every value rounded here)."""
    m, e = torch.frexp(x)
    return torch.ldexp(torch.round(m * 256.0) / 256.0, e)


def bf16_ulp(x):
    mag = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(mag)) - 7)


def ideal_attention(q_rot, k_rot, v, qpos, scale: float | None = None, qdoc=None, kdoc=None,
                    rounded: bool = True):
    """The bf16 pipeline's output and W for causal GQA attention.

    q_rot [B, Tq, Hq, D], k_rot / v [B, Tk, Hkv, D] (float64: the oracle's
    rotated q and K, and the values); qpos [B, Tq] the absolute position of each
    query (key slot j is visible to it when j <= qpos); qdoc [B, Tq] / kdoc
    [B, Tk] optional document ids (a key is then visible only inside the
    query's document).  rounded=False skips every rounding (it then equals the
    oracle's attention).  Returns (ideal [B, Tq, Hq, D], W [B, Tq, Hq, D]) as
    float64 numpy arrays; rows that see no key are NaN.
    """
    q_rot = torch.as_tensor(np.asarray(q_rot, dtype=np.float64))
    k_rot = torch.as_tensor(np.asarray(k_rot, dtype=np.float64))
    v = torch.as_tensor(np.asarray(v, dtype=np.float64))
    B, Tq, Hq, D = q_rot.shape
    Tk, Hkv = k_rot.shape[1], k_rot.shape[2]
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    rnd = round_bf16 if rounded else (lambda t: t)
    qpos = torch.as_tensor(np.broadcast_to(np.asarray(qpos, dtype=np.int64), (B, Tq)).copy())
    out = torch.full((B, Tq, Hq, D), float("nan"), dtype=torch.float64)
    wsum = torch.full((B, Tq, Hq, D), float("nan"), dtype=torch.float64)
    keys = torch.arange(Tk)
    for b in range(B):
        vis = keys[None, :] <= qpos[b][:, None]                            # [Tq, Tk]
        if qdoc is not None:
            qd = torch.as_tensor(np.asarray(qdoc)[b].astype(np.int64))
            kd = torch.as_tensor(np.asarray(kdoc)[b].astype(np.int64))
            vis = vis & (kd[None, :] == qd[:, None])
        seen = vis.any(dim=1)
        for kh in range(Hkv):
            heads = slice(kh * g, (kh + 1) * g)
            Q = rnd(q_rot[b, :, heads, :]).reshape(Tq * g, D)              # row = t * g + h'
            K = rnd(k_rot[b, :, kh, :])
            V = v[b, :, kh, :]
            S = (Q @ K.T) * scale
            mask = vis.repeat_interleave(g, dim=0)
            S = S.masked_fill(~mask, float("-inf"))
            m = S.max(dim=1, keepdim=True).values
            m = torch.where(torch.isfinite(m), m, torch.zeros_like(m))
            P = torch.exp(S - m)                                           # 0 where masked
            L = P.sum(dim=1, keepdim=True)
            A = (rnd(P) @ V) / L
            Wt = (P @ V.abs()) / L
            ok = seen.repeat_interleave(g)
            A[~ok] = float("nan")
            Wt[~ok] = float("nan")
            out[b, :, heads, :] = rnd(A).reshape(Tq, g, D)
            wsum[b, :, heads, :] = Wt.reshape(Tq, g, D)
    return out.numpy(), wsum.numpy()


def assert_floor_close(got, exact, ideal, W, what: str, slack: float = SLACK,
                       mean_abs: float = MEAN_ABS):
    """Element by element: |got - ideal| <= 2^-7 W + one bf16 ulp + slack, i.e.
    the kernel is within the bf16 pipeline's floor (|ideal - exact|) plus that
    margin of the exact result; and mean |got - exact| <= mean_abs.  Returns
    (max |got - exact|, max |ideal - exact|, mean |got - exact|)."""
    g = got.detach().cpu().to(torch.float64).numpy() if isinstance(got, torch.Tensor) else got
    g = np.asarray(g, dtype=np.float64)
    assert g.shape == ideal.shape == exact.shape, (what, g.shape, ideal.shape, exact.shape)
    assert np.isfinite(g).all(), "%s: non-finite output" % what
    margin = P_ROUND * W + bf16_ulp(np.abs(ideal) + P_ROUND * W) + slack
    d_ideal = np.abs(g - ideal)
    d_exact = np.abs(g - exact)
    floor = np.abs(ideal - exact)
    over = d_ideal > margin
    if over.any() or d_exact.mean() > mean_abs:
        i = np.unravel_index(np.argmax(d_ideal - margin), d_ideal.shape)
        raise AssertionError(
            "%s: %d of %d elements beyond the floor margin; worst at %s: got %.6g ideal %.6g "
            "exact %.6g (|got-ideal| %.3g > margin %.3g, W %.3g); mean|got-exact| %.3g "
            "(<= %.3g)" % (what, int(over.sum()), g.size, i, g[i], ideal[i], exact[i],
                           d_ideal[i], margin[i], W[i], d_exact.mean(), mean_abs))
    return float(d_exact.max()), float(floor.max()), float(d_exact.mean())


def _f64(t) -> torch.Tensor:
    """float64 tensor of an array of values, or of bf16 bit patterns (uint16)."""
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu()
        return t.double() if t.dtype != torch.uint16 else t.view(torch.int16).view(torch.bfloat16).double()
    a = np.asarray(t)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).double()
    return torch.as_tensor(a.astype(np.float64))


def ideal_attention_backward(q, k, v, dout, o, lse, scale: float | None = None,
                             rounded: bool = True):
    """The bf16 floor of the attention backward, given the forward's outputs.

    q, dout [B, T, Hq, D]; k, v [B, T, Hkv, D] (values, or bf16 bit patterns as
    uint16); o [B, T, Hq, D] the forward output the backward is handed (bf16
    values); lse [B, Hq, T] the forward's row log-sum-exp (natural log, the
    float32 values handed).  Every step is
    exact (float64) but the three roundings a bf16 tensor-core backward makes:
    the probabilities P it feeds to dV = P^T dO, the dS = P (dP - Delta) it
    feeds to dK = c dS^T Q and dQ = c dS K (Delta = rowsum(dO * o)), and the
    three outputs.  P = exp(S - lse) is taken from the lse handed, as a kernel
    that recomputes P does.  rounded=False skips the roundings (with the exact o
    and lse it then equals the oracle's gradients).

    Returns {"dq": (ideal, W), "dk": (ideal, W), "dv": (ideal, W)} in float64
    numpy, dq [B, T, Hq, D], dk / dv [B, T, Hkv, D], with W the sum of the
    absolute values of the terms each output sums (for dv: sum_i P_ij |dO_id|;
    for dk: c sum_i |dS_ij| |Q_id|; for dq: c sum_j |dS_ij| |K_jd|; dk and dv
    summed over the query heads of a group).  Rounding each term to bf16 moves
    it by at most 2^-8 of itself, so a kernel that rounds the same terms after
    fp32 arithmetic is within 2^-7 W of this pipeline before the outputs are
    rounded: `assert_floor_close` applies unchanged.
    """
    q, k, v, do, o, lse = (_f64(t) for t in (q, k, v, dout, o, lse))
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    rnd = round_bf16 if rounded else (lambda t: t)
    dq = torch.zeros(B, T, Hq, D, dtype=torch.float64)
    wq = torch.zeros_like(dq)
    dk = torch.zeros(B, T, Hkv, D, dtype=torch.float64)
    wk, dv, wv = torch.zeros_like(dk), torch.zeros_like(dk), torch.zeros_like(dk)
    future = torch.ones(T, T, dtype=torch.bool).triu(1)
    for b in range(B):
        for h in range(Hq):
            kh = h // g
            Q, K, V, dO, O = q[b, :, h], k[b, :, kh], v[b, :, kh], do[b, :, h], o[b, :, h]
            S = (Q @ K.T) * scale
            P = torch.exp(S - lse[b, h][:, None]).masked_fill(future, 0.0)
            delta = (dO * O).sum(dim=1, keepdim=True)
            dS = P * (dO @ V.T - delta)
            Pr, dSr = rnd(P), rnd(dS)
            dv[b, :, kh] += Pr.T @ dO
            wv[b, :, kh] += P.T @ dO.abs()
            dk[b, :, kh] += dSr.T @ Q
            wk[b, :, kh] += dS.abs().T @ Q.abs()
            dq[b, :, h] = scale * (dSr @ K)
            wq[b, :, h] = scale * (dS.abs() @ K.abs())
    return {"dq": (rnd(dq).numpy(), wq.numpy()),
            "dk": (rnd(scale * dk).numpy(), (scale * wk).numpy()),
            "dv": (rnd(dv).numpy(), wv.numpy())}
