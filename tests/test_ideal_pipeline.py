"""Pins of the bf16 floor that bounds the tensor-core paths (CPU only).

`ideal_pipeline.ideal_attention` is the float64 oracle's attention with the
three roundings a bf16 tensor-core pipeline makes (rotated q and K, the
probabilities, the output).  Here: without the roundings it is the oracle; its
rounding is round-to-nearest-even with bf16's 8 significant bits; a pipeline
that rounds the probabilities at other scales (per key tile, against a running
maximum, as the kernels do) stays within the stated margin of it; and on the
smoke draw the floor itself fails 1e-2 plus half an ulp, which is why the
prefill paths are held to the floor and not to that flat bound.  The same for
the backward's floor (`ideal_attention_backward`): the oracle's gradients
without roundings, a float32 pipeline within its margin, and the flat bound
its floor needs.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from rope_gqa_kv_b200 import inputs

from ideal_pipeline import (BW_SLACK, P_ROUND, _f64, bf16_ulp, ideal_attention,
                            ideal_attention_backward, round_bf16)


def _bits(t):
    return inputs.bits(t)


def _prompt(B, T, Hq, Hkv, D, seed, qk_norm=True):
    w = inputs.custom("ideal", B=B, Hq=Hq, Hkv=Hkv, D=D, T=T, qk_norm=qk_norm, seed_index=seed)
    x = inputs.make_inputs(w)
    exact, k_rot, v = oracle.prefill(_bits(x["q"]), _bits(x["k"]), _bits(x["v"]), qk_norm)
    pos = oracle.positions(0, B, T)
    q_rot = oracle.prep(_bits(x["q"]), pos, qk_norm)
    return exact, q_rot, k_rot, v, pos


def test_without_roundings_it_is_the_oracle():
    exact, q_rot, k_rot, v, pos = _prompt(2, 150, 6, 2, 64, 1)
    got, _ = ideal_attention(q_rot, k_rot, v, pos, rounded=False)
    assert np.abs(got - exact).max() < 1e-12
    # documents: the oracle's document mask
    ids = inputs.packed_doc_ids(2, 150, 20.0, seed=3).numpy()
    want = oracle.attention(q_rot, k_rot, v, pos, qdoc=ids, kdoc=ids)
    got, _ = ideal_attention(q_rot, k_rot, v, pos, qdoc=ids, kdoc=ids, rounded=False)
    assert np.abs(got - want).max() < 1e-12
    # queries at later positions over a longer key range (a continuation chunk)
    qpos = pos[:, :50] + 100
    want = oracle.attention(q_rot[:, :50], k_rot, v, qpos)
    got, _ = ideal_attention(q_rot[:, :50], k_rot, v, qpos, rounded=False)
    assert np.abs(got - want).max() < 1e-12


def test_rounding_is_nearest_even_to_bf16():
    g = torch.Generator().manual_seed(0)
    x = (torch.randn(1 << 18, generator=g) * torch.exp(torch.randn(1 << 18, generator=g) * 4))
    # 9 significant bits with the last one set: exact ties at 8 bits
    ties = torch.ldexp(torch.randint(128, 256, (4096,), generator=g).double() * 2 + 1,
                       torch.randint(-40, 40, (4096,), generator=g)) / 256.0
    for v in (x.double(), ties, -ties):
        want = v.float().to(torch.bfloat16).double()    # float32 -> bf16: one rounding
        assert torch.equal(round_bf16(v), want)


def _tiled_pipeline(q_rot, k_rot, v, scale, tile=128, lazy_log2=8.0):
    """A kernel-like float64 pipeline for a prompt: keys in tiles of 128; each
    tile's probabilities are taken against the running maximum, which is only
    raised (and the accumulator rescaled) when the tile's maximum passes it by
    more than 2^lazy_log2; those probabilities are rounded to bf16 for the
    P.V sum, the row sum uses them unrounded; the output is rounded."""
    B, T, Hq, D = q_rot.shape
    Hkv = k_rot.shape[2]
    g = Hq // Hkv
    out = np.zeros(q_rot.shape)
    thr = lazy_log2 * math.log(2.0)
    for b in range(B):
        for h in range(Hq):
            Q = round_bf16(torch.as_tensor(q_rot[b, :, h]))
            K = round_bf16(torch.as_tensor(k_rot[b, :, h // g]))
            V = torch.as_tensor(v[b, :, h // g])
            S = (Q @ K.T) * scale
            for t in range(T):
                m, L, acc = -math.inf, 0.0, torch.zeros(D, dtype=torch.float64)
                for j0 in range(0, t + 1, tile):
                    s = S[t, j0:min(t + 1, j0 + tile)]
                    mt = float(s.max())
                    if mt > m + thr or m == -math.inf:
                        if m != -math.inf:
                            acc = acc * math.exp(m - mt)
                            L = L * math.exp(m - mt)
                        m = mt
                    p = torch.exp(s - m)
                    L += float(p.sum())
                    acc = acc + round_bf16(p) @ V[j0:j0 + len(s)]
                out[b, t, h] = round_bf16(acc / L).numpy()
    return out


def test_a_pipeline_rounding_p_per_tile_stays_within_the_margin():
    """The margin 2^-7 W + one ulp covers where a kernel rounds P."""
    exact, q_rot, k_rot, v, pos = _prompt(1, 400, 4, 2, 64, 5)
    ideal, W = ideal_attention(q_rot, k_rot, v, pos)
    for lazy in (0.0, 8.0):
        sim = _tiled_pipeline(q_rot, k_rot, v, 1.0 / 8.0, lazy_log2=lazy)
        margin = P_ROUND * W + bf16_ulp(np.abs(ideal) + P_ROUND * W)
        d = np.abs(sim - ideal)
        assert (d <= margin).all(), (lazy, float((d - margin).max()))
        # and the margin is not vacuous: the two pipelines do differ
        assert d.max() > 0


def test_the_floor_passes_the_flat_bound_on_the_smoke_draw():
    """The smoke draw (2 x 200 tokens, 6/2 heads, D=128, QK-norm): no bf16
    pipeline meets max |d| <= 1e-2 + half an ulp on every element -- its floor
    does not -- while its mean stays far below 1e-3."""
    w = inputs.custom("smoke", B=2, Hq=6, Hkv=2, D=128, T=200, decode_steps=1, qk_norm=True)
    x = inputs.make_inputs(w)
    exact, k_rot, v = oracle.prefill(_bits(x["q"]), _bits(x["k"]), _bits(x["v"]), True)
    pos = oracle.positions(0, w.B, w.T)
    ideal, _ = ideal_attention(oracle.prep(_bits(x["q"]), pos, True), k_rot, v, pos)
    floor = np.abs(ideal - exact)
    assert (floor > 1e-2 + 0.5 * bf16_ulp(exact)).any()
    assert 1.1e-2 < floor.max() < 1.5e-2
    assert floor.mean() < 1e-3


# --- the backward's floor ---------------------------------------------------

def _bw_case(B, T, Hq, Hkv, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, T, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, T, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, T, Hkv, D, generator=g).to(torch.bfloat16)
    do = torch.randn(B, T, Hq, D, generator=g).to(torch.bfloat16)
    return [_bits(t) for t in (q, k, v, do)]


def test_backward_without_roundings_is_the_oracle():
    q, k, v, do = _bw_case(2, 150, 6, 2, 64, 11)
    rq, rk, rv, ro, rl = oracle.attention_backward(q, k, v, do)
    got = ideal_attention_backward(q, k, v, do, ro, rl, rounded=False)
    for name, want in (("dq", rq), ("dk", rk), ("dv", rv)):
        assert np.abs(got[name][0] - want).max() < 1e-12 * max(1.0, np.abs(want).max()), name
        # W bounds the magnitude of what it sums
        assert (np.abs(want) <= got[name][1] * (1 + 1e-12) + 1e-15).all(), name


def _kernel_like_backward(q, k, v, do, o, lse, tile=128):
    """A float32 backward shaped like a tensor-core kernel's: scores and dP in
    float32, P = 2^(S c log2e - lse log2e), dS = P (dP - Delta), P and dS rounded
    to bf16 (float32 -> bf16, nearest even) before the products, the products
    summed in float32 a 128-row tile at a time, outputs c-scaled in float32 and
    rounded to bf16."""
    f32 = lambda t: torch.as_tensor(t).float()
    q, k, v, do, o = (f32(_f64(t)) for t in (q, k, v, do, o))
    lse = f32(lse)
    B, T, Hq, D = q.shape
    g = Hq // k.shape[2]
    c = 1.0 / math.sqrt(D)
    l2e = 1.0 / math.log(2.0)
    r16 = lambda t: t.to(torch.bfloat16).float()
    dq = torch.zeros(B, T, Hq, D)
    dk = torch.zeros(B, T, k.shape[2], D)
    dv = torch.zeros_like(dk)
    future = torch.ones(T, T, dtype=torch.bool).triu(1)
    for b in range(B):
        for h in range(Hq):
            kh = h // g
            Q, K, V, dO, O = q[b, :, h], k[b, :, kh], v[b, :, kh], do[b, :, h], o[b, :, h]
            P = torch.exp2((Q @ K.T) * (c * l2e) - lse[b, h][:, None] * l2e).masked_fill(future, 0)
            dS = P * (dO @ V.T - (dO * O).sum(dim=1, keepdim=True))
            Pr, dSr = r16(P), r16(dS)
            for i0 in range(0, T, tile):              # query tiles into dK, dV
                dv[b, :, kh] += Pr[i0:i0 + tile].T @ dO[i0:i0 + tile]
                dk[b, :, kh] += dSr[i0:i0 + tile].T @ Q[i0:i0 + tile]
            for j0 in range(0, T, tile):              # key tiles into dQ
                dq[b, :, h] += dSr[:, j0:j0 + tile] @ K[j0:j0 + tile]
    return {"dq": r16(dq * c).double().numpy(), "dk": r16(dk * c).double().numpy(),
            "dv": r16(dv).double().numpy()}


def test_a_float32_backward_stays_within_the_margin():
    """The margin 2^-7 W + one ulp + the stated slack covers a pipeline that
    takes every step in float32 and rounds where a bf16 backward does."""
    q, k, v, do = _bw_case(1, 300, 6, 2, 128, 12)
    rq, rk, rv, ro, rl = oracle.attention_backward(q, k, v, do)
    o16 = round_bf16(torch.as_tensor(ro)).numpy()
    l32 = rl.astype(np.float32).astype(np.float64)
    ideal = ideal_attention_backward(q, k, v, do, o16, l32)
    sim = _kernel_like_backward(q, k, v, do, o16, l32)
    for name in ("dq", "dk", "dv"):
        want, W = ideal[name]
        d = np.abs(sim[name] - want)
        margin = P_ROUND * W + bf16_ulp(np.abs(want) + P_ROUND * W) + BW_SLACK
        assert (d <= margin).all(), (name, float((d - margin).max()))
        assert d.max() > 0, name


def test_the_backward_floor_needs_the_flat_gradient_bound():
    """One sequence of the 3.8B layer's heads (T = 2048, 24/8 heads, D = 128):
    the floor itself misses 1e-2 + one ulp of the exact gradient on some
    element but meets 2e-2 + one ulp on all, with its mean far below 1e-3 --
    why the flat gradient bound is 2e-2 and the per-element one the floor."""
    q, k, v, do = _bw_case(1, 2048, 24, 8, 128, 2048 + 128)
    rq, rk, rv, ro, rl = oracle.attention_backward(q, k, v, do)
    ideal = ideal_attention_backward(q, k, v, do, round_bf16(torch.as_tensor(ro)).numpy(),
                                     rl.astype(np.float32).astype(np.float64))
    over_1e2 = 0
    for name, exact in (("dq", rq), ("dk", rk), ("dv", rv)):
        floor = np.abs(ideal[name][0] - exact)
        assert (floor <= 2e-2 + bf16_ulp(exact)).all(), name
        assert floor.mean() < 1e-3, name
        over_1e2 += int((floor > 1e-2 + bf16_ulp(exact)).sum())
    assert over_1e2 > 0
