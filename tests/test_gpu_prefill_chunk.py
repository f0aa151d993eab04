"""GPU parity: continuation chunks (gqa_prefill_chunk) against the float64 oracle.

A chunk is T new tokens per sequence after a cached prefix of pos0[b] tokens:
gqa_rope_append writes their rotated K and raw V at slots pos0[b] .. and
gqa_prefill_chunk runs the causal attention of query t at position pos0[b] + t
over the cache.  Cases: whole outputs at sizes the oracle finishes in seconds
(several tiles, prefixes that are not multiples of 128, ragged tails, every
head_dim, MHA / GQA / MQA), per-sequence token counts with NaN padding, invalid
sequences, agreement with gqa_prefill when every prefix is empty, a prompt
prefilled in three chunks against one prefill, and every output element at
the 3.8B-style chunk size the benchmark times.  The bound is the bf16 floor
of a tensor-core pipeline plus its stated margin (ideal_pipeline.py), and mean
|d| <= 1e-3 against the exact result.
"""
import numpy as np
import pytest
import torch

import oracle
import rope_gqa_kv_b200 as gqa
from rope_gqa_kv_b200 import inputs

from helpers import assert_floor_close, bits, chunk_refs, ideal_attention, prompt_refs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run_chunk(x, w, n_tok=None, out=None):
    dq, dk, dv = x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV)
    dkc, dvc = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
    pos0 = x["lens"].to(DEV)
    max_pos0 = int(x["lens"].max())
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gqa.gqa_rope_append(dq, dk, dv, dkc, dvc, pos0=pos0, max_pos0=max_pos0, qk_norm=w.qk_norm,
                        status=status)
    nt = None if n_tok is None else torch.as_tensor(n_tok, dtype=torch.int32, device=DEV)
    o = gqa.gqa_prefill_chunk(dq, dkc, dvc, pos0, max_pos0, n_tok=nt, out=out, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, "device status %#x" % status.item()
    return o, dkc, dvc


def _refs(x, w, n_tok=None, sl=slice(None)):
    """(exact, ideal, W) of the chunk of sequences `sl`."""
    return chunk_refs(bits(x["q"][sl]), bits(x["k"][sl]), bits(x["v"][sl]),
                      bits(x["k_cache"][sl]), bits(x["v_cache"][sl]), x["lens"][sl].numpy(),
                      w.qk_norm, n_tok=n_tok)


@pytest.mark.parametrize("B,T,Hq,Hkv,D,qk,lo,hi", [
    (3, 300, 12, 4, 128, True, 0, 600),     # prefixes of any length, ragged pair
    (2, 200, 8, 8, 96, False, 100, 400),    # MHA, D = 96
    (2, 129, 8, 1, 64, True, 1, 300),       # MQA, one row into the second tile
    (4, 1, 6, 2, 128, True, 0, 900),        # one new token: a decode step
    (1, 512, 4, 2, 64, False, 128, 128),    # prefix exactly one tile
    (2, 64, 6, 3, 128, True, 1000, 1300),   # long prefix, short chunk
])
def test_chunk_shapes(cuda_lib, B, T, Hq, Hkv, D, qk, lo, hi):
    w = inputs.custom("chk", B=B, Hq=Hq, Hkv=Hkv, D=D, T=T, qk_norm=qk,
                      cached_len_range=(lo, hi), seed_index=T + D + lo)
    x = inputs.make_inputs(w)
    o, _, _ = _run_chunk(x, w)
    exact, ideal, W = _refs(x, w)
    assert_floor_close(o, exact, ideal, W,
                       "chunk B%d T%d Hq%d Hkv%d D%d prefix U[%d,%d]" % (B, T, Hq, Hkv, D, lo, hi))


def test_chunk_token_counts_with_nan_padding(cuda_lib):
    """Per-sequence token counts; the padding rows of q, k, v are NaN, so the
    appended padding fills cache slots past the valid keys with NaN too."""
    w = inputs.custom("chk", B=3, Hq=6, Hkv=2, D=128, T=300, qk_norm=True,
                      cached_len_range=(50, 700), seed_index=71)
    x = inputs.make_inputs(w)
    n_tok = [300, 1, 77]
    for b, n in enumerate(n_tok):
        for key in ("q", "k", "v"):
            x[key][b, n:] = float("nan")
    sentinel = torch.full((3, 300, 6, 128), 5.0, dtype=torch.bfloat16, device=DEV)
    o, _, _ = _run_chunk(x, w, n_tok=n_tok, out=sentinel)
    exact, ideal, W = _refs(x, w, n_tok=np.array(n_tok))
    for b, n in enumerate(n_tok):
        assert_floor_close(o[b, :n], exact[b, :n], ideal[b, :n], W[b, :n],
                           "sequence %d (%d tokens)" % (b, n))
        assert (o[b, n:] == 5.0).all(), "rows past n_tok[%d] were written" % b


def test_chunk_with_empty_prefix_is_prefill_bit_for_bit(cuda_lib):
    w = inputs.custom("pf", B=2, Hq=6, Hkv=2, D=128, T=333, qk_norm=True, seed_index=72)
    x = inputs.make_inputs(w)
    dq, dk, dv = x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV)
    kc, vc = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
    gqa.gqa_rope_append(dq, dk, dv, kc, vc, qk_norm=True)
    a = gqa.gqa_prefill(dq, kc, vc)
    zeros = torch.zeros(2, dtype=torch.int32, device=DEV)
    b = gqa.gqa_prefill_chunk(dq, kc, vc, zeros, 0)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_prompt_in_three_chunks_matches_one_prefill(cuda_lib):
    B, T, Hq, Hkv, D, L = 2, 1000, 8, 2, 128, 1024
    w = inputs.custom("pf", B=B, Hq=Hq, Hkv=Hkv, D=D, T=T, qk_norm=True, seed_index=73)
    x = inputs.make_inputs(w, Lmax=L)
    q, k, v = x["q"], x["k"], x["v"]
    kc1, vc1 = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
    qa = q.to(DEV)
    gqa.gqa_rope_append(qa, k.to(DEV), v.to(DEV), kc1, vc1, qk_norm=True)
    full = gqa.gqa_prefill(qa, kc1, vc1)
    kc2, vc2 = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
    outs = []
    for a, b in [(0, 400), (400, 800), (800, 1000)]:
        qc = q[:, a:b].contiguous().to(DEV)
        pos0 = torch.full((B,), a, dtype=torch.int32, device=DEV)
        gqa.gqa_rope_append(qc, k[:, a:b].contiguous().to(DEV), v[:, a:b].contiguous().to(DEV),
                            kc2, vc2, pos0=pos0, max_pos0=a, qk_norm=True)
        outs.append(gqa.gqa_prefill_chunk(qc, kc2, vc2, pos0, a))
    torch.cuda.synchronize()
    chunked = torch.cat(outs, dim=1)
    assert torch.equal(kc1[:, :, :T].view(torch.int16), kc2[:, :, :T].view(torch.int16))
    d = (chunked.float() - full.float()).abs()
    assert d.max().item() <= 1e-2, d.max().item()
    exact, ideal, W = prompt_refs(bits(q), bits(k), bits(v), True)
    assert_floor_close(chunked, exact, ideal, W, "prompt in three chunks")


def test_chunk_invalid_sequences(cuda_lib):
    B, T, Hq, Hkv, D, L = 3, 64, 4, 2, 64, 1024
    g = torch.Generator().manual_seed(74)
    q = torch.randn(B, T, Hq, D, generator=g).to(torch.bfloat16).to(DEV)
    kc = torch.randn(B, Hkv, L, D, generator=g).to(torch.bfloat16).to(DEV)
    vc = torch.randn(B, Hkv, L, D, generator=g).to(torch.bfloat16).to(DEV)
    pos0 = torch.tensor([-1, 10, 1000], dtype=torch.int32, device=DEV)   # 1000 + 64 > 1024
    out = torch.full_like(q, 7.0)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gqa.gqa_prefill_chunk(q, kc, vc, pos0, 900, out=out, status=status)
    torch.cuda.synchronize()
    st = status.item()
    assert st & gqa.GQA_DEV_BAD_LEN and st & gqa.GQA_DEV_CAPACITY
    assert (out[0] == 7.0).all() and (out[2] == 7.0).all()
    keys = bits(kc[1:2].cpu())[:, :, :74].transpose(0, 2, 1, 3)
    vals = bits(vc[1:2].cpu())[:, :, :74].transpose(0, 2, 1, 3)
    q64 = oracle.bf16_to_f64(bits(q[1:2].cpu()))
    k64, v64 = oracle.bf16_to_f64(keys), oracle.bf16_to_f64(vals)
    qpos = (10 + np.arange(T))[None, :]
    exact = oracle.attention(q64, k64, v64, qpos)
    ideal, W = ideal_attention(q64, k64, v64, qpos)
    assert_floor_close(out[1:2], exact, ideal, W, "valid sequence between invalid ones")


def test_chunk_3p8b_size_every_element(cuda_lib):
    """8 sequences, prefixes U[512, 1536], 1024 new tokens, 24/8 heads, D=128,
    QK-norm: the launch the benchmark times for continuation chunks, every
    output element against the oracle, one sequence at a time."""
    w = inputs.BY_NAME["chunked_prefill_3p8b"]
    x = inputs.make_inputs(w)
    o, _, _ = _run_chunk(x, w)
    o = o.cpu()
    worst, means = 0.0, []
    for b in range(w.B):
        exact, ideal, W = _refs(x, w, sl=slice(b, b + 1))
        d, _, m = assert_floor_close(o[b:b + 1], exact, ideal, W, "3.8B chunk, sequence %d" % b)
        worst = max(worst, d)
        means.append(m)
    assert np.mean(means) <= 1e-3
    print("3.8B chunk: max|d| %.4g, mean|d| %.3g over %d elements" % (worst, np.mean(means),
                                                                     o.numel()))
