"""GPU parity: QK-RMSNorm + RoPE on q, and the fused K/V append into the cache.

Compared with the float64 oracle on the same bf16 inputs:
* rotated q and the cached K: every element within one bf16 ulp of the exact value;
* cached V: the input bits, exactly;
* cache slots outside [pos0, pos0 + T): their previous (sentinel) bits, exactly.
"""
import numpy as np
import pytest
import torch

import oracle
import rope_gqa_kv_b200 as gqa
from rope_gqa_kv_b200 import inputs

from helpers import assert_within_one_ulp, bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(B, T, Hq, Hkv, D, L, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, T, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, T, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, T, Hkv, D, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, Hkv, L, D, generator=g).to(torch.bfloat16)   # sentinel contents
    vc = torch.randn(B, Hkv, L, D, generator=g).to(torch.bfloat16)
    return q, k, v, kc, vc


@pytest.mark.parametrize("D", [64, 96, 128])
@pytest.mark.parametrize("qk_norm", [False, True])
def test_rope_append_matches_oracle(cuda_lib, D, qk_norm):
    B, T, Hq, Hkv, L = 3, 37, 6, 2, 256
    q, k, v, kc, vc = _case(B, T, Hq, Hkv, D, L, seed=D + qk_norm)
    pos0 = torch.tensor([0, 50, 219], dtype=torch.int32)
    dq, dk, dv = q.to(DEV), k.to(DEV), v.to(DEV)
    dkc, dvc = kc.to(DEV), vc.to(DEV)
    dpos = pos0.to(DEV)
    new_len = torch.full((B,), -7, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gqa.gqa_rope_append(dq, dk, dv, dkc, dvc, pos0=dpos, max_pos0=int(pos0.max()),
                        new_len=new_len, qk_norm=qk_norm, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert new_len.cpu().tolist() == (pos0 + T).tolist()

    want_q = oracle.rope_apply(bits(q), pos0.numpy(), qk_norm)
    want_k = oracle.rope_apply(bits(k), pos0.numpy(), qk_norm)
    assert_within_one_ulp(dq, want_q, "q")
    got_kc, got_vc = dkc.cpu(), dvc.cpu()
    for b in range(B):
        p = int(pos0[b])
        sl = slice(p, p + T)
        assert_within_one_ulp(got_kc[b, :, sl].transpose(0, 1), want_k[b], "k_cache[%d]" % b)
        assert torch.equal(got_vc[b, :, sl].transpose(0, 1).view(torch.int16),
                           v[b].view(torch.int16)), "v_cache must hold the input bits"
        keep = torch.ones(L, dtype=torch.bool)
        keep[sl] = False
        assert torch.equal(got_kc[b][:, keep].view(torch.int16), kc[b][:, keep].view(torch.int16))
        assert torch.equal(got_vc[b][:, keep].view(torch.int16), vc[b][:, keep].view(torch.int16))


@pytest.mark.parametrize("Hq,Hkv,D,T", [(2, 1, 128, 5), (4, 2, 64, 6), (3, 1, 96, 4),
                                        (1, 1, 128, 9), (8, 8, 64, 3), (2, 2, 128, 2),
                                        (12, 4, 128, 7)])
def test_rope_append_head_mixes_and_short_chunks(cuda_lib, Hq, Hkv, D, T):
    """Head counts whose query, key and value vectors share a warp's pass (the
    prompt kernel walks a token's Hq + 2 Hkv vectors 4 (D = 64: 8) at a time),
    chunks of 4 to 9 tokens with a ragged last block, and 2 or 3 tokens (the
    per-token kernel)."""
    B, L = 2, 128
    q, k, v, kc, vc = _case(B, T, Hq, Hkv, D, L, seed=100 + Hq + D + T)
    pos0 = torch.tensor([0, 117 - T], dtype=torch.int32)
    dq, dk, dv = q.to(DEV), k.to(DEV), v.to(DEV)
    dkc, dvc = kc.to(DEV), vc.to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gqa.gqa_rope_append(dq, dk, dv, dkc, dvc, pos0=pos0.to(DEV), max_pos0=int(pos0.max()),
                        qk_norm=True, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert_within_one_ulp(dq, oracle.rope_apply(bits(q), pos0.numpy(), True), "q")
    want_k = oracle.rope_apply(bits(k), pos0.numpy(), True)
    got_kc, got_vc = dkc.cpu(), dvc.cpu()
    for b in range(B):
        p = int(pos0[b])
        sl = slice(p, p + T)
        assert_within_one_ulp(got_kc[b, :, sl].transpose(0, 1), want_k[b], "k_cache[%d]" % b)
        assert torch.equal(got_vc[b, :, sl].transpose(0, 1).view(torch.int16),
                           v[b].view(torch.int16))
        keep = torch.ones(L, dtype=torch.bool)
        keep[sl] = False
        assert torch.equal(got_kc[b][:, keep].view(torch.int16), kc[b][:, keep].view(torch.int16))
        assert torch.equal(got_vc[b][:, keep].view(torch.int16), vc[b][:, keep].view(torch.int16))


def test_fused_equals_separate_calls(cuda_lib):
    B, T, Hq, Hkv, D, L = 2, 129, 8, 2, 128, 384
    q, k, v, kc, vc = _case(B, T, Hq, Hkv, D, L, seed=11)
    pos0 = torch.tensor([3, 200], dtype=torch.int32, device=DEV)
    a = [t.to(DEV) for t in (q, k, v, kc, vc)]
    bq, bk, bv, bkc, bvc = [t.to(DEV) for t in (q, k, v, kc, vc)]
    gqa.gqa_rope_append(*a, pos0=pos0, qk_norm=True)
    gqa.gqa_rope_apply(bq, pos0=pos0, qk_norm=True)
    gqa.kv_cache_append(bk, bv, bkc, bvc, pos0=pos0, qk_norm=True)
    torch.cuda.synchronize()
    assert torch.equal(a[0].view(torch.int16), bq.view(torch.int16))
    assert torch.equal(a[3].view(torch.int16), bkc.view(torch.int16))
    assert torch.equal(a[4].view(torch.int16), bvc.view(torch.int16))


def test_device_capacity_overflow_skips_only_that_sequence(cuda_lib):
    B, T, Hq, Hkv, D, L = 2, 10, 2, 1, 64, 128
    q, k, v, kc, vc = _case(B, T, Hq, Hkv, D, L, seed=12)
    pos0 = torch.tensor([5, 125], dtype=torch.int32, device=DEV)   # 125 + 10 > 128
    dkc, dvc = kc.to(DEV), vc.to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gqa.kv_cache_append(k.to(DEV), v.to(DEV), dkc, dvc, pos0=pos0, status=status)
    torch.cuda.synchronize()
    assert status.item() & gqa.GQA_DEV_CAPACITY
    assert torch.equal(dkc[1].cpu().view(torch.int16), kc[1].view(torch.int16))
    assert torch.equal(dvc[1].cpu().view(torch.int16), vc[1].view(torch.int16))
    assert not torch.equal(dkc[0].cpu().view(torch.int16), kc[0].view(torch.int16))


def test_host_capacity_check_raises(cuda_lib):
    k = torch.zeros(1, 8, 1, 64, dtype=torch.bfloat16, device=DEV)
    kc = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(gqa.GqaError):
        gqa.kv_cache_append(k, k, kc, kc.clone(), max_pos0=121)


def test_prefill_sized_rope_append_3p8b(cuda_lib):
    """The 3.8B-style layer at full size: B=8, T=2048, 24/8 heads, D=128, QK-norm."""
    w = inputs.BY_NAME["prefill_3p8b"]
    x = inputs.make_inputs(w)
    dq, dk, dv = x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV)
    dkc, dvc = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
    gqa.gqa_rope_append(dq, dk, dv, dkc, dvc, qk_norm=True, max_pos0=0)
    torch.cuda.synchronize()
    # sampled sequences and heads against the oracle
    for b in (0, 7):
        want_q = oracle.rope_apply(bits(x["q"][b:b + 1]), [0], True)
        assert_within_one_ulp(dq[b:b + 1], want_q, "q[%d]" % b)
        want_k = oracle.rope_apply(bits(x["k"][b:b + 1]), [0], True)
        assert_within_one_ulp(dkc[b].transpose(0, 1).unsqueeze(0).contiguous(), want_k,
                              "k_cache[%d]" % b)
    assert torch.equal(dvc.transpose(1, 2).reshape(x["v"].shape).view(torch.int16),
                       dv.view(torch.int16))
