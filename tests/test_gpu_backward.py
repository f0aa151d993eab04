"""GPU parity: the attention backward (gqa_prefill_lse + gqa_attention_backward)
against the float64 oracle's gradients.

Full gradients at sizes the oracle finishes in seconds (ragged tails, MHA, GQA,
MQA, every head_dim) and at the 3.8B layer's heads and length (T = 2048, 24/8
heads, D = 128; one sequence), two ways: forward and backward on the GPU, every
element within 2e-2 + one ulp of the oracle's gradient; and the backward alone,
handed the oracle's own forward (its output rounded to bf16, its log-sum-exp to
float32), every element within the bf16 floor of a tensor-core backward plus
its margin (ideal_pipeline.py).  Also the forward's log-sum-exp; the forward
output of gqa_prefill_lse equal to gqa_prefill's bit for bit; cache slots past
T of dk / dv untouched; repeat runs bit-identical.
"""
import numpy as np
import pytest
import torch

import oracle
import rope_gqa_kv_b200 as gqa

from helpers import assert_grad_close, bits
from ideal_pipeline import BW_SLACK, assert_floor_close, ideal_attention_backward

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(B, T, Hq, Hkv, D, seed, L=None):
    g = torch.Generator().manual_seed(seed)
    L = L or (T + 127) // 128 * 128
    q = torch.randn(B, T, Hq, D, generator=g).to(torch.bfloat16)
    kt = torch.randn(B, T, Hkv, D, generator=g).to(torch.bfloat16)
    vt = torch.randn(B, T, Hkv, D, generator=g).to(torch.bfloat16)
    dout = torch.randn(B, T, Hq, D, generator=g).to(torch.bfloat16)
    kc = torch.full((B, Hkv, L, D), float("nan"), dtype=torch.bfloat16)
    vc = kc.clone()
    kc[:, :, :T] = kt.transpose(1, 2)
    vc[:, :, :T] = vt.transpose(1, 2)
    return q, kt, vt, dout, kc, vc


def _run(q, dout, kc, vc, dk=None, dv=None):
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    dq_, dkc, dvc = q.to(DEV), kc.to(DEV), vc.to(DEV)
    o, lse = gqa.gqa_prefill_lse(dq_, dkc, dvc, status=st)
    grads = gqa.gqa_attention_backward(dq_, dkc, dvc, o, dout.to(DEV), lse, dk=dk, dv=dv,
                                       status=st)
    torch.cuda.synchronize()
    assert st.item() == 0, "device status %#x" % st.item()
    return o, lse, grads


@pytest.mark.parametrize("B,T,Hq,Hkv,D", [
    (1, 128, 2, 1, 64),       # one tile
    (2, 300, 6, 2, 128),      # GQA, ragged last tile
    (1, 513, 8, 8, 96),       # MHA, one row into the fifth tile
    (1, 385, 8, 1, 64),       # MQA
    (2, 1000, 8, 2, 128),
])
def test_backward_vs_oracle(cuda_lib, B, T, Hq, Hkv, D):
    q, kt, vt, dout, kc, vc = _case(B, T, Hq, Hkv, D, seed=T + D)
    o, lse, (dq, dk, dv) = _run(q, dout, kc, vc)
    rq, rk, rv, ro, rl = oracle.attention_backward(bits(q), bits(kt), bits(vt), bits(dout))
    np.testing.assert_allclose(lse[:, :, :T].double().cpu().numpy(), rl, rtol=0, atol=1e-5)
    assert_grad_close(dq, rq, "dq")
    assert_grad_close(dk[:, :, :T].transpose(1, 2), rk, "dk")
    assert_grad_close(dv[:, :, :T].transpose(1, 2), rv, "dv")


def test_backward_3p8b_heads_full_length(cuda_lib):
    """One sequence of the 3.8B layer's shape: T = 2048, 24 query / 8 KV heads, D = 128."""
    q, kt, vt, dout, kc, vc = _case(1, 2048, 24, 8, 128, seed=2048)
    _, _, (dq, dk, dv) = _run(q, dout, kc, vc)
    rq, rk, rv, _, _ = oracle.attention_backward(bits(q), bits(kt), bits(vt), bits(dout))
    assert_grad_close(dq, rq, "dq")
    assert_grad_close(dk[:, :, :2048].transpose(1, 2), rk, "dk")
    assert_grad_close(dv[:, :, :2048].transpose(1, 2), rv, "dv")


def _backward_alone(q, kt, vt, dout, kc, vc, what):
    """gqa_attention_backward handed the oracle's forward, against the floor."""
    B, T, Hq, D = q.shape
    rq, rk, rv, ro, rl = oracle.attention_backward(bits(q), bits(kt), bits(vt), bits(dout))
    o16 = torch.as_tensor(ro).to(torch.bfloat16)
    lse = torch.zeros(B, Hq, (T + 3) // 4 * 4, dtype=torch.float32)
    lse[:, :, :T] = torch.as_tensor(rl).float()
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    dq, dk, dv = gqa.gqa_attention_backward(q.to(DEV), kc.to(DEV), vc.to(DEV), o16.to(DEV),
                                            dout.to(DEV), lse.to(DEV), status=st)
    torch.cuda.synchronize()
    assert st.item() == 0, "device status %#x" % st.item()
    ideal = ideal_attention_backward(bits(q), bits(kt), bits(vt), bits(dout), o16.double(),
                                     lse[:, :, :T].double())
    for name, got, exact in (("dq", dq, rq), ("dk", dk[:, :, :T].transpose(1, 2), rk),
                             ("dv", dv[:, :, :T].transpose(1, 2), rv)):
        d, f, m = assert_floor_close(got, exact, *ideal[name], "%s %s" % (what, name),
                                     slack=BW_SLACK)
        print("%s %s: max|d| %.4g (floor %.4g), mean|d| %.3g" % (what, name, d, f, m))


@pytest.mark.parametrize("B,T,Hq,Hkv,D", [
    (1, 128, 2, 1, 64),
    (2, 300, 6, 2, 128),
    (1, 513, 8, 8, 96),
    (1, 385, 8, 1, 64),
    (2, 1000, 8, 2, 128),
    (1, 2048, 24, 8, 128),    # the 3.8B layer's heads, one sequence
])
def test_backward_alone_within_the_floor(cuda_lib, B, T, Hq, Hkv, D):
    q, kt, vt, dout, kc, vc = _case(B, T, Hq, Hkv, D, seed=T + D + 1)
    _backward_alone(q, kt, vt, dout, kc, vc, "B%d T%d Hq%d Hkv%d D%d" % (B, T, Hq, Hkv, D))


def test_forward_with_lse_is_prefill_bit_for_bit(cuda_lib):
    q, _, _, _, kc, vc = _case(2, 333, 6, 2, 128, seed=5)
    dq_, dkc, dvc = q.to(DEV), kc.to(DEV), vc.to(DEV)
    a = gqa.gqa_prefill(dq_, dkc, dvc)
    b, _ = gqa.gqa_prefill_lse(dq_, dkc, dvc)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_slots_past_t_untouched_and_deterministic(cuda_lib):
    q, _, _, dout, kc, vc = _case(1, 200, 4, 2, 64, seed=6, L=384)
    sentinel = torch.full((1, 2, 384, 64), 9.0, dtype=torch.bfloat16, device=DEV)
    _, _, (dq1, dk1, dv1) = _run(q, dout, kc, vc, dk=sentinel.clone(), dv=sentinel.clone())
    assert (dk1[:, :, 200:] == 9.0).all() and (dv1[:, :, 200:] == 9.0).all()
    _, _, (dq2, dk2, dv2) = _run(q, dout, kc, vc, dk=sentinel.clone(), dv=sentinel.clone())
    for a, b in ((dq1, dq2), (dk1, dk2), (dv1, dv2)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_back_to_back_calls_share_a_workspace(cuda_lib):
    """Five backward calls on one stream with no synchronisation between them,
    one workspace, a different output gradient each time and the results read
    only at the end: each call's three launches are programmatic dependents
    (the dQ launch starts while the dK/dV launch still runs, and waits for it
    before it ends), so a call must not overwrite the workspace's Delta while
    the call before still reads it, and each result must equal that of the same
    call run alone, bit for bit."""
    B, T, Hq, Hkv, D = 2, 700, 6, 2, 128
    q, _, _, _, kc, vc = _case(B, T, Hq, Hkv, D, seed=77)
    dq_, dkc, dvc = q.to(DEV), kc.to(DEV), vc.to(DEV)
    o, lse = gqa.gqa_prefill_lse(dq_, dkc, dvc)
    g = torch.Generator().manual_seed(78)
    douts = [torch.randn(B, T, Hq, D, generator=g).to(torch.bfloat16).to(DEV) for _ in range(5)]
    ws = torch.empty(gqa.gqa_backward_workspace_bytes(B, T, Hq), dtype=torch.uint8, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    chained = [gqa.gqa_attention_backward(dq_, dkc, dvc, o, d, lse, workspace=ws, status=st)
               for d in douts]
    torch.cuda.synchronize()
    assert st.item() == 0, "device status %#x" % st.item()
    for i, d in enumerate(douts):
        alone = gqa.gqa_attention_backward(dq_, dkc, dvc, o, d, lse)
        torch.cuda.synchronize()
        for a, b, name in zip(chained[i], alone, ("dq", "dk", "dv")):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16)), "call %d: %s differs" % (i, name)
