"""GPU parity: document-masked prefill (gqa_doc_start + gqa_prefill_docs).

Packed documents: query t sees only the earlier keys of its own document.  The
GPU path (QK-norm + RoPE + append, document starts from the ids, the masked
tcgen05 prefill) against the float64 oracle's prefill with the same document
ids, at sizes the oracle finishes in seconds and on sampled rows of the
3.8B-style packed workload; the start helper exactly; one document equal to
gqa_prefill bit for bit; decreasing ids reported.
"""
import numpy as np
import pytest
import torch

import oracle
import rope_gqa_kv_b200 as gqa
from rope_gqa_kv_b200 import inputs

from helpers import assert_close, bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run_docs(x, w, doc_id):
    dq, dk, dv = x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV)
    kc, vc = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gqa.gqa_rope_append(dq, dk, dv, kc, vc, qk_norm=w.qk_norm, status=status)
    starts = gqa.gqa_doc_start(doc_id.to(DEV), status=status)
    o = gqa.gqa_prefill_docs(dq, kc, vc, starts, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, "device status %#x" % status.item()
    return o


def _starts_np(ids):
    ids = np.asarray(ids)
    out = np.zeros_like(ids)
    for b in range(ids.shape[0]):
        for t in range(ids.shape[1]):
            out[b, t] = t if t == 0 or ids[b, t] != ids[b, t - 1] else out[b, t - 1]
    return out


def test_doc_start_helper_exact(cuda_lib):
    ids = inputs.packed_doc_ids(3, 1000, 40.0, seed=90)
    got = gqa.gqa_doc_start(ids.to(DEV)).cpu().numpy()
    np.testing.assert_array_equal(got, _starts_np(ids.numpy()))


def test_decreasing_ids_are_reported(cuda_lib):
    ids = torch.tensor([[0, 0, 1, 1, 0, 2]], dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gqa.gqa_doc_start(ids, status=status)
    torch.cuda.synchronize()
    assert status.item() & gqa.GQA_DEV_BAD_LEN


@pytest.mark.parametrize("B,T,Hq,Hkv,D,mean", [
    (2, 700, 6, 2, 128, 60.0),      # many short documents, several per tile
    (2, 600, 8, 8, 96, 250.0),      # MHA, documents spanning tiles
    (3, 385, 4, 1, 64, 1000.0),     # MQA, mostly one document per row
])
def test_docs_vs_oracle(cuda_lib, B, T, Hq, Hkv, D, mean):
    w = inputs.custom("doc", B=B, Hq=Hq, Hkv=Hkv, D=D, T=T, qk_norm=True, seed_index=T + D)
    x = inputs.make_inputs(w)
    ids = inputs.packed_doc_ids(B, T, mean, seed=T + Hq)
    ids[0, 5] = ids[0, 4] + 1          # a one-token document
    ids[0, 6:] += 2
    o = _run_docs(x, w, ids)
    want, _, _ = oracle.prefill(bits(x["q"]), bits(x["k"]), bits(x["v"]), True,
                                doc_id=ids.numpy())
    assert_close(o, want, "documents B%d T%d D%d mean %g" % (B, T, D, mean))


def test_one_document_is_prefill_bit_for_bit(cuda_lib):
    w = inputs.custom("doc", B=2, Hq=6, Hkv=2, D=128, T=500, qk_norm=True, seed_index=91)
    x = inputs.make_inputs(w)
    o = _run_docs(x, w, torch.zeros(2, 500, dtype=torch.int32))
    dq, dk, dv = x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV)
    kc, vc = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
    gqa.gqa_rope_append(dq, dk, dv, kc, vc, qk_norm=True)
    ref = gqa.gqa_prefill(dq, kc, vc)
    torch.cuda.synchronize()
    assert torch.equal(o.view(torch.int16), ref.view(torch.int16))


def test_packed_docs_3p8b_size_sampled(cuda_lib):
    """8 x 2048 tokens of packed documents (mean 512 tokens), 24/8 heads, D=128,
    QK-norm: the launch the benchmark times for document masking."""
    w = inputs.BY_NAME["prefill_3p8b"]
    x = inputs.make_inputs(w)
    ids = inputs.packed_doc_ids(w.B, w.T, 512.0, seed=2048)
    o = _run_docs(x, w, ids)
    rng = np.random.default_rng(2)
    rows = rng.integers(0, w.B * w.T * w.Hq, size=400)
    starts = _starts_np(ids.numpy())
    # rows at document starts and ends, where the mask changes
    for b in (0, 5):
        for t in np.flatnonzero(np.diff(starts[b]) != 0)[:20]:
            for tt in (t, t + 1):
                rows = np.append(rows, (b * w.T + tt) * w.Hq + 7)
    rows = np.unique(rows).astype(np.int64)
    want, _, _ = oracle.prefill(bits(x["q"]), bits(x["k"]), bits(x["v"]), True, rows=rows,
                                doc_id=ids.numpy())
    got = o.reshape(-1, w.D)[torch.as_tensor(rows, device=DEV)]
    assert_close(got, want.reshape(-1, w.D)[rows], "packed documents (%d rows)" % len(rows))
    assert torch.isfinite(o.float()).all()
