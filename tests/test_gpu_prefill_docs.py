"""GPU parity: document-masked prefill (gqa_doc_start + gqa_prefill_docs).

Packed documents: query t sees only the earlier keys of its own document.  The
GPU path (QK-norm + RoPE + append, document starts from the ids, the masked
tcgen05 prefill) against the float64 oracle's prefill with the same document
ids, at sizes the oracle finishes in seconds and on every output element of
the 3.8B-style packed workload, held to the bf16 floor of a tensor-core
pipeline plus its stated margin (ideal_pipeline.py) and mean |d| <= 1e-3; the
start helper exactly; one document equal to gqa_prefill bit for bit;
decreasing ids reported; the start kernel and the prefill back to back.
"""
import numpy as np
import pytest
import torch

import oracle
import rope_gqa_kv_b200 as gqa
from rope_gqa_kv_b200 import inputs

from helpers import assert_floor_close, bits, prompt_refs

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
    (2, 300, 6, 2, 128, 90.0),      # 3 heads per KV head over 3 tiles (a single-tile item)
])
def test_docs_vs_oracle(cuda_lib, B, T, Hq, Hkv, D, mean):
    w = inputs.custom("doc", B=B, Hq=Hq, Hkv=Hkv, D=D, T=T, qk_norm=True, seed_index=T + D)
    x = inputs.make_inputs(w)
    ids = inputs.packed_doc_ids(B, T, mean, seed=T + Hq)
    ids[0, 5] = ids[0, 4] + 1          # a one-token document
    ids[0, 6:] += 2
    o = _run_docs(x, w, ids)
    exact, ideal, W = prompt_refs(bits(x["q"]), bits(x["k"]), bits(x["v"]), True,
                                  doc_id=ids.numpy())
    assert_floor_close(o, exact, ideal, W, "documents B%d T%d D%d mean %g" % (B, T, D, mean))


def _sweep_shapes(n, seed):
    """n seeded small shapes with a mean document length each (B <= 3, T <= 420,
    1-6 query heads per KV head, D in {64, 96, 128})."""
    r = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        G = int(r.choice([1, 2, 3, 4, 6]))
        Hkv = int(r.integers(1, 4))
        out.append((int(r.integers(1, 4)), int(r.integers(1, 421)), G * Hkv, Hkv,
                    int(r.choice([64, 96, 128])), float(r.choice([20.0, 100.0, 400.0]))))
    return out


@pytest.mark.parametrize("B,T,Hq,Hkv,D,mean", _sweep_shapes(6, 2027))
def test_docs_seeded_shape_sweep(cuda_lib, B, T, Hq, Hkv, D, mean):
    w = inputs.custom("doc", B=B, Hq=Hq, Hkv=Hkv, D=D, T=T, qk_norm=True, seed_index=5 * T + D)
    x = inputs.make_inputs(w)
    ids = inputs.packed_doc_ids(B, T, mean, seed=7 * T + Hq)
    o = _run_docs(x, w, ids)
    exact, ideal, W = prompt_refs(bits(x["q"]), bits(x["k"]), bits(x["v"]), True,
                                  doc_id=ids.numpy())
    assert_floor_close(o, exact, ideal, W, "documents sweep B%d T%d Hq%d Hkv%d D%d" % (B, T, Hq, Hkv, D))


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


def test_doc_start_then_prefill_back_to_back(cuda_lib):
    """gqa_doc_start followed at once by gqa_prefill_docs on the same stream, with
    no synchronisation, five times with different document ids written into the
    same start buffer: the prefill is a programmatic dependent of the start
    kernel (which lets it begin its prologue early), so every role of the
    prefill must wait for the starts of its own iteration, never read the
    previous iteration's."""
    B, T, Hq, Hkv, D = 2, 700, 6, 2, 128
    w = inputs.custom("doc", B=B, Hq=Hq, Hkv=Hkv, D=D, T=T, qk_norm=True, seed_index=77)
    x = inputs.make_inputs(w)
    dq, dk, dv = x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV)
    kc, vc = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gqa.gqa_rope_append(dq, dk, dv, kc, vc, qk_norm=True, status=status)
    means = (30.0, 700.0, 90.0, 1e6, 15.0)       # short, long, one per row, ...
    ids_dev = [inputs.packed_doc_ids(B, T, m, seed=300 + i).to(DEV) for i, m in enumerate(means)]
    starts = torch.full((B, T), -1, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    outs = []
    for ids in ids_dev:
        gqa.gqa_doc_start(ids, out=starts, status=status)
        outs.append(gqa.gqa_prefill_docs(dq, kc, vc, starts, status=status))
    torch.cuda.synchronize()
    assert status.item() == 0, "device status %#x" % status.item()
    for i, (ids, o) in enumerate(zip(ids_dev, outs)):
        exact, ideal, W = prompt_refs(bits(x["q"]), bits(x["k"]), bits(x["v"]), True,
                                      doc_id=ids.cpu().numpy())
        assert_floor_close(o, exact, ideal, W, "back-to-back iteration %d" % i)


def test_packed_docs_3p8b_size_every_element(cuda_lib):
    """8 x 2048 tokens of packed documents (mean 512 tokens), 24/8 heads, D=128,
    QK-norm: the launch the benchmark times for document masking, every output
    element against the oracle, one sequence at a time."""
    w = inputs.BY_NAME["prefill_3p8b"]
    x = inputs.make_inputs(w)
    ids = inputs.packed_doc_ids(w.B, w.T, 512.0, seed=2048)
    o = _run_docs(x, w, ids).cpu()
    worst, means = 0.0, []
    for b in range(w.B):
        sl = slice(b, b + 1)
        exact, ideal, W = prompt_refs(bits(x["q"][sl]), bits(x["k"][sl]), bits(x["v"][sl]), True,
                                      doc_id=ids[sl].numpy())
        d, _, m = assert_floor_close(o[sl], exact, ideal, W, "packed documents, sequence %d" % b)
        worst = max(worst, d)
        means.append(m)
    assert np.mean(means) <= 1e-3
    print("packed documents: max|d| %.4g, mean|d| %.3g over %d elements"
          % (worst, np.mean(means), o.numel()))
