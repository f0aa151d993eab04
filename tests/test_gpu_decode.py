"""GPU parity: single-token decode against the KV cache (split-K kernel + merge).

The batched-decode workload at full size (B=64, 24/8 heads, D=128, cached
lengths U[256, 2048], QK-norm, NaN in every slot past each length), the
generation loops of the tiny and 512+100 workloads, and the edge cases: a
cache of one token, a full cache, MHA and MQA groupings, head_dim 96, and
invalid lengths; and the shapes that stress the split over 64-slot chunks: one
long sequence of 313 chunks per row, problems with fewer chunks than SMs, and
lengths on and around multiples of 64.
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


def _decode_step(q, k, v, kc, vc, pos, qk_norm, max_len, status=None):
    """rope(q) + append(k, v) at pos, then decode over pos + 1 keys (all on the GPU)."""
    new_len = torch.empty_like(pos)
    gqa.gqa_rope_append(q, k, v, kc, vc, pos0=pos, new_len=new_len, qk_norm=qk_norm,
                        status=status)
    return gqa.gqa_decode(q, kc, vc, new_len, max_len, status=status)


def test_batched_decode_full_size(cuda_lib):
    w = inputs.BY_NAME["batched_decode"]
    x = inputs.make_inputs(w)
    q, k, v = x["steps"][0]
    lens = x["lens"]
    dkc, dvc = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = _decode_step(q.to(DEV), k.to(DEV), v.to(DEV), dkc, dvc, lens.to(DEV), True,
                       int(lens.max()) + 1, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    want, _ = oracle.decode_step(bits(q), bits(k), bits(v), bits(x["k_cache"]),
                                 bits(x["v_cache"]), lens.numpy(), True)
    assert_close(out, want, "batched decode")


@pytest.mark.parametrize("name", ["tiny_gqa", "generation"])
def test_generation_loop(cuda_lib, name):
    """Prompt prefill, then every decode step, each against the oracle's own cache."""
    w = inputs.BY_NAME[name]
    x = inputs.make_inputs(w)
    B, T = w.B, w.T
    dkc, dvc = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
    dq = x["q"].to(DEV)
    gqa.gqa_rope_append(dq, x["k"].to(DEV), x["v"].to(DEV), dkc, dvc, qk_norm=w.qk_norm)
    # oracle cache from the oracle's own prefill
    _, k_rot, v64 = oracle.prefill(bits(x["q"]), bits(x["k"]), bits(x["v"]), w.qk_norm)
    kc = np.zeros((B, w.Hkv, w.Lmax, w.D))
    vc = np.zeros((B, w.Hkv, w.Lmax, w.D))
    kc[:, :, :T] = k_rot.transpose(0, 2, 1, 3)
    vc[:, :, :T] = v64.transpose(0, 2, 1, 3)
    pos = torch.full((B,), T, dtype=torch.int32, device=DEV)
    lens = np.full(B, T)
    worst = 0.0
    for s, (q, k, v) in enumerate(x["steps"]):
        out = _decode_step(q.to(DEV), k.to(DEV), v.to(DEV), dkc, dvc, pos, w.qk_norm, w.Lmax)
        want, knew = oracle.decode_step(bits(q), bits(k), bits(v), kc, vc, lens, w.qk_norm)
        worst = max(worst, assert_close(out, want, "%s step %d" % (name, s))[0])
        kc[:, :, T + s] = knew
        vc[:, :, T + s] = oracle.bf16_to_f64(bits(v))
        lens = lens + 1
        pos = pos + 1


def test_decode_graph_replays_the_eager_loop(cuda_lib):
    """The 512-token prompt + 100 generated tokens through DecodeGraph (the step
    captured in CUDA graphs): every step's output bit-identical to the eager
    calls (which test_generation_loop holds against the oracle), the same
    caches at the end, and the lengths advanced by one per step."""
    w = inputs.BY_NAME["generation"]
    x = inputs.make_inputs(w)
    B, T = w.B, w.T
    caches = []
    for _ in range(2):
        kc, vc = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
        gqa.gqa_rope_append(x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV), kc, vc,
                            qk_norm=w.qk_norm)
        caches.append((kc, vc))
    pos = torch.full((B,), T, dtype=torch.int32, device=DEV)
    dg = gqa.DecodeGraph(caches[1][0], caches[1][1], pos, w.Hq, qk_norm=w.qk_norm)
    for s, (q, k, v) in enumerate(x["steps"]):
        eager = _decode_step(q.to(DEV), k.to(DEV), v.to(DEV), caches[0][0], caches[0][1], pos,
                             w.qk_norm, w.Lmax)
        dg.q.copy_(q)
        dg.k.copy_(k)
        dg.v.copy_(v)
        got = dg.step()
        assert torch.equal(got.view(torch.int16), eager.view(torch.int16)), "step %d" % s
        pos = pos + 1
    torch.cuda.synchronize()
    assert dg.status.item() == 0
    assert torch.equal(dg.lens, pos)
    for a, b in zip(caches[0], caches[1]):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("Hq,Hkv,D", [(8, 8, 64), (8, 1, 64), (12, 4, 96), (16, 2, 128),
                                      (4, 4, 128), (6, 2, 96)])
def test_groupings_and_head_dims(cuda_lib, Hq, Hkv, D):
    B, L = 5, 512
    w = inputs.custom("dec", B=B, Hq=Hq, Hkv=Hkv, D=D, decode_steps=1, qk_norm=True,
                      cached_len_range=(1, 500), seed_index=Hq * 10 + Hkv + D)
    x = inputs.make_inputs(w, Lmax=L)
    q, k, v = x["steps"][0]
    lens = x["lens"].clone()
    lens[0] = 0            # only the new token will be visible
    lens[1] = L - 1        # the new token fills the last slot
    kc_cpu, vc_cpu = x["k_cache"].clone(), x["v_cache"].clone()
    kc_cpu[0] = float("nan")
    vc_cpu[0] = float("nan")
    g1 = torch.Generator().manual_seed(77)
    kc_cpu[1] = torch.randn(Hkv, L, D, generator=g1).to(torch.bfloat16)
    vc_cpu[1] = torch.randn(Hkv, L, D, generator=g1).to(torch.bfloat16)
    out = _decode_step(q.to(DEV), k.to(DEV), v.to(DEV), kc_cpu.to(DEV), vc_cpu.to(DEV),
                       lens.to(DEV), True, L)
    torch.cuda.synchronize()
    want, _ = oracle.decode_step(bits(q), bits(k), bits(v), bits(kc_cpu), bits(vc_cpu),
                                 lens.numpy(), True)
    assert_close(out, want, "decode Hq=%d Hkv=%d D=%d" % (Hq, Hkv, D))
    # one visible token: the output is that token's value
    g = Hq // Hkv
    for h in range(Hq):
        assert torch.equal(out[0, h].cpu().view(torch.int16), v[0, h // g].view(torch.int16))


def test_invalid_lengths_report_and_zero(cuda_lib):
    B, Hq, Hkv, D, L = 3, 4, 2, 64, 256
    g = torch.Generator().manual_seed(5)
    q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16).to(DEV)
    kc = torch.randn(B, Hkv, L, D, generator=g).to(torch.bfloat16).to(DEV)
    vc = torch.randn(B, Hkv, L, D, generator=g).to(torch.bfloat16).to(DEV)
    lens = torch.tensor([0, 100, 200], dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = gqa.gqa_decode(q, kc, vc, lens, 150, status=status)
    torch.cuda.synchronize()
    st = status.item()
    assert st & gqa.GQA_DEV_BAD_LEN and st & gqa.GQA_DEV_CAPACITY
    assert (out[0] == 0).all() and (out[2] == 0).all()
    # sequence 1 is valid: compare against the oracle on the cache as is
    keys = bits(kc[1:2].cpu())[:, :, :100].transpose(0, 2, 1, 3)
    vals = bits(vc[1:2].cpu())[:, :, :100].transpose(0, 2, 1, 3)
    want = oracle.attention(oracle.bf16_to_f64(bits(q[1:2].cpu()))[:, None],
                            oracle.bf16_to_f64(keys), oracle.bf16_to_f64(vals),
                            np.array([[99]]))[:, 0]
    assert_close(out[1:2], want, "valid sequence next to invalid ones")


def test_workspace_too_small_raises(cuda_lib):
    q = torch.zeros(1, 4, 64, dtype=torch.bfloat16, device=DEV)
    kc = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16, device=DEV)
    lens = torch.ones(1, dtype=torch.int32, device=DEV)
    ws = torch.empty(64, dtype=torch.uint8, device=DEV)
    with pytest.raises(gqa.GqaError):
        gqa.gqa_decode(q, kc, kc.clone(), lens, 100, workspace=ws)


def test_cached_decode_matches_longer_prefill_on_gpu(cuda_lib):
    """The pages' cached-vs-uncached check, both sides on the GPU path."""
    B, T0, steps, Hq, Hkv, D, L = 2, 200, 5, 8, 2, 128, 256
    g = torch.Generator().manual_seed(21)
    q = torch.randn(B, T0 + steps, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, T0 + steps, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, T0 + steps, Hkv, D, generator=g).to(torch.bfloat16)
    # uncached: one prefill over all T0 + steps tokens
    kc = torch.zeros(B, Hkv, L, D, dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    qa = q.to(DEV)
    gqa.gqa_rope_append(qa, k.to(DEV), v.to(DEV), kc, vc, qk_norm=True)
    full = gqa.gqa_prefill(qa, kc, vc)
    # cached: prefill T0, then one token at a time
    kc2 = torch.zeros_like(kc)
    vc2 = torch.zeros_like(kc)
    qb = q[:, :T0].contiguous().to(DEV)
    gqa.gqa_rope_append(qb, k[:, :T0].contiguous().to(DEV), v[:, :T0].contiguous().to(DEV),
                        kc2, vc2, qk_norm=True)
    pos = torch.full((B,), T0, dtype=torch.int32, device=DEV)
    for s in range(steps):
        t = T0 + s
        out = _decode_step(q[:, t].contiguous().to(DEV), k[:, t].contiguous().to(DEV),
                           v[:, t].contiguous().to(DEV), kc2, vc2, pos, True, L)
        d = (out.float() - full[:, t].float()).abs()
        assert d.max().item() <= 1e-2, (s, d.max().item())
        pos = pos + 1
    torch.cuda.synchronize()
    assert torch.equal(kc.view(torch.int16), kc2.view(torch.int16))


def test_workspace_reuse_and_garbage_contents(cuda_lib):
    """One workspace serves consecutive calls (same bits each time), whatever it
    held before (it is filled with garbage first)."""
    w = inputs.custom("dec", B=7, Hq=12, Hkv=4, D=128, decode_steps=1, qk_norm=False,
                      cached_len_range=(1, 900), seed_index=33)
    x = inputs.make_inputs(w)
    q = x["steps"][0][0].to(DEV)
    kc, vc = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
    lens = x["lens"].to(DEV)
    max_len = int(x["lens"].max())
    ws = gqa.decode_workspace(w.B, w.Hq, w.D, max_len, DEV)
    ws.random_(0, 256)
    outs = []
    for _ in range(3):
        outs.append(gqa.gqa_decode(q, kc, vc, lens, max_len, workspace=ws))
        torch.cuda.synchronize()
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    assert torch.equal(outs[0].view(torch.int16), outs[2].view(torch.int16))
    want = oracle.attention(oracle.bf16_to_f64(bits(x["steps"][0][0]))[:, None],
                            oracle.bf16_to_f64(bits(x["k_cache"])).transpose(0, 2, 1, 3),
                            oracle.bf16_to_f64(bits(x["v_cache"])).transpose(0, 2, 1, 3),
                            (x["lens"].numpy() - 1)[:, None].astype(np.int64))[:, 0]
    assert_close(outs[0], want, "decode with a reused workspace")


def _decode_vs_oracle(B, Hq, Hkv, D, L, lens_list, seed, label):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, Hkv, L, D, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hkv, L, D, generator=g).to(torch.bfloat16)
    lens = torch.tensor(lens_list, dtype=torch.int32)
    for b, n in enumerate(lens_list):          # NaN past every length
        kc[b, :, n:] = float("nan")
        vc[b, :, n:] = float("nan")
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = gqa.gqa_decode(q.to(DEV), kc.to(DEV), vc.to(DEV), lens.to(DEV), max(lens_list),
                         status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    want = oracle.attention(oracle.bf16_to_f64(bits(q))[:, None],
                            oracle.bf16_to_f64(bits(kc)).transpose(0, 2, 1, 3),
                            oracle.bf16_to_f64(bits(vc)).transpose(0, 2, 1, 3),
                            (lens.numpy() - 1)[:, None].astype(np.int64))[:, 0]
    assert_close(out, want, label)


def test_long_sequence_many_chunks(cuda_lib):
    # one sequence of 20000 slots, MQA with 8 query heads (4 subgroups of 2
    # heads): 313 chunks per subgroup for the merge to combine
    _decode_vs_oracle(1, 8, 1, 128, 20096, [20000], 91, "one long MQA sequence")


def test_fewer_chunks_than_sms(cuda_lib):
    # 2 sequences of 1 and 2 chunks, 2 KV heads each: 6 chunk CTAs in all
    _decode_vs_oracle(2, 4, 2, 64, 256, [30, 70], 92, "six chunks")


def test_lengths_around_unit_edges(cuda_lib):
    lens = [1, 63, 64, 65, 127, 128, 129, 191, 192, 640, 1, 2]
    _decode_vs_oracle(len(lens), 12, 4, 96, 640, lens, 93, "lengths around multiples of 64")


def test_resume_from_host_copies_continues_bit_identically(cuda_lib):
    """Checkpoint and resume of a generation (page "750美元从零训练3个LLM：一位开发者的
    实战复盘", sections "3. 难点不在训练循环，而在基础设施" -- resuming after an
    interruption -- and "5. 充分的冒烟测试与全程追踪" -- a checkpoint must load and
    resume).  The caller owns the whole decode state: the caches and the
    lengths.  Saved to host memory mid-generation, dropped from the device and
    restored into fresh device buffers, the session continues exactly as an
    uninterrupted one: every later output and the final caches bit for bit."""
    w = inputs.BY_NAME["generation"]                 # 512-token prompt, 16q/4kv, D=64
    x = inputs.make_inputs(w, decode_steps=24)
    B, T = w.B, w.T
    split = 9                                        # save after 9 generated tokens

    def start():
        kc, vc = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
        gqa.gqa_rope_append(x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV), kc, vc,
                            qk_norm=w.qk_norm)
        return kc, vc, torch.full((B,), T, dtype=torch.int32, device=DEV)

    def steps(kc, vc, pos, lo, hi):
        outs = []
        for q, k, v in x["steps"][lo:hi]:
            outs.append(_decode_step(q.to(DEV), k.to(DEV), v.to(DEV), kc, vc, pos, w.qk_norm,
                                     w.Lmax))
            pos = pos + 1
        return outs, pos

    kc, vc, pos = start()
    ref, pos = steps(kc, vc, pos, 0, len(x["steps"]))
    torch.cuda.synchronize()
    ref_k, ref_v = kc.cpu(), vc.cpu()

    kc, vc, pos = start()
    first, pos = steps(kc, vc, pos, 0, split)
    torch.cuda.synchronize()
    saved = (kc.cpu(), vc.cpu(), pos.cpu())          # the checkpoint: host copies
    del kc, vc, pos
    torch.cuda.empty_cache()
    kc, vc, pos = (t.to(DEV) for t in saved)         # restored into new device buffers
    rest, pos = steps(kc, vc, pos, split, len(x["steps"]))
    torch.cuda.synchronize()
    for s, (a, b) in enumerate(zip(ref, first + rest)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), "step %d" % s
    assert torch.equal(kc.cpu().view(torch.int16), ref_k.view(torch.int16))
    assert torch.equal(vc.cpu().view(torch.int16), ref_v.view(torch.int16))
    assert int(pos[0]) == T + len(x["steps"])
