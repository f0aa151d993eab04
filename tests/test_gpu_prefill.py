"""GPU parity: the prefill phase (QK-norm + RoPE + append, then the tcgen05 kernel).

Each case runs the whole phase on the GPU through the C ABI -- gqa_rope_append
on the prompt's q, k, v, then gqa_prefill -- and compares the output with the
float64 oracle's prefill on the same bf16 inputs, element by element, at the
sizes the oracle finishes in seconds (which still span several tiles and a
ragged tail) and at the 3.8B-style full size the benchmark times (every one of
its 50M outputs, a sequence at a time).  The bound is the bf16 floor of a
tensor-core pipeline plus its stated margin (ideal_pipeline.py), and mean
|d| <= 1e-3 against the exact result.
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


def _run_phase(x, w, out=None):
    dq, dk, dv = x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV)
    dkc, dvc = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gqa.gqa_rope_append(dq, dk, dv, dkc, dvc, qk_norm=w.qk_norm, max_pos0=0, status=status)
    o = gqa.gqa_prefill(dq, dkc, dvc, out=out, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, "device status %#x" % status.item()
    return o


@pytest.mark.parametrize("name", ["tiny_gqa", "mha_prefill", "generation"])
def test_named_workload_full_output(cuda_lib, name):
    w = inputs.BY_NAME[name]
    x = inputs.make_inputs(w, decode_steps=0)
    o = _run_phase(x, w)
    exact, ideal, W = prompt_refs(bits(x["q"]), bits(x["k"]), bits(x["v"]), w.qk_norm)
    assert_floor_close(o, exact, ideal, W, name)


def _sweep_shapes(n, seed):
    """n seeded small shapes (B <= 3, T <= 420, 1-6 query heads per KV head,
    D in {64, 96, 128}), for the pairing of (query tile, head) tiles into items:
    odd and even tile counts, single-tile items, T below one tile."""
    r = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        G = int(r.choice([1, 2, 3, 4, 6]))
        Hkv = int(r.integers(1, 4))
        out.append((int(r.integers(1, 4)), int(r.integers(1, 421)), G * Hkv, Hkv,
                    int(r.choice([64, 96, 128])), bool(r.integers(0, 2))))
    return out


@pytest.mark.parametrize("B,T,Hq,Hkv,D,qk", _sweep_shapes(10, 2026))
def test_seeded_shape_sweep(cuda_lib, B, T, Hq, Hkv, D, qk):
    w = inputs.custom("pf", B=B, Hq=Hq, Hkv=Hkv, D=D, T=T, qk_norm=qk, seed_index=3 * T + D)
    x = inputs.make_inputs(w)
    o = _run_phase(x, w)
    exact, ideal, W = prompt_refs(bits(x["q"]), bits(x["k"]), bits(x["v"]), qk)
    assert_floor_close(o, exact, ideal, W, "sweep B%d T%d Hq%d Hkv%d D%d" % (B, T, Hq, Hkv, D))


@pytest.mark.parametrize("B,T,Hq,Hkv,D,qk", [
    (2, 1, 4, 2, 64, False),          # a single token
    (1, 200, 6, 2, 128, True),        # ragged second tile
    (2, 300, 3, 3, 96, False),        # MHA, ragged pair
    (1, 385, 8, 1, 64, True),         # MQA, three pairs, ragged
    (1, 256, 4, 2, 128, False),       # T == Lmax exactly
    (3, 129, 6, 3, 96, True),         # one row into the second tile
    (2, 300, 6, 2, 128, True),        # 3 heads per KV head, 3 tiles: items of one tile
                                      # and two heads, of two tiles, and one single tile
])
def test_shapes_and_tails(cuda_lib, B, T, Hq, Hkv, D, qk):
    w = inputs.custom("pf", B=B, Hq=Hq, Hkv=Hkv, D=D, T=T, qk_norm=qk, seed_index=T + D)
    x = inputs.make_inputs(w)
    o = _run_phase(x, w)
    exact, ideal, W = prompt_refs(bits(x["q"]), bits(x["k"]), bits(x["v"]), qk)
    assert_floor_close(o, exact, ideal, W, "B%d T%d Hq%d Hkv%d D%d" % (B, T, Hq, Hkv, D))


def test_output_rows_beyond_t_untouched(cuda_lib):
    w = inputs.custom("pf", B=1, Hq=2, Hkv=1, D=64, T=70)
    x = inputs.make_inputs(w)
    big = torch.full((1, 128, 2, 64), 3.0, dtype=torch.bfloat16, device=DEV)
    out = big[:, :70]     # a view: rows 70.. of `big` must keep their value
    o = _run_phase(x, w, out=out.contiguous())
    assert o.shape == (1, 70, 2, 64)
    assert (big[:, 70:] == 3.0).all()


def test_prefill_3p8b_full_size_every_element(cuda_lib):
    """B=8, T=2048, Hq=24, Hkv=8, D=128, QK-norm: the launch the benchmark times,
    every output element against the oracle (one sequence at a time: the
    attention of a sequence depends on its own tokens only)."""
    w = inputs.BY_NAME["prefill_3p8b"]
    x = inputs.make_inputs(w)
    o = _run_phase(x, w).cpu()
    worst, floor_max, means = 0.0, 0.0, []
    for b in range(w.B):
        sl = slice(b, b + 1)
        exact, ideal, W = prompt_refs(bits(x["q"][sl]), bits(x["k"][sl]), bits(x["v"][sl]), True)
        d, f, m = assert_floor_close(o[sl], exact, ideal, W, "3.8B prefill, sequence %d" % b)
        worst, floor_max = max(worst, d), max(floor_max, f)
        means.append(m)
    assert np.mean(means) <= 1e-3
    print("3.8B prefill: max|d| %.4g (floor %.4g), mean|d| %.3g over %d elements"
          % (worst, floor_max, np.mean(means), o.numel()))


def test_prefill_deterministic(cuda_lib):
    w = inputs.custom("pf", B=2, Hq=6, Hkv=2, D=128, T=700, qk_norm=True)
    x = inputs.make_inputs(w)
    a = _run_phase(x, w)
    b = _run_phase(x, w)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_item_counter_slots_recycle_and_run_concurrently(cuda_lib):
    """Items are taken from a launch-wide counter (one of 256 slots, round robin,
    reset by the launch's last CTA): 300 launches in a row -- every slot used
    more than once -- and two launches in flight at once on two streams all give
    the same output bits."""
    w = inputs.BY_NAME["prefill_3p8b"]
    x = inputs.make_inputs(w)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    dq, dk, dv = x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV)
    dkc, dvc = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
    gqa.gqa_rope_append(dq, dk, dv, dkc, dvc, qk_norm=True, max_pos0=0, status=st)
    ref = gqa.gqa_prefill(dq, dkc, dvc, status=st)
    out = torch.empty_like(ref)
    for _ in range(300):
        gqa.gqa_prefill(dq, dkc, dvc, out=out, status=st)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    o1, o2 = torch.empty_like(ref), torch.empty_like(ref)
    torch.cuda.synchronize()
    for _ in range(5):
        with torch.cuda.stream(s1):
            gqa.gqa_prefill(dq, dkc, dvc, out=o1, status=st, stream=s1)
        with torch.cuda.stream(s2):
            gqa.gqa_prefill(dq, dkc, dvc, out=o2, status=st, stream=s2)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(o1.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(o2.view(torch.int16), ref.view(torch.int16))
