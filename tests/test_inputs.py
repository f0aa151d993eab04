"""Host-side checks of the seeded workload generator (no GPU, no attention math)."""
import pytest
import torch

from rope_gqa_kv_b200 import inputs


def test_named_workloads_and_capacities():
    got = {w.name: (w.B, w.Hq, w.Hkv, w.D, w.T, w.decode_steps, w.qk_norm, w.Lmax)
           for w in inputs.WORKLOADS}
    assert got == {
        "tiny_gqa": (1, 4, 2, 64, 128, 16, False, 256),
        "mha_prefill": (8, 8, 8, 96, 1024, 0, False, 1024),
        "generation": (1, 16, 4, 64, 512, 100, False, 640),
        "prefill_3p8b": (8, 24, 8, 128, 2048, 0, True, 2048),
        "batched_decode": (64, 24, 8, 128, 0, 1, True, 2176),
        "chunked_prefill_3p8b": (8, 24, 8, 128, 1024, 0, True, 2560),
    }
    assert [w.seed for w in inputs.WORKLOADS] == [1000, 1001, 1002, 1003, 1004, 1005]


def test_config_assertions():
    with pytest.raises(AssertionError):
        inputs.custom("bad", B=1, Hq=6, Hkv=4, D=64, T=8)
    with pytest.raises(AssertionError):
        inputs.custom("bad", B=1, Hq=4, Hkv=4, D=80, T=8)


def test_generation_is_deterministic_and_poisoned():
    w = inputs.custom("c", B=3, Hq=4, Hkv=2, D=64, decode_steps=2, cached_len_range=(5, 40))
    a = inputs.make_inputs(w)
    b = inputs.make_inputs(w)
    assert torch.equal(a["lens"], b["lens"])
    assert torch.equal(a["k_cache"].view(torch.int16), b["k_cache"].view(torch.int16))
    assert a["k_cache"].shape == (3, 2, 128, 64)
    lens = a["lens"].tolist()
    assert all(5 <= n <= 40 for n in lens)
    nan_bits = a["k_cache"].view(torch.int16) == inputs.BF16_QNAN_BITS
    for bi, n in enumerate(lens):
        assert not nan_bits[bi, :, :n].any()
        assert nan_bits[bi, :, n:].all()
        assert (a["v_cache"].view(torch.int16)[bi, :, n:] == inputs.BF16_QNAN_BITS).all()
    assert len(a["steps"]) == 2 and a["steps"][0][0].shape == (3, 4, 64)
    assert a["q"] is None


def test_prefill_workload_cache_starts_empty():
    w = inputs.custom("p", B=2, Hq=4, Hkv=2, D=96, T=70)
    a = inputs.make_inputs(w)
    assert a["q"].shape == (2, 70, 4, 96) and a["q"].dtype == torch.bfloat16
    assert (a["k_cache"].view(torch.int16) == inputs.BF16_QNAN_BITS).all()
    assert a["k_cache"].shape == (2, 2, 128, 96)


def test_chunk_workload_has_prefix_and_new_tokens():
    w = inputs.custom("k", B=3, Hq=4, Hkv=2, D=64, T=50, cached_len_range=(10, 100))
    a = inputs.make_inputs(w)
    assert w.Lmax == 256                    # 100 cached + 50 new, rounded up to 128
    assert a["q"].shape == (3, 50, 4, 64)
    for bi, n in enumerate(a["lens"].tolist()):
        assert 10 <= n <= 100
        assert not torch.isnan(a["k_cache"][bi, :, :n].float()).any()
        assert torch.isnan(a["k_cache"][bi, :, n:].float()).all()
