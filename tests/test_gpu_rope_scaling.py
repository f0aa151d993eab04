"""GPU parity: the RoPE context-extension variants (linear interpolation,
NTK-aware, YaRN) in gqa_rope_apply and the fused append, against the float64
oracle: rotated q and cached K within one bf16 ulp of the exact value, V bit for
bit, and one end-to-end prefill past the trained length with YaRN."""
import numpy as np
import pytest
import torch

import oracle
import rope_gqa_kv_b200 as gqa
from rope_gqa_kv_b200 import inputs

from helpers import assert_floor_close, assert_within_one_ulp, bits, prompt_refs

pytestmark = pytest.mark.gpu
DEV = "cuda"

VARIANTS = {
    "linear4": ("linear", 4.0, 0),
    "ntk8": ("ntk", 8.0, 0),
    "yarn16": ("yarn", 16.0, 4096),
    "yarn1": ("yarn", 1.0, 2048),
}


def _pair(name):
    kind, s, L = VARIANTS[name]
    return gqa.RopeScaling(kind, s, original_max_pos=L), oracle.RopeScaling(kind, s, original_max_pos=L)


@pytest.mark.parametrize("name", sorted(VARIANTS))
@pytest.mark.parametrize("D", [64, 96, 128])
def test_scaled_rope_apply(cuda_lib, name, D):
    g = torch.Generator().manual_seed(D + len(name))
    B, T, H = 2, 150, 6
    q = torch.randn(B, T, H, D, generator=g).to(torch.bfloat16)
    pos0 = torch.tensor([0, 60000], dtype=torch.int32)       # far past any trained length
    dq = q.to(DEV)
    sg, so = _pair(name)
    gqa.gqa_rope_apply(dq, pos0=pos0.to(DEV), qk_norm=True, scaling=sg)
    torch.cuda.synchronize()
    want = oracle.rope_apply(bits(q), pos0.numpy(), True, scaling=so)
    assert_within_one_ulp(dq, want, "q, %s, D=%d" % (name, D))


@pytest.mark.parametrize("name", ["ntk8", "yarn16"])
def test_scaled_rope_append(cuda_lib, name):
    g = torch.Generator().manual_seed(31)
    B, T, Hq, Hkv, D, L = 2, 40, 8, 2, 128, 8192
    q = torch.randn(B, T, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, T, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, T, Hkv, D, generator=g).to(torch.bfloat16)
    pos0 = torch.tensor([5000, 8100], dtype=torch.int32)
    kc = torch.zeros(B, Hkv, L, D, dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    dq = q.to(DEV)
    sg, so = _pair(name)
    gqa.gqa_rope_append(dq, k.to(DEV), v.to(DEV), kc, vc, pos0=pos0.to(DEV),
                        max_pos0=int(pos0.max()), qk_norm=True, scaling=sg)
    torch.cuda.synchronize()
    assert_within_one_ulp(dq, oracle.rope_apply(bits(q), pos0.numpy(), True, scaling=so), "q")
    want_k = oracle.rope_apply(bits(k), pos0.numpy(), True, scaling=so)
    for b in range(B):
        p = int(pos0[b])
        assert_within_one_ulp(kc[b, :, p:p + T].transpose(0, 1), want_k[b], "k_cache[%d]" % b)
        assert torch.equal(vc[b, :, p:p + T].transpose(0, 1).cpu().view(torch.int16),
                           v[b].view(torch.int16))


def test_yarn_prefill_end_to_end(cuda_lib):
    """A 700-token prompt with YaRN (s = 4 over a 256-token trained length): the
    whole prefill phase against the oracle's prefill with the same variant."""
    w = inputs.custom("pf", B=2, Hq=8, Hkv=2, D=128, T=700, qk_norm=True, seed_index=81)
    x = inputs.make_inputs(w)
    sg = gqa.RopeScaling("yarn", 4.0, original_max_pos=256)
    so = oracle.RopeScaling("yarn", 4.0, original_max_pos=256)
    dq, dk, dv = x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV)
    kc, vc = x["k_cache"].to(DEV), x["v_cache"].to(DEV)
    gqa.gqa_rope_append(dq, dk, dv, kc, vc, qk_norm=True, scaling=sg)
    o = gqa.gqa_prefill(dq, kc, vc)
    torch.cuda.synchronize()
    exact, ideal, W = prompt_refs(bits(x["q"]), bits(x["k"]), bits(x["v"]), True, scaling=so)
    assert_floor_close(o, exact, ideal, W, "YaRN prefill")
