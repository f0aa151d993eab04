"""Pins for the float64 oracle: what the pages and the mathematics fix.

None of these tests retypes the oracle's formulas.  Each checks the oracle
against something independent of it:
* hand-worked closed forms (tests/golden/hand_worked.json);
* library routines for special cases (torch float64 scaled_dot_product_attention,
  rms_norm, bfloat16 widening);
* invariants the pages state: RoPE scores depend only on m - n, rotation keeps
  the norm, softmax rows are a probability vector, GQA with Hkv = Hq is MHA and
  equals MHA on repeat_interleave'd K/V, cached decode equals full recomputation;
* the complex-number form of RoPE (each pair is a complex number multiplied by
  exp(i p theta)), a derivation different from the oracle's pairwise rotation.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")
MATH_NS = {"cos": math.cos, "sin": math.sin, "exp": math.exp, "sqrt": math.sqrt}


def _bits(x):
    """Float values (exact in bf16) -> uint16 bf16 bit patterns."""
    t = torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _eval(e):
    return np.vectorize(lambda s: float(eval(s, {"__builtins__": {}}, MATH_NS)))(np.asarray(e))


def _rand_bits(rng, *shape):
    return _bits(rng.standard_normal(shape).astype(np.float32))


# ---------------------------------------------------------------------------
# hand-worked closed forms
# ---------------------------------------------------------------------------
def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_hand_worked(case):
    want = _eval(case["expect"])
    op = case["op"]
    if op == "rope":
        x = np.asarray(case["x"], dtype=np.float64)
        got = oracle.rope(x, np.asarray(case["pos"]))
    elif op == "rmsnorm":
        got = oracle.rmsnorm(np.asarray(case["x"], dtype=np.float64), case["eps"])
    elif op == "prefill":
        got, _, _ = oracle.prefill(_bits(case["q"]), _bits(case["k"]), _bits(case["v"]),
                                   case["qk_norm"])
    elif op == "decode":
        got, _ = oracle.decode_step(_bits(case["q"]), _bits(case["k"]), _bits(case["v"]),
                                    _bits(case["k_cache"]), _bits(case["v_cache"]),
                                    case["lens"], case["qk_norm"])
    else:
        raise AssertionError(op)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# bf16 widening and RMSNorm against library routines
# ---------------------------------------------------------------------------
def test_bf16_widening_matches_torch():
    rng = np.random.default_rng(1)
    raw = rng.integers(0, 1 << 16, size=4096, dtype=np.uint16)
    raw = raw[~np.isnan(torch.tensor(raw.view(np.int16)).view(torch.bfloat16).float().numpy())]
    want = torch.tensor(raw.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.bf16_to_f64(raw), want)


@pytest.mark.parametrize("D", [4, 64, 96, 128])
def test_rmsnorm_matches_library(D):
    rng = np.random.default_rng(D)
    x = rng.standard_normal((37, D)) * rng.uniform(0.01, 10, size=(37, 1))
    want = F.rms_norm(torch.tensor(x), (D,), eps=1e-6).numpy()
    np.testing.assert_allclose(oracle.rmsnorm(x, 1e-6), want, rtol=1e-13, atol=1e-14)


def test_rmsnorm_output_mean_square():
    # mean(y^2) = ms / (ms + eps) exactly, ms = mean(x^2)
    rng = np.random.default_rng(2)
    x = rng.standard_normal((16, 128)) * 1e-3
    eps = 1e-6
    y = oracle.rmsnorm(x, eps)
    ms = (x ** 2).mean(-1)
    np.testing.assert_allclose((y ** 2).mean(-1), ms / (ms + eps), rtol=1e-12)


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------
def _rope_complex(x, pos, base=10000.0, interleaved=False):
    """RoPE as complex multiplication: pair i is z_i = x_a + i x_b, z_i *= e^{i p th_i}."""
    D = x.shape[-1]
    half = D // 2
    if interleaved:
        z = x[..., 0::2] + 1j * x[..., 1::2]
    else:
        z = x[..., :half] + 1j * x[..., half:]
    th = base ** (-np.arange(0, D, 2, dtype=np.float64) / D)
    z = z * np.exp(1j * np.asarray(pos, dtype=np.float64)[..., None, None] * th)
    out = np.empty_like(x)
    if interleaved:
        out[..., 0::2], out[..., 1::2] = z.real, z.imag
    else:
        out[..., :half], out[..., half:] = z.real, z.imag
    return out


@pytest.mark.parametrize("interleaved", [False, True])
@pytest.mark.parametrize("D", [2, 8, 64, 96, 128])
def test_rope_equals_complex_rotation(D, interleaved):
    rng = np.random.default_rng(D)
    x = rng.standard_normal((50, 3, D))
    pos = rng.integers(0, 5000, size=50)
    got = oracle.rope(x, pos, interleaved=interleaved)
    np.testing.assert_allclose(got, _rope_complex(x, pos, interleaved=interleaved),
                               rtol=0, atol=1e-11)


def test_rope_position_zero_is_identity_and_keeps_norm():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((20, 4, 128))
    np.testing.assert_array_equal(oracle.rope(x, np.zeros(20, dtype=np.int64)), x)
    y = oracle.rope(x, rng.integers(0, 4096, size=20))
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1),
                               rtol=1e-13)


@pytest.mark.parametrize("D", [64, 128])
def test_rope_scores_depend_on_distance_only(D):
    # q_m . k_n is unchanged when both positions shift by the same s.
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 1, D))
    k = rng.standard_normal((1, 1, D))
    for m, n, s in [(5, 3, 100), (0, 0, 777), (2047, 1, 9), (10, 400, 1234)]:
        a = (oracle.rope(q, [m]) * oracle.rope(k, [n])).sum()
        b = (oracle.rope(q, [m + s]) * oracle.rope(k, [n + s])).sum()
        assert abs(a - b) < 1e-10 * max(1.0, abs(a))
    # ... and it does depend on the distance
    a = (oracle.rope(q, [5]) * oracle.rope(k, [3])).sum()
    c = (oracle.rope(q, [6]) * oracle.rope(k, [3])).sum()
    assert abs(a - c) > 1e-6


def test_norm_and_rope_commute():
    # Unit-gain RMSNorm scales the whole vector; rotation keeps its norm.
    rng = np.random.default_rng(5)
    x = rng.standard_normal((30, 2, 128))
    pos = rng.integers(0, 3000, size=30)
    a = oracle.rope(oracle.rmsnorm(x, 1e-6), pos)
    b = oracle.rmsnorm(oracle.rope(x, pos), 1e-6)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------
# attention core: library special case, softmax, GQA reductions
# ---------------------------------------------------------------------------
def _sdpa(q, k, v, causal=True, scale=None):
    """torch float64 SDPA on [B, T, H, D] arrays (K/V heads repeated per group)."""
    qt = torch.tensor(q).transpose(1, 2)
    kt = torch.tensor(k).transpose(1, 2)
    vt = torch.tensor(v).transpose(1, 2)
    g = qt.shape[1] // kt.shape[1]
    kt = kt.repeat_interleave(g, dim=1)
    vt = vt.repeat_interleave(g, dim=1)
    o = F.scaled_dot_product_attention(qt, kt, vt, is_causal=causal, scale=scale)
    return o.transpose(1, 2).numpy()


@pytest.mark.parametrize("B,T,Hq,Hkv,D", [(2, 37, 4, 2, 64), (1, 130, 8, 8, 96),
                                          (2, 19, 6, 1, 32), (1, 64, 24, 8, 128)])
def test_attention_core_matches_library_sdpa(B, T, Hq, Hkv, D):
    rng = np.random.default_rng(B * T + Hq)
    q = rng.standard_normal((B, T, Hq, D))
    k = rng.standard_normal((B, T, Hkv, D))
    v = rng.standard_normal((B, T, Hkv, D))
    pos = oracle.positions(0, B, T)
    got = oracle.attention(q, k, v, pos)
    np.testing.assert_allclose(got, _sdpa(q, k, v), rtol=0, atol=1e-12)


def test_attention_probabilities_form_a_distribution():
    # With v_u = e_u (one-hot), output row t is the probability vector itself.
    rng = np.random.default_rng(6)
    T, D = 24, 32
    q = rng.standard_normal((1, T, 1, D)) * 3
    k = rng.standard_normal((1, T, 1, D)) * 3
    v = np.eye(D)[:T].reshape(1, T, 1, D)
    p = oracle.attention(q, k, v, oracle.positions(0, 1, T))[0, :, 0, :]
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert (p >= 0).all()
    # causal: row t puts no weight on keys after t
    for t in range(T):
        assert np.all(p[t, t + 1:] == 0)


def test_first_row_returns_first_value_and_equal_keys_average():
    rng = np.random.default_rng(7)
    B, T, H, D = 2, 9, 3, 16
    q = rng.standard_normal((B, T, H, D))
    k = np.broadcast_to(rng.standard_normal((B, 1, H, D)), (B, T, H, D)).copy()
    v = rng.standard_normal((B, T, H, D))
    o = oracle.attention(q, k, v, oracle.positions(0, B, T))
    np.testing.assert_array_equal(o[:, 0], v[:, 0])
    for t in range(T):
        np.testing.assert_allclose(o[:, t], v[:, :t + 1].mean(1), rtol=0, atol=1e-13)


def test_gqa_reductions():
    rng = np.random.default_rng(8)
    B, T, D = 2, 33, 64
    pos = oracle.positions(0, B, T)
    # GQA equals MHA on K/V repeated per group (query head h -> K/V head h // g)
    q = rng.standard_normal((B, T, 6, D))
    k = rng.standard_normal((B, T, 2, D))
    v = rng.standard_normal((B, T, 2, D))
    got = oracle.attention(q, k, v, pos)
    mha = oracle.attention(q, np.repeat(k, 3, axis=2), np.repeat(v, 3, axis=2), pos)
    np.testing.assert_allclose(got, mha, rtol=0, atol=1e-14)
    # Hkv = Hq is MHA: each head alone equals single-head attention
    k6 = rng.standard_normal((B, T, 6, D))
    v6 = rng.standard_normal((B, T, 6, D))
    full = oracle.attention(q, k6, v6, pos)
    for h in range(6):
        one = oracle.attention(q[:, :, h:h + 1], k6[:, :, h:h + 1], v6[:, :, h:h + 1], pos)
        np.testing.assert_array_equal(full[:, :, h:h + 1], one)
    # Hkv = 1 is MQA: every query head reads the same K/V
    k1, v1 = k6[:, :, :1], v6[:, :, :1]
    mqa = oracle.attention(q, k1, v1, pos)
    for h in range(6):
        one = oracle.attention(q[:, :, h:h + 1], k1, v1, pos)
        np.testing.assert_array_equal(mqa[:, :, h:h + 1], one)


def test_row_subset_matches_full():
    rng = np.random.default_rng(9)
    B, T, Hq, Hkv, D = 2, 50, 4, 2, 64
    q = rng.standard_normal((B, T, Hq, D))
    k = rng.standard_normal((B, T, Hkv, D))
    v = rng.standard_normal((B, T, Hkv, D))
    pos = oracle.positions(0, B, T)
    full = oracle.attention(q, k, v, pos)
    rows = np.array([0, 7, 199, 399])
    part = oracle.attention(q, k, v, pos, rows=rows)
    flat_f = full.reshape(-1, D)
    flat_p = part.reshape(-1, D)
    np.testing.assert_array_equal(flat_p[rows], flat_f[rows])
    assert np.isnan(flat_p[1]).all()


def test_hq_not_multiple_of_hkv_is_rejected():
    q = np.zeros((1, 2, 3, 8))
    k = np.zeros((1, 2, 2, 8))
    with pytest.raises(ValueError):
        oracle.attention(q, k, k, oracle.positions(0, 1, 2))


# ---------------------------------------------------------------------------
# the pages' own check: decode with the cache == full recomputation
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("qk_norm", [False, True])
def test_cached_decode_equals_full_recompute(qk_norm):
    rng = np.random.default_rng(10)
    B, T0, steps, Hq, Hkv, D = 2, 20, 6, 4, 2, 64
    T = T0 + steps
    q = _rand_bits(rng, B, T, Hq, D)
    k = _rand_bits(rng, B, T, Hkv, D)
    v = _rand_bits(rng, B, T, Hkv, D)
    o_full, k_rot, v_all = oracle.prefill(q, k, v, qk_norm)
    # prompt, then token-by-token with a float64 cache
    Lmax = 32
    kc = np.zeros((B, Hkv, Lmax, D))
    vc = np.zeros((B, Hkv, Lmax, D))
    _, k0, v0 = oracle.prefill(q[:, :T0], k[:, :T0], v[:, :T0], qk_norm)
    kc[:, :, :T0] = k0.transpose(0, 2, 1, 3)
    vc[:, :, :T0] = v0.transpose(0, 2, 1, 3)
    lens = np.full(B, T0)
    for s in range(steps):
        t = T0 + s
        o, knew = oracle.decode_step(q[:, t], k[:, t], v[:, t], kc, vc, lens, qk_norm)
        np.testing.assert_allclose(o, o_full[:, t], rtol=0, atol=1e-13)
        np.testing.assert_allclose(knew, k_rot[:, t], rtol=0, atol=1e-15)
        kc[:, :, t] = knew
        vc[:, :, t] = v_all[:, t]
        lens = lens + 1


def test_decode_ignores_slots_beyond_length():
    rng = np.random.default_rng(11)
    B, Hq, Hkv, D, L = 3, 4, 2, 64, 40
    lens = np.array([5, 17, 39])
    kc = rng.standard_normal((B, Hkv, L, D))
    vc = rng.standard_normal((B, Hkv, L, D))
    q, k, v = (_rand_bits(rng, B, Hq, D), _rand_bits(rng, B, Hkv, D), _rand_bits(rng, B, Hkv, D))
    o1, _ = oracle.decode_step(q, k, v, kc, vc, lens, True)
    for b in range(B):
        kc[b, :, lens[b]:] = np.nan
        vc[b, :, lens[b]:] = np.nan
    o2, _ = oracle.decode_step(q, k, v, kc, vc, lens, True)
    np.testing.assert_array_equal(o1, o2)


# ---------------------------------------------------------------------------
# continuation chunks: the same check a chunk of tokens at a time
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("qk_norm", [False, True])
def test_chunked_prefill_equals_one_prefill(qk_norm):
    """A prompt taken in chunks (different cut points per sequence, the last
    chunk ragged) gives the rows and the rotated keys of one prefill."""
    rng = np.random.default_rng(12)
    B, T, Hq, Hkv, D, Lmax = 2, 37, 6, 2, 16, 64
    q = _rand_bits(rng, B, T, Hq, D)
    k = _rand_bits(rng, B, T, Hkv, D)
    v = _rand_bits(rng, B, T, Hkv, D)
    o_full, k_rot, v_all = oracle.prefill(q, k, v, qk_norm)
    cuts = [[0, 15, 30, 37], [0, 22, 37]]
    kc = np.full((B, Hkv, Lmax, D), np.nan)     # slots past the prefix are never read
    vc = np.full((B, Hkv, Lmax, D), np.nan)
    got = np.full(o_full.shape, np.nan)
    pos0 = np.zeros(B, dtype=np.int64)
    for step in range(3):
        n_tok = np.array([max(0, (c[step + 1] - c[step]) if step + 1 < len(c) else 0)
                          for c in cuts])
        Tc = int(n_tok.max())
        qc = np.zeros((B, Tc, Hq, D), np.uint16)
        kc_new = np.zeros((B, Tc, Hkv, D), np.uint16)
        vc_new = np.zeros((B, Tc, Hkv, D), np.uint16)
        for b in range(B):
            P, n = int(pos0[b]), int(n_tok[b])
            qc[b, :n], kc_new[b, :n], vc_new[b, :n] = q[b, P:P + n], k[b, P:P + n], v[b, P:P + n]
        o, kr = oracle.prefill_chunk(qc, kc_new, vc_new, kc, vc, pos0, qk_norm, n_tok=n_tok)
        for b in range(B):
            P, n = int(pos0[b]), int(n_tok[b])
            got[b, P:P + n] = o[b, :n]
            assert np.isnan(o[b, n:]).all()
            np.testing.assert_allclose(kr[b, :n], k_rot[b, P:P + n], rtol=0, atol=1e-15)
            kc[b, :, P:P + n] = kr[b, :n].transpose(1, 0, 2)
            vc[b, :, P:P + n] = v_all[b, P:P + n].transpose(1, 0, 2)
        pos0 = pos0 + n_tok
    np.testing.assert_allclose(got, o_full, rtol=0, atol=1e-13)


def test_chunk_of_one_token_is_a_decode_step():
    rng = np.random.default_rng(13)
    B, Hq, Hkv, D, L = 3, 4, 1, 32, 48
    lens = np.array([1, 20, 47])
    kc = rng.standard_normal((B, Hkv, L, D))
    vc = rng.standard_normal((B, Hkv, L, D))
    q, k, v = (_rand_bits(rng, B, Hq, D), _rand_bits(rng, B, Hkv, D), _rand_bits(rng, B, Hkv, D))
    o_dec, k_dec = oracle.decode_step(q, k, v, kc, vc, lens, True)
    o_chk, k_chk = oracle.prefill_chunk(q[:, None], k[:, None], v[:, None], kc, vc, lens, True)
    np.testing.assert_array_equal(o_chk[:, 0], o_dec)
    np.testing.assert_array_equal(k_chk[:, 0], k_dec)


# ---------------------------------------------------------------------------
# RoPE context-extension variants (linear interpolation, NTK-aware, YaRN)
# ---------------------------------------------------------------------------
def test_theta_table_path_reproduces_plain_rope():
    rng = np.random.default_rng(20)
    x = rng.standard_normal((5, 3, 64))
    pos = np.array([0, 1, 7, 100, 4095])
    plain = oracle.rope(x, pos)
    class Plain(oracle.RopeScaling):        # the plain table through the table path
        def theta(self, D, base):
            return base ** (-2.0 * np.arange(D // 2) / D)
    # numpy's power and C's pow may round theta differently by an ulp, which the
    # position multiplies: allow |p| * 2^-52 on top of the rotation's rounding
    np.testing.assert_allclose(oracle.rope(x, pos, scaling=Plain("linear", 1.0)), plain,
                               rtol=0, atol=4e-16 * pos.max() + 1e-15)


@pytest.mark.parametrize("kind", ["linear", "ntk", "yarn"])
def test_scaling_with_factor_one_is_plain_rope(kind):
    rng = np.random.default_rng(21)
    x = rng.standard_normal((4, 2, 128))
    pos = np.array([3, 64, 1000, 9000])
    sc = oracle.RopeScaling(kind, 1.0, original_max_pos=2048)
    np.testing.assert_allclose(oracle.rope(x, pos, scaling=sc), oracle.rope(x, pos),
                               rtol=0, atol=4e-16 * pos.max() + 1e-15)


def test_linear_interpolation_closed_form():
    """Position interpolation by s: position s*m rotates like position m."""
    rng = np.random.default_rng(22)
    x = rng.standard_normal((6, 2, 96))
    m = np.array([0, 1, 5, 77, 512, 2047])
    s = 4
    got = oracle.rope(x, s * m, scaling=oracle.RopeScaling("linear", s))
    np.testing.assert_allclose(got, oracle.rope(x, m), rtol=0, atol=1e-11)


def test_ntk_is_plain_rope_with_the_larger_base():
    rng = np.random.default_rng(23)
    D, s, base = 64, 8.0, 10000.0
    x = rng.standard_normal((5, 2, D))
    pos = np.array([0, 9, 300, 5000, 30000])
    got = oracle.rope(x, pos, base, scaling=oracle.RopeScaling("ntk", s))
    np.testing.assert_allclose(got, oracle.rope(x, pos, base * s ** (D / (D - 2))),
                               rtol=0, atol=1e-10)
    th = oracle.RopeScaling("ntk", s).theta(D, base)
    # the fastest pair keeps its frequency; the slowest is divided by exactly s
    assert th[0] == 1.0
    np.testing.assert_allclose(th[-1], base ** (-(D - 2) / D) / s, rtol=1e-13)


def test_yarn_limits_and_temperature():
    D, s, base, L = 128, 8.0, 10000.0, 4096
    sc = oracle.RopeScaling("yarn", s, original_max_pos=L, alpha=1.0, beta=32.0)
    plain = base ** (-2.0 * np.arange(D // 2) / D)
    turns = L * plain / (2 * math.pi)
    th = sc.theta(D, base)
    fast, slow = turns >= 32.0, turns <= 1.0
    assert fast.any() and slow.any() and (~fast & ~slow).any()
    np.testing.assert_allclose(th[fast], plain[fast], rtol=1e-15)        # kept
    np.testing.assert_allclose(th[slow], plain[slow] / s, rtol=1e-15)    # interpolated
    mid = ~fast & ~slow                                                   # in between
    assert ((th[mid] < plain[mid]) & (th[mid] > plain[mid] / s)).all()
    rng = np.random.default_rng(24)
    x = rng.standard_normal((3, 4, D))
    y = oracle.rope(x, np.array([0, 17, 40000]), base, scaling=sc)
    mscale = 0.1 * math.log(s) + 1.0
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), mscale * np.linalg.norm(x, axis=-1),
                               rtol=1e-13)


@pytest.mark.parametrize("kind", ["linear", "ntk", "yarn"])
def test_scaled_scores_depend_on_distance_only(kind):
    rng = np.random.default_rng(25)
    D = 64
    sc = oracle.RopeScaling(kind, 4.0, original_max_pos=1024)
    qv, kv = rng.standard_normal((1, 1, D)), rng.standard_normal((1, 1, D))
    def score(m, n):
        return float((oracle.rope(qv, np.array([m]), scaling=sc) *
                      oracle.rope(kv, np.array([n]), scaling=sc)).sum())
    for m, n in [(10, 3), (700, 5), (40, 40)]:
        for shift in (1, 333, 20000):
            assert abs(score(m + shift, n + shift) - score(m, n)) < 1e-9


# ---------------------------------------------------------------------------
# document masking (packed documents, a query sees only its own document)
# ---------------------------------------------------------------------------
def test_one_document_is_plain_causal_attention():
    rng = np.random.default_rng(30)
    B, T, Hq, Hkv, D = 2, 33, 4, 2, 16
    q, k, v = (_rand_bits(rng, B, T, Hq, D), _rand_bits(rng, B, T, Hkv, D),
               _rand_bits(rng, B, T, Hkv, D))
    o1, _, _ = oracle.prefill(q, k, v, True)
    o2, _, _ = oracle.prefill(q, k, v, True, doc_id=np.full((B, T), 7))
    np.testing.assert_array_equal(o1, o2)


def test_each_document_is_its_own_prefill():
    """Rows of a packed document equal a prefill of that document alone, started
    at position 0: the mask removes the other documents, and RoPE's dependence
    on position differences alone removes the offset."""
    rng = np.random.default_rng(31)
    B, T, Hq, Hkv, D = 2, 60, 6, 2, 32
    q, k, v = (_rand_bits(rng, B, T, Hq, D), _rand_bits(rng, B, T, Hkv, D),
               _rand_bits(rng, B, T, Hkv, D))
    bounds = [[0, 1, 17, 40, 60], [0, 31, 60]]      # a one-token document included
    doc = np.zeros((B, T), dtype=np.int64)
    for b, cuts in enumerate(bounds):
        for i in range(len(cuts) - 1):
            doc[b, cuts[i]:cuts[i + 1]] = i
    o, _, _ = oracle.prefill(q, k, v, True, doc_id=doc)
    for b, cuts in enumerate(bounds):
        for i in range(len(cuts) - 1):
            a, e = cuts[i], cuts[i + 1]
            alone, _, _ = oracle.prefill(q[b:b + 1, a:e], k[b:b + 1, a:e], v[b:b + 1, a:e], True)
            np.testing.assert_allclose(o[b:b + 1, a:e], alone, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# attention backward
# ---------------------------------------------------------------------------
def _loss(q, k, v, dout):
    """L = sum(dout * o) through the forward oracle (no RoPE: q, k as given)."""
    T = q.shape[1]
    o = oracle.attention(q, k, v, np.arange(T)[None, :].repeat(q.shape[0], 0))
    return float((dout * o).sum())


def test_backward_matches_finite_differences():
    rng = np.random.default_rng(40)
    B, T, Hq, Hkv, D = 1, 5, 4, 2, 4
    q, k, v = (rng.standard_normal((B, T, Hq, D)), rng.standard_normal((B, T, Hkv, D)),
               rng.standard_normal((B, T, Hkv, D)))
    dout = rng.standard_normal((B, T, Hq, D))
    dq, dk, dv, _, _ = oracle.attention_backward(q, k, v, dout)
    eps = 1e-6
    for x, grad in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [xp if a is x else a for a in (q, k, v)]
            args_m = [xm if a is x else a for a in (q, k, v)]
            num[idx] = (_loss(*args_p, dout) - _loss(*args_m, dout)) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=0, atol=2e-8)


def test_backward_matches_torch_autograd_sdpa():
    rng = np.random.default_rng(41)
    B, T, Hq, Hkv, D = 2, 37, 6, 2, 16
    q, k, v = (rng.standard_normal((B, T, Hq, D)), rng.standard_normal((B, T, Hkv, D)),
               rng.standard_normal((B, T, Hkv, D)))
    dout = rng.standard_normal((B, T, Hq, D))
    dq, dk, dv, o, lse = oracle.attention_backward(q, k, v, dout)
    tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    g = Hq // Hkv
    out = F.scaled_dot_product_attention(tq.transpose(1, 2),
                                         tk.repeat_interleave(g, dim=2).transpose(1, 2),
                                         tv.repeat_interleave(g, dim=2).transpose(1, 2),
                                         is_causal=True).transpose(1, 2)
    out.backward(torch.tensor(dout))
    np.testing.assert_allclose(o, out.detach().numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=0, atol=1e-11)
    # log-sum-exp of the first row: one key
    s00 = float(q[0, 0, 0] @ k[0, 0, 0]) / math.sqrt(D)
    assert abs(lse[0, 0, 0] - s00) < 1e-12
    # every row: torch's logsumexp over the row's visible keys
    sc = (tq.detach().transpose(1, 2) @ tk.detach().repeat_interleave(g, dim=2)
          .transpose(1, 2).transpose(-1, -2)) / math.sqrt(D)
    sc = sc.masked_fill(torch.ones(T, T, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(sc, dim=-1).numpy(), rtol=0, atol=1e-12)


def test_backward_sums():
    """dV summed over keys is dO summed over the group's queries (softmax rows
    sum to one), and dS rows sum to zero, so dQ is unchanged by adding a
    constant vector to every key."""
    rng = np.random.default_rng(42)
    B, T, Hq, Hkv, D = 1, 20, 4, 1, 8
    q, k, v = (rng.standard_normal((B, T, Hq, D)), rng.standard_normal((B, T, Hkv, D)),
               rng.standard_normal((B, T, Hkv, D)))
    dout = rng.standard_normal((B, T, Hq, D))
    dq, dk, dv, _, _ = oracle.attention_backward(q, k, v, dout)
    np.testing.assert_allclose(dv.sum(axis=1)[0, 0], dout.sum(axis=(1, 2))[0], rtol=0, atol=1e-12)
    dq2, _, _, _, _ = oracle.attention_backward(q, k + rng.standard_normal((1, 1, Hkv, D)), v, dout)
    np.testing.assert_allclose(dq2, dq, rtol=0, atol=1e-11)
