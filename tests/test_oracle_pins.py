"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks one oracle function against something other than itself:
a closed form, an invariant, a hand-worked case from the pages, a library
routine the special case reduces to, or an independent formulation (the
full-sequence causal "prefill" form in float64 NumPy, the formulation the
karpathy-notes Q&A page says llama2.c's own test compared its C code with).
"""
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


# ---------------------------------------------------------------- RMSNorm --
def test_rmsnorm_constant_vector_closed_form():
    for c in (0.3, -2.0, 1e-3, 17.0):
        n = 96
        x = np.full(n, c, dtype=np.float32)
        w = np.linspace(0.5, 1.5, n).astype(np.float32)
        o = oracle.rmsnorm(x, w)
        expect = w.astype(np.float64) * c / np.sqrt(c * c + 1e-5)
        np.testing.assert_allclose(o, expect, rtol=2e-7, atol=0)


def test_rmsnorm_unit_rms_and_scale_invariance():
    x = rng.standard_normal(288).astype(np.float32) * 3
    w = np.ones(288, np.float32)
    o = oracle.rmsnorm(x, w)
    assert abs(np.sqrt(np.mean(o.astype(np.float64) ** 2)) - 1) < 1e-5
    o2 = oracle.rmsnorm(x * 8, w)  # exact power-of-two scale; eps contributes < 1e-7
    np.testing.assert_allclose(o2, o, rtol=1e-6)


# ----------------------------------------------------------------- matvec --
def test_matvec_one_hot_returns_column():
    W = rng.standard_normal((7, 13)).astype(np.float32)
    for j in (0, 5, 12):
        x = np.zeros(13, np.float32)
        x[j] = 1
        assert np.array_equal(oracle.matvec(W, x), W[:, j])


def test_matvec_brute_force():
    W = rng.standard_normal((37, 53)).astype(np.float32)
    x = rng.standard_normal(53).astype(np.float32)
    exact = np.array([sum(float(W[i, j]) * float(x[j]) for j in range(53)) for i in range(37)])
    np.testing.assert_allclose(oracle.matvec(W, x), exact, rtol=1e-6, atol=1e-6)


# ------------------------------------------------------------------- RoPE --
def test_rope_pos0_identity_and_norms():
    v = rng.standard_normal(64).astype(np.float32)
    assert np.array_equal(oracle.rope(v, 16, 0), v)
    for pos in (1, 17, 255, 4095):
        r = oracle.rope(v, 16, pos).astype(np.float64)
        n0 = np.hypot(v[0::2].astype(np.float64), v[1::2])
        n1 = np.hypot(r[0::2], r[1::2])
        np.testing.assert_allclose(n1, n0, rtol=3e-7)


def test_rope_direction_and_frequencies():
    hs = 8
    # pair (1, 0) rotated by theta lands on (cos theta, sin theta): counter-clockwise
    v = np.tile(np.array([1.0, 0.0], np.float32), hs // 2)
    pos = 3
    r = oracle.rope(v, hs, pos)
    for j in range(0, hs, 2):
        theta = np.float32(pos) * np.float32(10000.0 ** (-j / hs))
        assert abs(r[j] - np.cos(np.float64(theta))) < 2e-7
        assert abs(r[j + 1] - np.sin(np.float64(theta))) < 2e-7
    # frequency closed form: 1 at j = 0, 10000^(-j/hs) otherwise
    assert oracle.rope_freq(0, 128) == 1.0
    for j in (2, 64, 126):
        assert abs(oracle.rope_freq(j, 128) / 10000.0 ** (-j / 128) - 1) < 2e-7


def test_rope_relative_position_invariant():
    hs = 64
    q = rng.standard_normal(hs).astype(np.float32)
    k = rng.standard_normal(hs).astype(np.float32)
    for m, n in ((5, 2), (100, 37), (1000, 999)):
        a = np.dot(oracle.rope(q, hs, m).astype(np.float64), oracle.rope(k, hs, n))
        for delta in (1, 11, 300):
            b = np.dot(oracle.rope(q, hs, m + delta).astype(np.float64), oracle.rope(k, hs, n + delta))
            assert abs(a - b) < 1e-4 * (np.linalg.norm(q) * np.linalg.norm(k))


def test_rope_matches_precomputed_complex_table():
    # the Q&A page: PyTorch precomputes the cos/sin table (freqs_cis) and views
    # adjacent pairs as complex numbers; the C code evaluates cosf/sinf on the fly.
    hs, H, S = 16, 3, 50
    freqs = np.array([np.float32(10000.0 ** (-j / hs)) for j in range(0, hs, 2)], np.float32)
    theta = np.outer(np.arange(S, dtype=np.float32), freqs).astype(np.float32)
    cis = np.exp(1j * theta.astype(np.float64))
    v = rng.standard_normal(H * hs).astype(np.float32)
    for pos in (0, 1, 7, 49):
        z = (v[0::2].astype(np.float64) + 1j * v[1::2]).reshape(H, hs // 2) * cis[pos]
        ref = np.stack([z.real, z.imag], -1).reshape(-1)
        np.testing.assert_allclose(oracle.rope(v, hs, pos), ref, rtol=0, atol=3e-6)


# ---------------------------------------------------------------- softmax --
def test_softmax_invariants():
    x = rng.standard_normal(101) * 5
    p = oracle.softmax(x)
    assert abs(p.sum() - 1) < 1e-12
    np.testing.assert_allclose(oracle.softmax(x + 123.0), p, rtol=1e-12)
    assert oracle.softmax(np.array([3.7]))[0] == 1.0
    a, b = 0.3, -1.1
    np.testing.assert_allclose(oracle.softmax(np.array([a, b]))[0], 1 / (1 + np.exp(b - a)), rtol=1e-14)


# -------------------------------------------------------------- attention --
def test_attention_pos0_returns_matching_v():
    H, Hkv, hs = 8, 2, 16
    q = rng.standard_normal(H * hs).astype(np.float32)
    kc = rng.standard_normal((4, Hkv * hs)).astype(np.float32)
    vc = rng.standard_normal((4, Hkv * hs)).astype(np.float32)
    o = oracle.attention(q, kc, vc, 0, H, Hkv).reshape(H, hs)
    rep = H // Hkv
    for h in range(H):
        g = h // rep  # contiguous groups of query heads share one KV head
        assert np.array_equal(o[h], vc[0, g * hs:(g + 1) * hs])


def test_attention_equal_keys_give_mean_of_v():
    H, Hkv, hs, T = 4, 4, 8, 9
    q = rng.standard_normal(H * hs).astype(np.float32)
    kc = np.tile(rng.standard_normal(Hkv * hs).astype(np.float32), (T, 1))
    vc = rng.standard_normal((T, Hkv * hs)).astype(np.float32)
    o = oracle.attention(q, kc, vc, T - 1, H, Hkv)
    np.testing.assert_allclose(o, vc.astype(np.float64).mean(0), rtol=1e-6, atol=1e-7)


def test_attention_two_positions_closed_form_and_scale():
    hs = 4
    q = np.array([1, 0, 0, 0], np.float32)
    kc = np.array([[0, 0, 0, 0], [2, 0, 0, 0]], np.float32)
    vc = np.array([[1, 0, 0, 0], [0, 1, 0, 0]], np.float32)
    o = oracle.attention(q, kc, vc, 1, 1, 1)
    w1 = 1 / (1 + np.exp(-2 / np.sqrt(hs)))  # scores 0 and 2/sqrt(hs)
    np.testing.assert_allclose(o, [1 - w1, w1, 0, 0], rtol=1e-7, atol=1e-8)


def test_attention_gqa_equals_mha_with_repeated_kv():
    H, Hkv, hs, T = 8, 2, 16, 21
    q = rng.standard_normal(H * hs).astype(np.float32)
    kc = rng.standard_normal((T, Hkv * hs)).astype(np.float32)
    vc = rng.standard_normal((T, Hkv * hs)).astype(np.float32)
    rep = H // Hkv
    k_mha = np.repeat(kc.reshape(T, Hkv, hs), rep, axis=1).reshape(T, H * hs)
    v_mha = np.repeat(vc.reshape(T, Hkv, hs), rep, axis=1).reshape(T, H * hs)
    a = oracle.attention(q, kc, vc, T - 1, H, Hkv)
    b = oracle.attention(q, k_mha, v_mha, T - 1, H, H)
    assert np.array_equal(a, b)


# ----------------------------------------------------------------- SwiGLU --
def test_silu_special_values():
    assert oracle.silu(0.0) == 0.0
    assert abs(oracle.silu(40.0) - 40.0) < 1e-12
    assert abs(oracle.silu(-40.0)) < 1e-15
    assert abs(oracle.silu(1.0) - 1 / (1 + np.exp(-1.0))) < 1e-15
    a = np.array([0.0, 1.0, -2.0], np.float32)
    b = np.array([5.0, 3.0, 2.0], np.float32)
    np.testing.assert_allclose(oracle.swiglu(a, b), [0.0, 3 / (1 + np.exp(-1.0)), -4 / (1 + np.exp(2.0))],
                               rtol=1e-7)


# ------------------------------------------------------------------- Q8_0 --
def _golden_cases():
    cases, cur = [], None
    for ln in open(os.path.join(GOLDEN, "q80_quantize_cases.txt")):
        ln = ln.strip()
        if not ln or ln.startswith("#"):
            continue
        key, *vals = ln.split()
        if key == "case":
            cur = {"name": vals[0]}
            cases.append(cur)
        else:
            cur[key] = vals
    return cases


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_quantize_listing_cases(case):
    gs = int(case["gs"][0])
    x = np.array([float(v) for v in case["x"]], np.float32)
    q, s = oracle.quantize(x, gs)
    assert q.tolist() == [int(v) for v in case["q"]]
    np.testing.assert_allclose(s, [float(v) for v in case["scale"]], rtol=1e-7, atol=0)


def test_quantize_bounds_and_error():
    for gs in (32, 64):
        x = (rng.standard_normal(64 * 50) * rng.uniform(0.01, 10, 64 * 50)).astype(np.float32)
        q, s = oracle.quantize(x, gs)
        assert q.min() >= -127 and q.max() <= 127
        g = x.reshape(-1, gs)
        qg = q.reshape(-1, gs).astype(np.int64)
        imax = np.argmax(np.abs(g), axis=1)
        assert np.all(np.abs(qg[np.arange(len(g)), imax]) == 127)
        deq = oracle.dequantize(q, s, gs).reshape(-1, gs).astype(np.float64)
        err = np.abs(deq - g)
        assert np.all(err <= s[:, None].astype(np.float64) * (0.5 + 1e-5))
    with pytest.raises(ValueError):
        oracle.quantize(np.zeros(33, np.float32), 32)


def _golden_q4_cases():
    cases, cur = [], None
    for ln in open(os.path.join(GOLDEN, "q40_quantize_cases.txt")):
        ln = ln.strip()
        if not ln or ln.startswith("#"):
            continue
        key, *vals = ln.split()
        if key == "case":
            cur = {"name": vals[0]}
            cases.append(cur)
        else:
            cur[key] = vals
    return cases


@pytest.mark.parametrize("case", _golden_q4_cases(), ids=lambda c: c["name"])
def test_quantize4_cases(case):
    gs = int(case["gs"][0])
    x = np.array([float(v) for v in case["x"]], np.float32)
    q, s = oracle.quantize4(x, gs)
    assert q.tolist() == [int(v) for v in case["q"]]
    np.testing.assert_allclose(s, [float(v) for v in case["scale"]], rtol=1e-7, atol=0)


def test_quantize4_is_the_nearest_code():
    """Every Q4_0 code is the integer in [-7, 7] nearest to x / scale (brute force over
    the 15 codes; ties, which random inputs do not hit, aside), the group's largest
    magnitude maps to +-7, and the scale is max|x| / 7 in fp32."""
    for gs in (32, 64, 128):
        x = (rng.standard_normal(128 * 20) * rng.uniform(0.01, 10, 128 * 20)).astype(np.float32)
        q, s = oracle.quantize4(x, gs)
        g = x.reshape(-1, gs)
        np.testing.assert_array_equal(s, (np.abs(g).max(1) / np.float32(7)).astype(np.float32))
        quot = (g / s[:, None]).astype(np.float32).astype(np.float64)
        codes = np.arange(-7, 8, dtype=np.float64)
        best = codes[np.argmin(np.abs(quot[..., None] - codes), axis=-1)]
        np.testing.assert_array_equal(q.reshape(-1, gs), best)
        imax = np.argmax(np.abs(g), axis=1)
        assert np.all(np.abs(q.reshape(-1, gs)[np.arange(len(g)), imax]) == 7)
        deq = oracle.dequantize(q, s, gs).reshape(-1, gs).astype(np.float64)
        assert np.all(np.abs(deq - g) <= s[:, None].astype(np.float64) * (0.5 + 1e-5))
    q, s = oracle.quantize4(np.zeros(64, np.float32), 32)
    assert not q.any() and not s.any()
    with pytest.raises(ValueError):
        oracle.quantize4(np.zeros(33, np.float32), 32)


def test_group_dots_brute_force():
    gs, n, d = 32, 96, 5
    qw = rng.integers(-127, 128, (d, n)).astype(np.int8)
    qx = rng.integers(-127, 128, n).astype(np.int8)
    got = oracle.q80_group_dots(qw, qx, gs)
    for i in range(d):
        for g in range(n // gs):
            assert got[i, g] == sum(int(qw[i, g * gs + k]) * int(qx[g * gs + k]) for k in range(gs))
    # extreme magnitudes stay exact (|sum| <= 64 * 127^2 < 2^31)
    big = oracle.q80_group_dots(np.full((1, 64), -127, np.int8), np.full(64, -127, np.int8), 64)
    assert big[0, 0] == 64 * 127 * 127


def test_matvec_q80_equals_dequantized_matvec():
    # with power-of-two scales every product is exact, so the Q8_0 matvec must equal the
    # fp32 matvec of the dequantized operands
    gs, n, d = 64, 256, 9
    qw = rng.integers(-127, 128, (d, n)).astype(np.int8)
    qx = rng.integers(-127, 128, n).astype(np.int8)
    sw = (2.0 ** rng.integers(-8, 0, (d, n // gs))).astype(np.float32)
    sx = (2.0 ** rng.integers(-8, 0, n // gs)).astype(np.float32)
    Wd = qw.astype(np.float64) * np.repeat(sw, gs, axis=1)
    xd = qx.astype(np.float64) * np.repeat(sx, gs)
    np.testing.assert_allclose(oracle.matvec_q80(qw, sw, qx, sx, gs), Wd @ xd, rtol=1e-7)


def test_argmax_lowest_index_on_ties():
    x = np.array([0.1, 0.9, -3, 0.9, 0.2], np.float32)
    assert oracle.argmax(x) == 1
    assert oracle.argmax(np.array([-1.0, -1.0], np.float32)) == 0
    y = rng.standard_normal(32000).astype(np.float32)
    assert oracle.argmax(y) == int(np.argmax(y))
