"""Whole-step pins of the oracle: the decode-step form against the full-sequence
prefill form (independent float64 NumPy), tied vs untied classifier storage,
KV-cache slot placement, and the distance of the pages' own fp32 loops."""
import numpy as np
import pytest

import oracle
import synth
from prefill_form import prefill_logits

# brute-force-sized shape: d=8, one layer, 2 query heads sharing 1 KV head, V=16, S=8
BRUTE = synth.ModelSpec("brute", 8, 12, 1, 2, 1, 16, 8, 1, seed=9, wsigma=0.5, nsigma=0.2)
ODD = synth.ModelSpec("odd", 48, 100, 2, 6, 2, 50, 24, 0, seed=10, wsigma=0.2, nsigma=0.1)
ODDQ = synth.ModelSpec("oddq", 48, 112, 2, 6, 2, 50, 24, 0, seed=10, wsigma=0.2, nsigma=0.1)


def _decode_all(spec, toks, q80=False, gs=0, q40=False):
    b = synth.blob(spec)
    m = oracle.Model(spec.cfg, b, spec.shared_weights)
    if q80:
        m.enable_q80(gs)
    if q40:
        m.enable_q40(gs)
    return np.stack([m.forward(int(t), p, q80=q80, q40=q40) for p, t in enumerate(toks)]), b


@pytest.mark.parametrize("spec,T", [(BRUTE, 8), (ODD, 24), (synth.TINY, 40), (synth.M15, 24)],
                         ids=["brute", "odd", "tiny", "15M"])
def test_decode_equals_prefill_fp32(spec, T):
    toks = synth.tokens(spec.seed, 7, T, spec.vocab_size)
    got, b = _decode_all(spec, toks)
    ref = prefill_logits(spec.cfg, b, spec.shared_weights, toks)
    scale = np.abs(ref).max()
    assert np.abs(got - ref).max() <= 2e-6 * scale


@pytest.mark.parametrize("spec,gs,T", [(ODDQ, 16, 12), (synth.M15, 32, 12)], ids=["oddq", "15M"])
def test_decode_equals_prefill_q80(spec, gs, T):
    toks = synth.tokens(spec.seed, 8, T, spec.vocab_size)
    got, b = _decode_all(spec, toks, q80=True, gs=gs)
    ref = prefill_logits(spec.cfg, b, spec.shared_weights, toks, q80_gs=gs, quantize=oracle.quantize)
    scale = np.abs(ref).max()
    # both formulations round to fp32 at the same points, so every Q8_0 code is decided
    # on the same fp32 value: the codes agree and only double rounding noise remains
    assert np.abs(got - ref).max() <= 2e-6 * scale


@pytest.mark.parametrize("spec,gs,T", [(ODDQ, 16, 12), (synth.M15, 32, 12)], ids=["oddq", "15M"])
def test_decode_equals_prefill_q40(spec, gs, T):
    toks = synth.tokens(spec.seed, 8, T, spec.vocab_size)
    got, b = _decode_all(spec, toks, q40=True, gs=gs)
    ref = prefill_logits(spec.cfg, b, spec.shared_weights, toks, q80_gs=gs, quantize=oracle.quantize,
                         wquantize=oracle.quantize4)
    assert np.abs(got - ref).max() <= 2e-6 * np.abs(ref).max()


def test_q40_coarser_than_q80_and_q80_set_untouched():
    """Q4_0 moves the logits further from fp32 than Q8_0 does; enabling it beside the
    Q8_0 set (another group size) leaves the Q8_0 step as it was."""
    spec = synth.M15
    toks = synth.tokens(spec.seed, 9, 8, spec.vocab_size)
    f, b = _decode_all(spec, toks)
    q8, _ = _decode_all(spec, toks, q80=True, gs=32)
    q4, _ = _decode_all(spec, toks, q40=True, gs=32)
    e8, e4 = np.abs(f - q8).max(), np.abs(f - q4).max()
    assert e8 < e4 <= 0.5 * np.abs(f).max()
    m = oracle.Model(spec.cfg, b, spec.shared_weights)
    m.enable_q80(32)
    m.enable_q40(96)
    both = np.stack([m.forward(int(t), p, q80=True) for p, t in enumerate(toks)])
    assert np.array_equal(both, q8)
    with pytest.raises(ValueError):
        m.enable_q40(32)  # already made with another group size


def test_q80_close_to_fp32():
    spec = synth.M15
    toks = synth.tokens(spec.seed, 9, 8, spec.vocab_size)
    f, _ = _decode_all(spec, toks)
    q, _ = _decode_all(spec, toks, q80=True, gs=32)
    assert np.abs(f - q).max() <= 0.05 * np.abs(f).max()
    assert np.abs(f - q).max() > 0  # quantization does change the logits


def test_tied_equals_untied_with_copied_classifier():
    spec = synth.TINY
    b = synth.blob(spec)
    d, V = spec.dim, spec.vocab_size
    untied = np.concatenate([b, b[:V * d]])  # Wcls := E appended after the legacy tables
    m1 = oracle.Model(spec.cfg, b, 1)
    m2 = oracle.Model(spec.cfg, untied, 0)
    for p, t in enumerate((1, 77, 300)):
        assert np.array_equal(m1.forward(t, p), m2.forward(t, p))
    # and a different classifier changes the logits
    untied[-V * d:] = -untied[-V * d:]
    m3 = oracle.Model(spec.cfg, untied, 0)
    m1.kv_reset()
    np.testing.assert_allclose(m3.forward(1, 0), -m1.forward(1, 0), rtol=1e-6, atol=1e-7)


def test_kv_slot_written_at_pos():
    spec = synth.TINY
    b = synth.blob(spec)
    m = oracle.Model(spec.cfg, b, 1)
    m.forward(5, 0)
    k0, v0 = m.kv_read(3)
    assert np.all(k0[:, 1:] == 0) and np.any(k0[:, 0] != 0)
    m.forward(9, 2)  # position 1 skipped: slot 1 stays empty
    k1, v1 = m.kv_read(3)
    assert np.array_equal(k1[:, 0], k0[:, 0]) and np.all(k1[:, 1] == 0) and np.any(k1[:, 2] != 0)
    # layer 0's k at pos 0 is RoPE(identity at pos 0) of Wk @ rmsnorm(E[5])
    d, h, L, H, Hkv, V, S = spec.cfg
    hs = d // H
    E = b[:V * d].reshape(V, d)
    w_att = b[V * d:V * d + d]
    off_wk = V * d + L * d + L * d * d
    Wk = b[off_wk:off_wk + Hkv * hs * d].reshape(Hkv * hs, d)
    xn = E[5].astype(np.float64) / np.sqrt(np.mean(E[5].astype(np.float64) ** 2) + 1e-5) * w_att
    np.testing.assert_allclose(k0[0, 0], Wk.astype(np.float64) @ xn, rtol=1e-5, atol=1e-6)


def test_kv_load_then_forward_matches_prefill():
    # a cache filled with the oracle's own k/v from positions 0..P-1 must give the same
    # step as having decoded those positions
    spec = synth.TINY
    b = synth.blob(spec)
    toks = synth.tokens(0, 11, 12, spec.vocab_size)
    m = oracle.Model(spec.cfg, b, 1)
    for p in range(11):
        m.forward(int(toks[p]), p)
    k, v = m.kv_read(11)
    ref = m.forward(int(toks[11]), 11)
    m2 = oracle.Model(spec.cfg, b, 1)
    m2.kv_load(k, v)
    assert np.array_equal(m2.forward(int(toks[11]), 11), ref)


def test_pages_fp32_loops_within_tolerance_of_double():
    # The pages' run.c sums in fp32 left to right; the oracle sums in double.  The
    # gap between the two is the scale of rounding noise that the GPU tolerance
    # (1e-4 * max|logit| for fp32) must cover with margin.
    spec = synth.M15
    b = synth.blob(spec)
    toks = synth.tokens(spec.seed, 12, 16, spec.vocab_size)
    m = oracle.Model(spec.cfg, b, 1)
    ref = np.stack([m.forward(int(t), p) for p, t in enumerate(toks)])
    m2 = oracle.Model(spec.cfg, b, 1)
    with oracle.fp32_accum():
        f32 = np.stack([m2.forward(int(t), p) for p, t in enumerate(toks)])
    gap = np.abs(ref - f32).max() / np.abs(ref).max()
    assert 0 < gap < 1e-5


def test_generate_is_greedy_chain():
    spec = synth.TINY
    b = synth.blob(spec)
    m = oracle.Model(spec.cfg, b, 1)
    toks, lg = m.generate(1, 10)
    m2 = oracle.Model(spec.cfg, b, 1)
    tok = 1
    for t in range(10):
        l = m2.forward(tok, t)
        assert np.array_equal(l, lg[t])
        tok = int(np.argmax(l))
        assert tok == toks[t]


def test_rejects_bad_arguments():
    spec = synth.TINY
    b = synth.blob(spec)
    m = oracle.Model(spec.cfg, b, 1)
    for tok, pos in ((-1, 0), (spec.vocab_size, 0), (0, -1), (0, spec.seq_len)):
        with pytest.raises(ValueError):
            m.forward(tok, pos)
    with pytest.raises(ValueError):
        oracle.Model(spec.cfg, b[:-1].copy(), 1)
    with pytest.raises(ValueError):
        m.forward(1, 0, q80=True)  # Q8_0 weights not made yet
