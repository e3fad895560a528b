"""Pins of the oracle's int8 KV cache (orc_enable_kv8, orc_kv8_row).

Reading (the pages give no int8 KV cache; the variant is this build's): every K
and V row, when stored, becomes Q8_0 groups of head_size values quantized with
the quantize() rule of "超精简LLM部署" §1 INT8量化压缩, and attention reads
code * scale rounded to fp32.  Pins: the row invariants a Q8_0 group must
satisfy (codes in [-127, 127], the group max at +-127, error at most scale/2, a
zero group kept), and the decode step with the int8 cache against the
independent full-sequence float64 restatement (prefill_form) with its K/V
rows quantized per head after RoPE, in fp32 and Q8_0."""
import numpy as np
import pytest

import oracle
import synth
from prefill_form import prefill_logits

ODD = synth.ModelSpec("odd-kv8", 48, 100, 2, 6, 2, 50, 24, 0, seed=10, wsigma=0.2, nsigma=0.1)
ODDQ = synth.ModelSpec("oddq-kv8", 48, 112, 2, 6, 2, 50, 24, 0, seed=10, wsigma=0.2, nsigma=0.1)


@pytest.mark.parametrize("hs", [8, 16, 48, 128])
def test_kv8_row_is_a_q80_group_per_head(hs):
    rng = np.random.default_rng(hs)
    n = 4 * hs
    row = (rng.standard_normal(n) * np.array([1e-3, 1.0, 50.0, 0.0]).repeat(hs)).astype(np.float32)
    out = oracle.kv8_row(row, hs)
    for g in range(4):
        x = row[g * hs:(g + 1) * hs].astype(np.float64)
        y = out[g * hs:(g + 1) * hs].astype(np.float64)
        wmax = np.abs(x).max()
        if wmax == 0:
            assert np.all(y == 0)
            continue
        scale = float(np.float32(np.float32(wmax) / np.float32(127.0)))
        codes = y / scale
        # each value is (fp32-rounded) code * scale with an integer code in [-127, 127]
        assert np.all(np.abs(codes - np.round(codes)) <= 127 * 2.0 ** -23)
        assert np.abs(np.round(codes)).max() == 127
        assert np.abs(y - x).max() <= scale / 2 * (1 + 1e-6) + wmax * 2.0 ** -23


def _decode(spec, toks, q80, gs, kv8):
    b = synth.blob(spec)
    m = oracle.Model(spec.cfg, b, spec.shared_weights)
    if q80:
        m.enable_q80(gs)
    if kv8:
        m.enable_kv8()
    out = np.stack([m.forward(int(t), p, q80=q80) for p, t in enumerate(toks)])
    m.close()
    return out, b


@pytest.mark.parametrize("spec,q80,gs", [(ODD, False, 0), (synth.TINY, False, 0), (ODDQ, True, 16),
                                         (synth.M15, True, 32)], ids=["odd-fp32", "tiny-fp32", "oddq-q80", "15M-q80"])
def test_decode_with_kv8_equals_prefill_form(spec, q80, gs):
    toks = synth.tokens(spec.seed, 11, 16, spec.vocab_size)
    got, b = _decode(spec, toks, q80, gs, kv8=True)
    ref = prefill_logits(spec.cfg, b, spec.shared_weights, toks, q80_gs=gs, quantize=oracle.quantize, kv8=True)
    scale = np.abs(ref).max()
    assert np.abs(got - ref).max() <= 2e-6 * scale
    # and the int8 cache does change the step (the pin would not see a no-op)
    plain, _ = _decode(spec, toks, q80, gs, kv8=False)
    assert np.abs(plain - got).max() > 1e-6 * scale


def test_enable_kv8_quantizes_loaded_rows():
    spec = ODD
    b = synth.blob(spec)
    m = oracle.Model(spec.cfg, b, spec.shared_weights)
    k, v = synth.kv_prefill(spec, seq=0, n_pos=10)
    m.kv_load(k, v)
    m.enable_kv8()
    kr, vr = m.kv_read(10)
    hs = spec.dim // spec.n_heads
    for l in range(spec.n_layers):
        for t in range(10):
            assert np.array_equal(kr[l, t], oracle.kv8_row(k[l, t], hs))
            assert np.array_equal(vr[l, t], oracle.kv8_row(v[l, t], hs))
    m.close()
