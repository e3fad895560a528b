"""l2c_prefill: a prompt run as GEMM chunks of up to 32 tokens, against the
oracle fed the same tokens one at a time (the pages' way: forward per prompt
token).

For every case the K/V cache rows the prompt writes and the last token's
logits must match the oracle's (fp32: logits within 1e-4 of max |logit|, K/V
within 1e-5; Q8_0: both within 1e-5, i.e. the activation codes are
reproduced), and a decode step after the prompt, reading the cache the
prefill wrote, must match the oracle's next step.  Cases: the tiny shape
(GQA ratio 2, head size 8, hidden 172: a ragged K tail in the GEMM), 45
tokens from position 0 (chunks of 32 and 13) and 7 more continuing at 45;
the 15M shape in fp32 and Q8_0 (GS=32); a GQA ratio 4 shape in Q8_0 whose
prompt starts at position 10 after 10 loaded cache rows; the 110M shape in
fp32, 64 tokens.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import TOL_F32, need_gpu, rel_err

pytestmark = pytest.mark.gpu

GQA4 = synth.ModelSpec("prefill-gqa4", 256, 640, 2, 8, 2, 1000, 300, 0, seed=21)


def _pair(spec, gs=0):
    torch, l2c = need_gpu()
    b = synth.blob(spec)
    dec = l2c.Decoder(spec.cfg, torch.from_numpy(b).cuda(), spec.shared_weights)
    orc = oracle.Model(spec.cfg, b, spec.shared_weights)
    if gs:
        dec.enable_q80(gs)
        orc.enable_q80(gs)
    return torch, l2c, dec, orc


def _check_prompt(torch, dec, orc, spec, toks, pos0, q80):
    n = len(toks)
    tol = 1e-5 if q80 else TOL_F32
    last = torch.empty(spec.vocab_size, dtype=torch.float32, device="cuda")
    dec.prefill(toks, pos0, q80=q80, logits_last=last)
    ref = None
    for i, t in enumerate(toks):
        ref = orc.forward(int(t), pos0 + i, q80=q80)
    assert rel_err(last.cpu().numpy(), ref) <= tol
    k, v = dec.kv_read(pos0 + n)
    kr, vr = orc.kv_read(pos0 + n)
    assert rel_err(k[:, pos0:], kr[:, pos0:]) <= 1e-5 and rel_err(v[:, pos0:], vr[:, pos0:]) <= 1e-5
    return pos0 + n


def _check_next_step(dec, orc, tok, pos, q80):
    got = dec.forward(tok, pos, q80=q80).cpu().numpy()
    ref = orc.forward(tok, pos, q80=q80)
    assert rel_err(got, ref) <= (1e-5 if q80 else TOL_F32)


def test_prefill_tiny_two_calls_ragged_chunks():
    spec = synth.TINY
    torch, l2c, dec, orc = _pair(spec)
    toks = synth.tokens(spec.seed, 50, 52, spec.vocab_size)
    p = _check_prompt(torch, dec, orc, spec, toks[:45], 0, False)
    p = _check_prompt(torch, dec, orc, spec, toks[45:], p, False)
    _check_next_step(dec, orc, 3, p, False)
    dec.close()
    orc.close()


@pytest.mark.parametrize("gs", [0, 32], ids=["fp32", "q80-gs32"])
def test_prefill_15m(gs):
    spec = synth.M15
    torch, l2c, dec, orc = _pair(spec, gs)
    toks = synth.tokens(spec.seed, 51, 40, spec.vocab_size)
    p = _check_prompt(torch, dec, orc, spec, toks, 0, bool(gs))
    _check_next_step(dec, orc, 7, p, bool(gs))
    dec.close()
    orc.close()


def test_prefill_gqa4_q80_after_loaded_rows():
    spec = GQA4
    torch, l2c, dec, orc = _pair(spec, 32)
    k, v = synth.kv_prefill(spec, seq=0, n_pos=10)
    dec.kv_load(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    orc.kv_load(k, v)
    toks = synth.tokens(spec.seed, 52, 70, spec.vocab_size)
    p = _check_prompt(torch, dec, orc, spec, toks, 10, True)
    _check_next_step(dec, orc, 11, p, True)
    dec.close()
    orc.close()


def test_prefill_110m_fp32():
    spec = synth.M110
    torch, l2c, dec, orc = _pair(spec)
    toks = synth.tokens(spec.seed, 53, 64, spec.vocab_size)
    p = _check_prompt(torch, dec, orc, spec, toks, 0, False)
    _check_next_step(dec, orc, 5, p, False)
    dec.close()
    orc.close()


def test_prefill_rejects_bad_arguments():
    spec = synth.TINY
    torch, l2c, dec, orc = _pair(spec)
    ok = np.zeros(4, np.int32)
    for toks, pos0 in ((np.zeros(0, np.int32), 0), (ok, spec.seq_len - 3), (ok, -1),
                       (np.array([spec.vocab_size], np.int32), 0)):
        with pytest.raises(l2c.L2CError) as e:
            dec.prefill(toks, pos0)
        assert e.value.code == l2c.L2C_E_ARG
    with pytest.raises(l2c.L2CError) as e:
        dec.prefill(ok, 0, q80=True)  # no Q8_0 weights yet
    assert e.value.code == l2c.L2C_E_STATE
    dec.close()
    orc.close()


def test_prefill_second_sequence_of_a_batch_handle():
    """A prompt into sequence 1 of a two-sequence handle: its cache rows and last
    logits match the oracle's sequence 1; sequence 0's cache stays untouched."""
    torch, l2c = need_gpu()
    spec = synth.M15
    b = synth.blob(spec)
    dec = l2c.Decoder(spec.cfg, torch.from_numpy(b).cuda(), spec.shared_weights, max_batch=2)
    orc = oracle.Model(spec.cfg, b, spec.shared_weights, n_seq=2)
    toks = synth.tokens(spec.seed, 54, 37, spec.vocab_size)
    last = torch.empty(spec.vocab_size, dtype=torch.float32, device="cuda")
    dec.prefill(toks, 0, logits_last=last, seq=1)
    ref = None
    for i, t in enumerate(toks):
        ref = orc.forward(int(t), i, seq=1)
    assert rel_err(last.cpu().numpy(), ref) <= TOL_F32
    k, v = dec.kv_read(37, seq=1)
    kr, vr = orc.kv_read(37, seq=1)
    assert rel_err(k, kr) <= 1e-5 and rel_err(v, vr) <= 1e-5
    k0, v0 = dec.kv_read(37, seq=0)
    assert not np.any(k0) and not np.any(v0)
    dec.close()
    orc.close()
