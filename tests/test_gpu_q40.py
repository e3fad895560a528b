"""The Q4_0 weight variant (l2c_enable_q40 / l2c_forward_q40) against the oracle's
(orc_enable_q40).

Reading ("技术深度解析", 整数量化路径: runq.c with 4-bit integer groups, no rule
given): quantize() of "超精简LLM部署" §1 with 4-bit codes, scale = max|x| / 7 and
codes in [-7, 7], on every matvec weight and the embedding table; the matvec
inputs stay Q8_0 at the same group size.  Both sides decide every code on the
same fp32 values and sum exact int32 group dots times both scales in double, so
the logits match to 1e-5 of their largest magnitude.  Cases: 15M (gs 32, widths
that are not multiples of 64), GQA ratio 4 at gs 64 and 128, the on-device greedy
loop, the int8 KV cache with Q4_0 weights, a Q8_0 and a Q4_0 set on one handle,
and the entry points that refuse Q4_0.  The 7B shape is in test_gpu_full_size.py.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import TOL_Q80, need_gpu, rel_err, top2_gap

pytestmark = pytest.mark.gpu

GQA4 = synth.ModelSpec("q4-gqa4", 256, 640, 2, 8, 2, 1000, 300, 0, seed=29)


def _pair(spec, gs4=0, gs8=0):
    torch, l2c = need_gpu()
    b = synth.blob(spec)
    dec = l2c.Decoder(spec.cfg, torch.from_numpy(b).cuda(), spec.shared_weights)
    orc = oracle.Model(spec.cfg, b, spec.shared_weights)
    if gs4:
        dec.enable_q40(gs4)
        orc.enable_q40(gs4)
    if gs8:
        dec.enable_q80(gs8)
        orc.enable_q80(gs8)
    return torch, l2c, dec, orc


def _teacher_forced(dec, orc, steps, p0=0, tok=1, q80=False, q40=True):
    for p in range(p0, p0 + steps):
        got = dec.forward(tok, p, q80=q80, q40=q40).cpu().numpy()
        ref = orc.forward(tok, p, q80=q80, q40=q40)
        assert rel_err(got, ref) <= 1e-5, (p, rel_err(got, ref))
        if int(np.argmax(got)) != int(oracle.argmax(ref)):
            assert top2_gap(ref) < TOL_Q80 * np.abs(ref).max(), p
        tok = int(oracle.argmax(ref))
    return tok


def test_q40_15m_teacher_forced():
    torch, l2c, dec, orc = _pair(synth.M15, gs4=32)
    _teacher_forced(dec, orc, 40)
    dec.close()
    orc.close()


@pytest.mark.parametrize("gs", [64, 128])
def test_q40_gqa4_on_a_loaded_cache(gs):
    torch, l2c, dec, orc = _pair(GQA4, gs4=gs)
    k, v = synth.kv_prefill(GQA4, seq=0, n_pos=200)
    dec.kv_load(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    orc.kv_load(k, v)
    _teacher_forced(dec, orc, 12, p0=200, tok=3)
    dec.close()
    orc.close()


def test_q40_generate_matches_oracle_chain():
    torch, l2c, dec, orc = _pair(synth.M15, gs4=32)
    toks = dec.generate(1, 32, q40=True)
    ref_toks, ref_logits = orc.generate(1, 32, q40=True)
    # a differing token is allowed only where the oracle's top two are within rounding
    for t in range(32):
        if toks[t] != ref_toks[t]:
            assert top2_gap(ref_logits[t]) < 1e-5 * np.abs(ref_logits[t]).max(), t
            break
    dec.close()
    orc.close()


def test_q40_with_int8_kv_cache():
    torch, l2c, dec, orc = _pair(GQA4, gs4=64)
    dec.enable_kv8()
    orc.enable_kv8()
    _teacher_forced(dec, orc, 24)
    dec.close()
    orc.close()


def test_q80_and_q40_sets_on_one_handle():
    """Both quantized sets at different group sizes; steps alternate between them
    (each writes its own K/V rows into the one cache, on both sides)."""
    torch, l2c, dec, orc = _pair(GQA4, gs4=128, gs8=32)
    tok = 1
    for p in range(16):
        q4 = p % 2 == 0
        got = dec.forward(tok, p, q80=not q4, q40=q4).cpu().numpy()
        ref = orc.forward(tok, p, q80=not q4, q40=q4)
        assert rel_err(got, ref) <= 1e-5, (p, q4, rel_err(got, ref))
        tok = int(oracle.argmax(ref))
    dec.close()
    orc.close()


def test_q40_refusals():
    torch, l2c, dec, orc = _pair(GQA4)
    with pytest.raises(l2c.L2CError) as e:
        dec.forward(1, 0, q40=True)  # no Q4_0 weights yet
    assert e.value.code == l2c.L2C_E_STATE
    with pytest.raises(l2c.L2CError) as e:
        dec.enable_q40(16)  # 4-bit groups of 32, 64 or 128 only
    assert e.value.code == l2c.L2C_E_ARG
    dec.enable_q40(64)
    dec.enable_q40(64)  # same gs: no-op
    with pytest.raises(l2c.L2CError) as e:
        dec.enable_q40(32)
    assert e.value.code == l2c.L2C_E_STATE
    toks = torch.tensor([1], dtype=torch.int32, device="cuda")
    pos = torch.tensor([0], dtype=torch.int32, device="cuda")
    out = torch.empty(GQA4.vocab_size, device="cuda")
    with pytest.raises(l2c.L2CError) as e:
        dec.forward_batch(toks, pos, out, q80=2)  # the batched step has no Q4_0 form
    assert e.value.code == l2c.L2C_E_ARG
    with pytest.raises(l2c.L2CError) as e:
        dec.prefill(np.array([1, 2], np.int32), 0, q80=2)
    assert e.value.code == l2c.L2C_E_ARG
    with pytest.raises(l2c.L2CError) as e:
        dec.generate(1, 2, q80=3)
    assert e.value.code == l2c.L2C_E_ARG
    # the handle still runs
    orc.enable_q40(64)
    _teacher_forced(dec, orc, 2)
    dec.close()
    orc.close()
