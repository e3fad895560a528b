"""The int8 KV cache (l2c_enable_kv8) against the oracle's (orc_enable_kv8).

Reading: every K and V row, when stored, becomes Q8_0 groups of head_size
values (one group per KV head, the quantize() rule of "超精简LLM部署" §1
INT8量化压缩), and attention reads code * scale.  The Q8_0 step reproduces the
oracle's K/V rows exactly, so its int8 codes and logits match to 1e-5; the
cache serves the Q8_0 step only (the fp32 step's rows match the oracle's to
fp32 rounding, so a code could flip at a rounding tie; at these random-weight
shapes one flip moves the logits by about 1%).  Cases: the 15M shape (Q8_0
GS=32), 48 teacher-forced steps and the on-device greedy loop; a GQA ratio 4
shape whose loaded rows are quantized by enabling the cache; reset; the entry
points that refuse to run with the cache on.  The 7B shape
at positions 0, 512 and 2048 is in test_gpu_full_size.py.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import TOL_Q80, need_gpu, rel_err, top2_gap

pytestmark = pytest.mark.gpu

GQA4 = synth.ModelSpec("kv8-gqa4", 256, 640, 2, 8, 2, 1000, 300, 0, seed=23)


def _pair(spec, gs=0):
    torch, l2c = need_gpu()
    b = synth.blob(spec)
    dec = l2c.Decoder(spec.cfg, torch.from_numpy(b).cuda(), spec.shared_weights)
    orc = oracle.Model(spec.cfg, b, spec.shared_weights)
    if gs:
        dec.enable_q80(gs)
        orc.enable_q80(gs)
    return torch, l2c, dec, orc


def _teacher_forced(dec, orc, steps, q80, tol, p0=0, tok=1):
    for p in range(p0, p0 + steps):
        got = dec.forward(tok, p, q80=q80).cpu().numpy()
        ref = orc.forward(tok, p, q80=q80)
        assert rel_err(got, ref) <= tol, (p, rel_err(got, ref))
        if int(np.argmax(got)) != int(oracle.argmax(ref)):
            assert top2_gap(ref) < TOL_Q80 * np.abs(ref).max(), p
        tok = int(oracle.argmax(ref))


def test_kv8_15m_q80_48_steps():
    torch, l2c, dec, orc = _pair(synth.M15, 32)
    dec.enable_kv8()
    orc.enable_kv8()
    _teacher_forced(dec, orc, 48, True, 1e-5)
    dec.sync()
    dec.close()
    orc.close()


def test_kv8_gqa4_q80_quantizes_loaded_rows():
    torch, l2c, dec, orc = _pair(GQA4, 32)
    k, v = synth.kv_prefill(GQA4, seq=0, n_pos=40)
    dec.kv_load(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    orc.kv_load(k, v)
    dec.enable_kv8()
    orc.enable_kv8()
    # the fp32 cache now holds code * scale, as the oracle's
    kd, vd = dec.kv_read(40)
    kr, vr = orc.kv_read(40)
    assert np.array_equal(kd, kr) and np.array_equal(vd, vr)
    _teacher_forced(dec, orc, 24, True, 1e-5, p0=40, tok=5)
    # rows loaded while the cache is on are quantized as well
    k2, v2 = synth.kv_prefill(GQA4, seq=0, n_pos=70, seed=99)
    dec.kv_load(torch.from_numpy(k2).cuda(), torch.from_numpy(v2).cuda())
    orc.kv_load(k2, v2)
    _teacher_forced(dec, orc, 8, True, 1e-5, p0=70, tok=9)
    dec.close()
    orc.close()


def test_kv8_15m_generate_and_refused_fp32_step():
    """The on-device greedy loop with the int8 cache against the oracle's chain (15M,
    GS=32), and the fp32 step, which the cache does not serve."""
    torch, l2c, dec, orc = _pair(synth.M15, 32)
    dec.enable_kv8()
    orc.enable_kv8()
    toks = dec.generate(1, 32, q80=True)
    ref_toks, ref_logits = orc.generate(1, 32, q80=True)
    mism = np.nonzero(toks != ref_toks)[0]
    if mism.size:
        t = int(mism[0])
        assert top2_gap(ref_logits[t]) < TOL_Q80 * np.abs(ref_logits[t]).max(), t
    with pytest.raises(l2c.L2CError) as e:
        dec.forward(1, 40)
    assert e.value.code == l2c.L2C_E_STATE
    with pytest.raises(l2c.L2CError) as e:
        dec.generate(1, 2, q80=False)
    assert e.value.code == l2c.L2C_E_STATE
    dec.close()
    orc.close()


def test_kv8_reset_and_refused_entry_points():
    torch, l2c, dec, orc = _pair(GQA4, 32)
    dec.enable_kv8()
    orc.enable_kv8()
    _teacher_forced(dec, orc, 6, True, 1e-5)
    dec.kv_reset()
    orc.kv_reset()
    _teacher_forced(dec, orc, 3, True, 1e-5)
    out = torch.empty((1, GQA4.vocab_size), dtype=torch.float32, device="cuda")
    with pytest.raises(l2c.L2CError) as e:
        dec.forward_batch(np.zeros(1, np.int32), np.zeros(1, np.int32), out)
    assert e.value.code == l2c.L2C_E_STATE
    with pytest.raises(l2c.L2CError) as e:
        dec.prefill(np.zeros(4, np.int32), 0, q80=True)
    assert e.value.code == l2c.L2C_E_STATE
    dec.enable_kv8(False)  # back to the fp32 cache: the batched step runs again
    dec.forward_batch(np.zeros(1, np.int32), np.zeros(1, np.int32), out)
    dec.sync()
    dec.close()
    orc.close()
