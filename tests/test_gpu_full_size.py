"""Full-size workloads in the launch configuration bench.py times, on outputs the
oracle computes one step at a time: the 7B shape (fp32, Q8_0 GS=64 and Q4_0
GS=64, a cache prefilled to 2048 positions) and the GQA 7B-width batch of 32 sequences (Q8_0
GS=64, ragged positions, 4 sequences sampled for the oracle)."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import TOL_F32, TOL_Q80, need_gpu, rel_err

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _device_blob(torch, spec, host):
    dev = torch.empty(host.size, dtype=torch.float32, device="cuda")
    chunk = 1 << 27
    for s in range(0, host.size, chunk):
        dev[s:s + chunk].copy_(torch.from_numpy(host[s:s + chunk]))
    return dev


def test_7b_step_matches_oracle():
    """The bench's 7B steps: token 1 at positions 0, 512 and 2048 of a cache
    prefilled N(0,1), fp32 and Q8_0 GS=64."""
    torch, l2c = need_gpu()
    spec = synth.L7B
    host = synth.blob(spec)
    dev = _device_blob(torch, spec, host)
    dec = l2c.Decoder(spec.cfg, dev, spec.shared_weights)
    del dev
    torch.cuda.empty_cache()
    dec.enable_q80(64)
    P_MAX = 2048
    k, v = synth.kv_prefill(spec, seq=0, n_pos=P_MAX)
    dec.kv_load(k, v)
    orc = oracle.Model(spec.cfg, host, spec.shared_weights)
    orc.kv_load(k, v)
    del k, v
    for q80 in (False, True):
        if q80:
            orc.enable_q80(64)
        for P in (0, 512, P_MAX):
            # each step writes slot P on both sides, so later steps see the same cache
            got = dec.forward(1, P, q80=q80).cpu().numpy()
            ref = orc.forward(1, P, q80=q80)
            err = rel_err(got, ref)
            assert err <= (TOL_Q80 if q80 else TOL_F32), (q80, P, err)
            if q80:
                assert err <= 1e-5, (P, err)
    # the Q4_0 weights (GS=64) on the same cache
    dec.enable_q40(64)
    orc.enable_q40(64)
    for P in (0, 512, P_MAX):
        got = dec.forward(1, P, q40=True).cpu().numpy()
        ref = orc.forward(1, P, q40=True)
        err = rel_err(got, ref)
        assert err <= 1e-5, ("q40", P, err)
    # the int8 KV cache on both sides: every row in the cache is quantized, then the
    # Q8_0 steps (each writes its slot through the int8 store) keep reproducing the
    # oracle's codes (1e-5)
    dec.enable_kv8()
    orc.enable_kv8()
    for P in (0, 512, P_MAX):
        got = dec.forward(1, P, q80=True).cpu().numpy()
        ref = orc.forward(1, P, q80=True)
        err = rel_err(got, ref)
        assert err <= 1e-5, ("kv8", P, err)
    dec.close()
    orc.close()


def test_gqa_7b_batch32_matches_oracle_on_samples():
    torch, l2c = need_gpu()
    spec = synth.GQA7B
    B = 32
    host = synth.blob(spec)
    dev = _device_blob(torch, spec, host)
    dec = l2c.Decoder(spec.cfg, dev, spec.shared_weights, max_batch=B)
    del dev
    torch.cuda.empty_cache()
    dec.enable_q80(64)
    toks = synth.tokens(spec.seed, 0, B, spec.vocab_size)
    pos = synth.positions(spec.seed, 0, B, spec.seq_len)
    for s in range(B):
        if pos[s]:
            k, v = synth.kv_prefill(spec, seq=s, n_pos=int(pos[s]))
            dec.kv_load(k, v, seq=s)
    out = torch.empty((B, spec.vocab_size), dtype=torch.float32, device="cuda")
    dec.forward_batch(toks, pos, out, q80=True)
    dec.sync()
    got = out.cpu().numpy()
    dec.close()
    orc = oracle.Model(spec.cfg, host, spec.shared_weights, n_seq=1)
    orc.enable_q80(64)
    for s in (0, int(np.argmax(pos)), int(np.argmin(pos)), B - 1):
        orc.kv_reset()
        if pos[s]:
            k, v = synth.kv_prefill(spec, seq=s, n_pos=int(pos[s]))
            orc.kv_load(k, v)
        ref = orc.forward(int(toks[s]), int(pos[s]), q80=True)
        assert rel_err(got[s], ref) <= TOL_Q80, s
        assert rel_err(got[s], ref) <= 1e-5, s
    orc.close()
