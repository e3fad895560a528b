"""Step-level parity of the GPU decode step with the oracle, through the C ABI.

fp32: max |logit - oracle| <= 1e-4 * max |oracle logit|.  Q8_0: <= 2e-3 (the
step reproduces the oracle's activation codes, so the observed gap is far
smaller).  Greedy sequences must match except where the oracle's top-2 gap is
below the tolerance.  Inputs are the seeded workloads and odd shapes with
ragged tails (hidden 172, head_size 8 and 48, GQA ratios 2 and 3)."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import TOL_F32, TOL_Q80, need_gpu, rel_err, top2_gap

pytestmark = pytest.mark.gpu

ODD = synth.ModelSpec("odd", 48, 100, 2, 6, 2, 50, 160, 0, seed=10, wsigma=0.2, nsigma=0.1)
ODDQ = synth.ModelSpec("oddq", 96, 160, 3, 6, 3, 300, 200, 0, seed=11, wsigma=0.1, nsigma=0.1)
GQA_SMALL = synth.ModelSpec("gqa-small", 256, 688, 2, 8, 2, 1000, 300, 0, seed=12)
# widths that are multiples of 64: the Q8_0 GEMV's 64-bytes-per-lane path
Q64 = synth.ModelSpec("q64", 256, 768, 2, 4, 2, 700, 200, 0, seed=14)


@pytest.fixture(scope="module")
def gpu():
    return need_gpu()


def _pair(gpu, spec, gs=0, max_batch=1):
    torch, l2c = gpu
    b = synth.blob(spec)
    dec = l2c.Decoder(spec.cfg, torch.from_numpy(b).cuda(), spec.shared_weights, max_batch=max_batch)
    orc = oracle.Model(spec.cfg, b, spec.shared_weights)
    if gs:
        dec.enable_q80(gs)
        orc.enable_q80(gs)
    return dec, orc


def _forced(gpu, spec, steps, gs=0, tok_sub=21):
    """Teacher-forced decode of `steps` seeded tokens; returns per-step relative errors."""
    dec, orc = _pair(gpu, spec, gs)
    toks = synth.tokens(spec.seed, tok_sub, steps, spec.vocab_size)
    errs = []
    for p, t in enumerate(toks):
        got = dec.forward(int(t), p, q80=bool(gs)).cpu().numpy()
        ref = orc.forward(int(t), p, q80=bool(gs))
        errs.append(rel_err(got, ref))
    dec.sync()
    dec.close()
    return np.array(errs)


@pytest.mark.parametrize("spec,steps", [(synth.TINY, 80), (ODD, 70), (GQA_SMALL, 70), (synth.M15, 40)],
                         ids=["tiny", "odd", "gqa-small", "15M"])
def test_fp32_teacher_forced(gpu, spec, steps):
    errs = _forced(gpu, spec, steps)
    assert errs.max() <= TOL_F32, errs


@pytest.mark.parametrize("spec,gs,steps", [(synth.M15, 32, 40), (ODDQ, 32, 70), (GQA_SMALL, 16, 70),
                                           (Q64, 32, 70), (Q64, 64, 70), (Q64, 128, 70)],
                         ids=["15M-gs32", "oddq-gs32", "gqa-small-gs16", "q64-gs32", "q64-gs64", "q64-gs128"])
def test_q80_teacher_forced(gpu, spec, gs, steps):
    errs = _forced(gpu, spec, steps, gs)
    assert errs.max() <= TOL_Q80, errs
    # identical activation codes leave only double-rounding noise
    assert errs.max() <= 1e-5, errs


def test_kv_cache_slots(gpu):
    spec = GQA_SMALL
    for gs in (0, 16):
        dec, orc = _pair(gpu, spec, gs)
        toks = synth.tokens(spec.seed, 3, 67, spec.vocab_size)
        for p, t in enumerate(toks):
            dec.forward(int(t), p, q80=bool(gs))
            orc.forward(int(t), p, q80=bool(gs))
        k, v = dec.kv_read(67)
        kr, vr = orc.kv_read(67)
        tol = 1e-5 if not gs else 1e-6
        assert rel_err(k, kr) <= tol and rel_err(v, vr) <= tol
        k2, _ = dec.kv_read(spec.seq_len)
        assert np.all(k2[:, 67:] == 0)  # nothing written beyond the decoded positions
        dec.close()


def test_prefilled_cache_chunks(gpu):
    """A step at positions that span several attention chunks, on a cache prefilled with N(0,1)."""
    torch, l2c = gpu
    spec = GQA_SMALL
    for gs in (0, 16):
        dec, orc = _pair(gpu, spec, gs)
        for P in (1, 63, 64, 65, 130, 299):
            k, v = synth.kv_prefill(spec, seq=0, n_pos=P)
            dec.kv_load(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
            orc.kv_load(k, v)
            got = dec.forward(17, P, q80=bool(gs)).cpu().numpy()
            ref = orc.forward(17, P, q80=bool(gs))
            assert rel_err(got, ref) <= (TOL_F32 if not gs else 1e-5), (gs, P)
        dec.close()


def test_bad_arguments(gpu):
    torch, l2c = gpu
    spec = synth.TINY
    dec, orc = _pair(gpu, spec)
    for tok, pos in ((-1, 0), (spec.vocab_size, 0), (0, -1), (0, spec.seq_len)):
        with pytest.raises(l2c.L2CError):
            dec.forward(tok, pos)
    with pytest.raises(l2c.L2CError) as e:
        dec.forward(1, 0, q80=True)
    assert e.value.code == l2c.L2C_E_STATE
    with pytest.raises(l2c.L2CError):
        dec.enable_q80(24)  # not a multiple of 16
    with pytest.raises(l2c.L2CError):
        dec.generate(1, spec.seq_len + 1)
    dec.sync()
    dec.close()
