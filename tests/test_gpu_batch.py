"""The batched step (l2c_forward_batch): B independent sequences, each at its own
position with its own prefilled KV cache, against the oracle run one sequence at
a time.  Q8_0 runs the tensor-core skinny GEMM; fp32 runs the single-sequence
kernels per sequence."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import TOL_F32, need_gpu, rel_err

pytestmark = pytest.mark.gpu

# GQA ratio 4, head_size 32, widths that tile the batched GEMM at gs = 32
BSPEC = synth.ModelSpec("batch-small", 256, 640, 2, 8, 2, 1000, 300, 0, seed=13)


@pytest.fixture(scope="module")
def pair():
    torch, l2c = need_gpu()
    spec = BSPEC
    B = 7
    b = synth.blob(spec)
    dec = l2c.Decoder(spec.cfg, torch.from_numpy(b).cuda(), spec.shared_weights, max_batch=B)
    dec.enable_q80(32)
    orc = oracle.Model(spec.cfg, b, spec.shared_weights, n_seq=B)
    orc.enable_q80(32)
    yield torch, l2c, dec, orc, B
    dec.close()


def _prefill(dec, orc, torch, pos):
    for s, p in enumerate(pos):
        if p:
            k, v = synth.kv_prefill(BSPEC, seq=s, n_pos=int(p))
            dec.kv_load(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(), seq=s)
            orc.kv_load(k, v, seq=s)


@pytest.mark.parametrize("q80", [True, False], ids=["q80", "fp32"])
def test_batch_matches_oracle_per_sequence(pair, q80):
    torch, l2c, dec, orc, B = pair
    spec = BSPEC
    toks = synth.tokens(spec.seed, 30 + q80, B, spec.vocab_size)
    pos = synth.positions(spec.seed, 30 + q80, B, spec.seq_len)
    pos[0], pos[1] = 0, spec.seq_len - 1          # both ends of the cache
    _prefill(dec, orc, torch, pos)
    out = torch.empty((B, spec.vocab_size), dtype=torch.float32, device="cuda")
    dec.forward_batch(toks, pos, out, q80=q80)
    dec.sync()
    got = out.cpu().numpy()
    tol = 1e-5 if q80 else TOL_F32
    for s in range(B):
        ref = orc.forward(int(toks[s]), int(pos[s]), q80=q80, seq=s)
        assert rel_err(got[s], ref) <= tol, (s, pos[s])
        k, v = dec.kv_read(int(pos[s]) + 1, seq=s)
        kr, vr = orc.kv_read(int(pos[s]) + 1, seq=s)
        assert rel_err(k[:, -1], kr[:, -1]) <= tol and rel_err(v[:, -1], vr[:, -1]) <= tol


def test_batch_sizes_and_device_arrays(pair):
    """Smaller batches reuse the handle (a graph per size); tokens/positions may live on the device."""
    torch, l2c, dec, orc, B = pair
    spec = BSPEC
    for nb in (1, 3):
        toks = synth.tokens(spec.seed, 40 + nb, nb, spec.vocab_size)
        pos = synth.positions(spec.seed, 40 + nb, nb, spec.seq_len)
        _prefill(dec, orc, torch, pos)
        out = torch.empty((nb, spec.vocab_size), dtype=torch.float32, device="cuda")
        dec.forward_batch(torch.from_numpy(toks).cuda(), torch.from_numpy(pos).cuda(), out, q80=True)
        dec.sync()
        got = out.cpu().numpy()
        for s in range(nb):
            ref = orc.forward(int(toks[s]), int(pos[s]), q80=True, seq=s)
            assert rel_err(got[s], ref) <= 1e-5


def test_batch_rejects_bad_arguments(pair):
    torch, l2c, dec, orc, B = pair
    spec = BSPEC
    out = torch.empty((B + 1, spec.vocab_size), dtype=torch.float32, device="cuda")
    with pytest.raises(l2c.L2CError):
        dec.forward_batch(np.zeros(B + 1, np.int32), np.zeros(B + 1, np.int32), out)
    with pytest.raises(l2c.L2CError):
        dec.forward_batch(np.array([spec.vocab_size], np.int32), np.zeros(1, np.int32), out)
    with pytest.raises(l2c.L2CError):
        dec.forward_batch(np.zeros(1, np.int32), np.array([spec.seq_len], np.int32), out)
