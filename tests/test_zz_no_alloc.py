"""l2c_attention_noalloc: attention for callers that cannot allocate device memory.

Such callers (a process whose GPU memory belongs to another allocator's pool,
or a latency-critical path where cudaMalloc may synchronize the device) pass
their own input and output buffers; the entry point keeps its scratch in a
fixed array inside the library and allocates nothing.  Each test checks it,
through the C ABI, against l2c_attention (the handle-based entry point that
runs the same kernel with allocated scratch), on two calls in a row.

The file name makes pytest collect it last, so a run that stops at the first
failure has already run every other test; it also passes alone in a fresh
process.
"""
import ctypes

import numpy as np
import pytest

import synth
from gpu_util import need_gpu

pytestmark = pytest.mark.gpu

SHAPES = [  # (n_heads, n_kv_heads, head_size, seq_len, pos)
    (32, 32, 128, 4096, 4095),   # 7B shape, last position
    (32, 8, 128, 2048, 1300),    # GQA 7B-width shape
    (8, 4, 8, 512, 77),          # tiny shape
]


def _noalloc(l2c, q, k, v, H, Hkv, hs, pos, precision, out, stream):
    return l2c.lib().l2c_attention_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), H, Hkv, hs, pos, precision,
                                           out.data_ptr(), ctypes.c_void_p(stream))


@pytest.mark.parametrize("H,Hkv,hs,S,pos", SHAPES, ids=["7B", "GQA-7B", "tiny"])
@pytest.mark.parametrize("precision,tol", [(0, 2e-6), (1, 1e-7)], ids=["fp32", "double"])
def test_noalloc_matches_handle_attention(H, Hkv, hs, S, pos, precision, tol):
    torch, l2c = need_gpu()
    d = H * hs
    spec = synth.ModelSpec("attn", d, 4 * d, 1, H, Hkv, 64, S, 1, seed=5)
    dec = l2c.Decoder(spec.cfg, synth.blob(spec), 1)
    k, v = synth.kv_prefill(spec, seq=0, n_pos=pos + 1)
    kd, vd = torch.from_numpy(k[0]).cuda(), torch.from_numpy(v[0]).cuda()
    stream = torch.cuda.current_stream().cuda_stream
    rng = np.random.default_rng(pos)
    for call in range(2):  # the second call sees the scratch the first one left
        q = torch.from_numpy(rng.standard_normal(d).astype(np.float32)).cuda()
        ref = torch.empty(d, dtype=torch.float32, device="cuda")
        got = torch.full((d,), float("nan"), dtype=torch.float32, device="cuda")
        dec.attention(q, kd, vd, pos, ref, precision)
        dec.sync()
        rc = _noalloc(l2c, q, kd, vd, H, Hkv, hs, pos, precision, got, stream)
        assert rc == l2c.L2C_OK, rc
        torch.cuda.synchronize()
        r, g = ref.cpu().numpy(), got.cpu().numpy()
        assert np.all(np.isfinite(g)), call
        assert np.abs(g - r).max() <= tol * np.abs(r).max(), call
    dec.close()


def test_noalloc_rejects_oversized_and_bad_shapes():
    torch, l2c = need_gpu()
    t = torch.zeros(16, dtype=torch.float32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    # 32 KV heads of 128 at 10000 positions in double need about 5.2 MB of scratch
    assert _noalloc(l2c, t, t, t, 32, 32, 128, 10000, 1, t, s) == l2c.L2C_E_SCRATCH
    assert _noalloc(l2c, t, t, t, 32, 5, 128, 10, 0, t, s) == l2c.L2C_E_ARG    # heads not a multiple
    assert _noalloc(l2c, t, t, t, 4, 4, 200, 10, 0, t, s) == l2c.L2C_E_ARG     # head size not built
    assert _noalloc(l2c, t, t, t, 4, 4, 64, -1, 0, t, s) == l2c.L2C_E_ARG      # negative position
    assert _noalloc(l2c, t, t, t, 4, 4, 64, 10, 2, t, s) == l2c.L2C_E_ARG      # unknown precision
    torch.cuda.synchronize()
