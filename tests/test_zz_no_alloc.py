"""l2c_attention_noalloc: attention for callers that cannot allocate device memory.

Such callers (a process whose GPU memory belongs to another allocator's pool,
or a latency-critical path where cudaMalloc may synchronize the device) pass
their own input and output buffers; the entry point keeps its scratch in a
fixed array inside the library and allocates nothing.  The tests call it
through the C ABI on two calls in a row (the second sees the scratch the first
left) and check it against the CPU oracle's attention and against
l2c_attention (the handle-based entry point that runs the same kernel with
allocated scratch and its own position split); that repeated calls leave the
device's free memory unchanged; and, in a child process, that a device reset
between calls (which loads the library's module, and its array, anew) is
handled.

The file name makes pytest collect it last, so a run that stops at the first
failure has already run every other test; it also passes alone in a fresh
process.
"""
import ctypes
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest

import oracle
import synth
from gpu_util import need_gpu

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SHAPES = [  # (n_heads, n_kv_heads, head_size, seq_len, pos)
    (32, 32, 128, 4096, 4095),   # 7B shape, last position
    (32, 8, 128, 2048, 1300),    # GQA 7B-width shape
    (8, 4, 8, 512, 77),          # tiny shape
]
TOL = {0: 2e-6, 1: 1e-7}  # max |got - ref| / max |ref|, as the attention kernel tests


def _noalloc(l2c, q, k, v, H, Hkv, hs, pos, precision, out, stream):
    return l2c.lib().l2c_attention_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), H, Hkv, hs, pos, precision,
                                           out.data_ptr(), ctypes.c_void_p(stream))


@pytest.mark.parametrize("H,Hkv,hs,S,pos", SHAPES, ids=["7B", "GQA-7B", "tiny"])
@pytest.mark.parametrize("precision", [0, 1], ids=["fp32", "double"])
def test_noalloc_matches_oracle_and_handle(H, Hkv, hs, S, pos, precision):
    torch, l2c = need_gpu()
    d = H * hs
    spec = synth.ModelSpec("attn", d, 4 * d, 1, H, Hkv, 64, S, 1, seed=5)
    dec = l2c.Decoder(spec.cfg, synth.blob(spec), 1)
    k, v = synth.kv_prefill(spec, seq=0, n_pos=pos + 1)
    kd, vd = torch.from_numpy(k[0]).cuda(), torch.from_numpy(v[0]).cuda()
    stream = torch.cuda.current_stream().cuda_stream
    rng = np.random.default_rng(pos)
    tol = TOL[precision]
    for call in range(2):  # the second call sees the scratch the first one left
        qh = rng.standard_normal(d).astype(np.float32)
        q = torch.from_numpy(qh).cuda()
        ref = oracle.attention(qh, k[0], v[0], pos, H, Hkv)
        handle = torch.empty(d, dtype=torch.float32, device="cuda")
        got = torch.full((d,), float("nan"), dtype=torch.float32, device="cuda")
        dec.attention(q, kd, vd, pos, handle, precision)
        dec.sync()
        rc = _noalloc(l2c, q, kd, vd, H, Hkv, hs, pos, precision, got, stream)
        assert rc == l2c.L2C_OK, rc
        torch.cuda.synchronize()
        g, hh = got.cpu().numpy(), handle.cpu().numpy()
        assert np.all(np.isfinite(g)), call
        scale = np.abs(ref).max()
        assert np.abs(g - ref).max() <= tol * scale, (call, np.abs(g - ref).max() / scale)
        assert np.abs(g - hh).max() <= 2 * tol * scale, call
    dec.close()


def test_noalloc_allocates_nothing():
    torch, l2c = need_gpu()
    H, Hkv, hs, pos = 32, 8, 128, 2047
    d, kvd = H * hs, Hkv * hs
    g = torch.Generator(device="cuda").manual_seed(0)
    q = torch.randn(d, device="cuda", generator=g)
    k = torch.randn(pos + 1, kvd, device="cuda", generator=g)
    v = torch.randn(pos + 1, kvd, device="cuda", generator=g)
    out = torch.empty(d, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    for precision in (0, 1):  # first calls: set-up and lazy module loading
        assert _noalloc(l2c, q, k, v, H, Hkv, hs, pos, precision, out, s) == l2c.L2C_OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for i in range(6):
        assert _noalloc(l2c, q, k, v, H, Hkv, hs, pos, i % 2, out, s) == l2c.L2C_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)


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
    u = t[1:]  # 4-byte offset: not 16-byte aligned
    assert l2c.lib().l2c_attention_noalloc(u.data_ptr(), t.data_ptr(), t.data_ptr(), 4, 4, 8, 1, 0, t.data_ptr(),
                                           ctypes.c_void_p(s)) == l2c.L2C_E_ARG
    torch.cuda.synchronize()


_CHILD = textwrap.dedent("""
    import ctypes, sys
    import numpy as np
    sys.path.insert(0, ROOT)
    sys.path.insert(0, ROOT + "/tests")
    import decode_llama_step_02_b200 as l2c
    import oracle
    L = l2c.lib()
    rt = ctypes.CDLL("libcudart.so.12")   # the runtime the library uses
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    rt.cudaMalloc.argtypes = [ctypes.POINTER(vp), sz]
    rt.cudaMemcpy.argtypes = [vp, vp, sz, ctypes.c_int]
    rt.cudaFree.argtypes = [vp]
    H, Hkv, hs, pos = 8, 4, 16, 200
    rng = np.random.default_rng(1)
    q = rng.standard_normal(H * hs).astype(np.float32)
    k = rng.standard_normal((pos + 1, Hkv * hs)).astype(np.float32)
    v = rng.standard_normal((pos + 1, Hkv * hs)).astype(np.float32)

    def up(a):
        p = vp()
        assert rt.cudaMalloc(ctypes.byref(p), a.nbytes) == 0
        assert rt.cudaMemcpy(p, a.ctypes.data, a.nbytes, 1) == 0
        return p

    def run(precision):
        dq, dk, dv = up(q), up(k), up(v)
        out = np.full(H * hs, np.nan, np.float32)
        do = up(out)
        rc = L.l2c_attention_noalloc(dq, dk, dv, H, Hkv, hs, pos, precision, do, None)
        assert rc == 0, rc
        assert rt.cudaDeviceSynchronize() == 0
        assert rt.cudaMemcpy(out.ctypes.data, do, out.nbytes, 2) == 0
        for p in (dq, dk, dv, do):
            rt.cudaFree(p)
        return out

    ref = oracle.attention(q, k, v, pos, H, Hkv)
    for precision, tol in ((0, 2e-6), (1, 1e-7)):
        a = run(precision)
        assert rt.cudaDeviceReset() == 0
        b = run(precision)
        assert np.array_equal(a, b), precision
        assert np.abs(b - ref).max() <= tol * np.abs(ref).max(), precision
    print("child ok")
""")


def test_noalloc_survives_device_reset():
    need_gpu()
    code = "ROOT = %r\n" % ROOT + _CHILD
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "child ok" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]
