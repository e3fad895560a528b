"""Kernel-level parity through the C ABI: Q8_0 quantize and int32 group dots must be
bit-exact with the oracle; argmax must return the first index of the maximum."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    torch, l2c = need_gpu()
    spec = synth.TINY
    b = synth.blob(spec)
    dec = l2c.Decoder(spec.cfg, b, spec.shared_weights)
    yield torch, l2c, dec
    dec.close()


def _quant_inputs(n, gs, seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal(n) * rng.uniform(1e-3, 10.0, n // gs).repeat(gs)).astype(np.float32)
    x[:gs] = 0.0                                        # an all-zero group
    x[gs:2 * gs] = np.float32(1.5) * np.arange(gs)       # exact values on .5 ties after scaling
    x[2 * gs] = np.float32(-127.0)
    return x


@pytest.mark.parametrize("gs,n", [(32, 288 * 37), (64, 4096 * 9), (64, 11008 * 3), (16, 1600), (128, 128 * 50)])
def test_quantize_bitexact(env, gs, n):
    torch, l2c, dec = env
    x = _quant_inputs(n, gs, gs + n)
    q_ref, s_ref = oracle.quantize(x, gs)
    xd = torch.from_numpy(x).cuda()
    q = torch.empty(n, dtype=torch.int8, device="cuda")
    s = torch.empty(n // gs, dtype=torch.float32, device="cuda")
    dec.quantize_q80(xd, gs, q, s)
    dec.sync()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def test_quantize_weight_blob_bitexact(env):
    # the 15M-shape embedding table: 9.2M seeded N(0, 0.02) weights, GS = 32
    torch, l2c, dec = env
    spec = synth.M15
    E = np.empty(spec.vocab_size * spec.dim, np.float32)
    synth.blob_into(spec, E)
    q_ref, s_ref = oracle.quantize(E, 32)
    q = torch.empty(E.size, dtype=torch.int8, device="cuda")
    s = torch.empty(E.size // 32, dtype=torch.float32, device="cuda")
    dec.quantize_q80(torch.from_numpy(E).cuda(), 32, q, s)
    dec.sync()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy(), s_ref)


# K % 64 == 0 with gs 32 / 64 / 128 runs the Q8_0 matvec's own 64-byte chunk
# routine (the 7B widths 4096 and 11008 among them); the others the 16-byte loop.
@pytest.mark.parametrize("rows,K,gs", [(7, 288, 32), (33, 4096, 64), (5, 11008, 64), (3, 768, 64), (9, 256, 128),
                                       (6, 4096, 32), (4, 11008, 32), (5, 4096, 128), (3, 11008, 128),
                                       (4, 160, 32), (3, 96, 16)])
def test_group_dots_bitexact(env, rows, K, gs):
    torch, l2c, dec = env
    rng = np.random.default_rng(rows * K + gs)
    qw = rng.integers(-127, 128, (rows, K)).astype(np.int8)
    qx = rng.integers(-127, 128, K).astype(np.int8)
    # extreme groups: +-127 everywhere gives |dot| = gs * 127^2 (both signs)
    qw[0, :] = -127
    qx[:gs] = -127
    qx[gs:2 * gs] = 127
    if rows > 1:
        qw[1, :] = 127
    ref = oracle.q80_group_dots(qw, qx, gs)
    assert ref[0, 0] == gs * 127 * 127 and ref[0, 1] == -gs * 127 * 127
    out = torch.empty((rows, K // gs), dtype=torch.int32, device="cuda")
    dec.q80_group_dots(torch.from_numpy(qw).cuda(), torch.from_numpy(qx).cuda(), gs, out)
    dec.sync()
    assert np.array_equal(out.cpu().numpy(), ref)


def test_argmax_first_index(env):
    torch, l2c, dec = env
    rng = np.random.default_rng(5)
    for n in (1, 31, 32000, 100_003):
        x = rng.standard_normal(n).astype(np.float32)
        if n > 10:
            x[n // 3] = x[n // 2] = x[-1] = x.max() + 1.0  # three-way tie
        assert dec.argmax(torch.from_numpy(x).cuda()) == oracle.argmax(x)
    neg = -np.abs(rng.standard_normal(500)).astype(np.float32) - 1
    assert dec.argmax(torch.from_numpy(neg).cuda()) == oracle.argmax(neg)


def test_argmax_nan_is_reported(env):
    torch, l2c, dec = env
    x = np.zeros(100, np.float32)
    x[7] = np.nan
    with pytest.raises(l2c.L2CError) as e:
        dec.argmax(torch.from_numpy(x).cuda())
    assert e.value.code == l2c.L2C_E_DEVICE


ATTN_SHAPES = [  # (n_heads, n_kv_heads, head_size, seq_len, positions)
    (32, 32, 128, 4096, (0, 63, 64, 1000, 4095)),   # 7B shape
    (32, 8, 128, 2048, (0, 130, 2047)),             # GQA-7B shape
    (8, 4, 8, 512, (0, 5, 511)),                     # tiny shape
    (6, 6, 48, 256, (0, 200, 255)),                  # 15M shape
]


@pytest.mark.parametrize("H,Hkv,hs,S,positions", ATTN_SHAPES, ids=["7B", "GQA-7B", "tiny", "15M"])
def test_attention_matches_oracle(H, Hkv, hs, S, positions):
    torch, l2c = need_gpu()
    d = H * hs
    spec = synth.ModelSpec("attn", d, 4 * d, 1, H, Hkv, 64, S, 1, seed=3)
    dec = l2c.Decoder(spec.cfg, synth.blob(spec), 1)
    rng = np.random.default_rng(H * S)
    kvd = Hkv * hs
    kc, vc = synth.kv_prefill(spec, seq=0, n_pos=S)
    kc, vc = kc[0], vc[0]
    kd, vd = torch.from_numpy(kc).cuda(), torch.from_numpy(vc).cuda()
    for pos in positions:
        q = rng.standard_normal(d).astype(np.float32)
        ref = oracle.attention(q, kc, vc, pos, H, Hkv)
        for precision, tol in ((0, 2e-6), (1, 1e-7)):
            out = torch.empty(d, dtype=torch.float32, device="cuda")
            dec.attention(torch.from_numpy(q).cuda(), kd, vd, pos, out, precision)
            dec.sync()
            got = out.cpu().numpy()
            assert np.abs(got - ref).max() <= tol * np.abs(ref).max(), (pos, precision)
    dec.close()


@pytest.mark.parametrize("precision", [0, 1], ids=["fp32", "double"])
@pytest.mark.parametrize("where,value", [("k", np.inf), ("k", np.nan), ("v", np.nan), ("v", np.inf)])
def test_attention_nonfinite_kv_is_not_finite(precision, where, value):
    """A non-finite K or V element at a position the query reaches leaves the heads of
    its KV head non-finite (the double path detects it: its integer widening alone
    would turn it into a large finite value) and every other head finite."""
    torch, l2c = need_gpu()
    H, Hkv, hs, S, pos = 8, 4, 16, 300, 250
    d = H * hs
    spec = synth.ModelSpec("attn-nf", d, 4 * d, 1, H, Hkv, 64, S, 1, seed=9)
    dec = l2c.Decoder(spec.cfg, synth.blob(spec), 1)
    kc, vc = synth.kv_prefill(spec, seq=0, n_pos=S)
    kc, vc = kc[0].copy(), vc[0].copy()
    g = 2  # KV head hit: query heads 4 and 5
    (kc if where == "k" else vc)[137, g * hs + 5] = value
    q = np.random.default_rng(1).standard_normal(d).astype(np.float32)
    rep = H // Hkv
    for h in range(g * rep, (g + 1) * rep):
        q[h * hs + 5] = 1.0  # an infinite key then scores +inf in both heads
    out = torch.empty(d, dtype=torch.float32, device="cuda")
    dec.attention(torch.from_numpy(q).cuda(), torch.from_numpy(kc).cuda(), torch.from_numpy(vc).cuda(), pos, out,
                  precision)
    dec.sync()
    got = out.cpu().numpy().reshape(H, hs)
    for h in range(H):
        if h // rep == g:
            assert not np.isfinite(got[h]).all(), h
        else:
            assert np.isfinite(got[h]).all(), h
    dec.close()
