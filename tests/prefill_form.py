"""An independent formulation of the Llama-2 forward for the oracle's pins.

The whole sequence at once, in float64 NumPy: causal-masked attention over a
[T x T] score matrix, RoPE as a complex multiply by a precomputed table of
e^{i pos freq} (the PyTorch "freqs_cis" form the karpathy-notes Q&A page
contrasts with llama2.c's on-the-fly cosf/sinf), grouped-query attention as
multi-head attention over K/V repeated per query head, and Q8_0 matvecs as
matrix products of dequantized operands (Q4_0 weights the same way, their inputs
Q8_0).  Row t of its logits must equal the
decode step at position t fed the same tokens.

Values are float64 between the points where the decode step stores fp32
(after each matvec, RoPE, attention, residual add, RMSNorm and SwiGLU); there
they are rounded to float32 too, so that a Q8_0 code is decided on the same
fp32 value in both formulations.
"""
import numpy as np


def unpack(cfg, blob, shared):
    d, h, L, H, Hkv, V, S = cfg
    hs = d // H
    kvd = Hkv * hs
    sizes = [("E", (V, d)), ("w_att", (L, d)), ("wq", (L, d, d)), ("wk", (L, kvd, d)),
             ("wv", (L, kvd, d)), ("wo", (L, d, d)), ("w_ffn", (L, d)), ("w1", (L, h, d)),
             ("w2", (L, d, h)), ("w3", (L, h, d)), ("w_final", (d,)), ("freq", (S * hs,))]
    if not shared:
        sizes.append(("wcls", (V, d)))
    out, off = {}, 0
    for name, shp in sizes:
        n = int(np.prod(shp))
        out[name] = blob[off:off + n].reshape(shp).astype(np.float64)
        off += n
    assert off == blob.size
    if shared:
        out["wcls"] = out["E"]
    return out


def f32(X):
    return np.asarray(X, np.float64).astype(np.float32).astype(np.float64)


def _rms(X, w):
    return f32(X / np.sqrt((X * X).mean(-1, keepdims=True) + 1e-5) * w)


def _q8_fake(M, gs, quantize):
    """Dequantized Q8_0 copy of M (rows of a multiple of gs), via the given quantize."""
    q, s = quantize(M.astype(np.float32).ravel(), gs)
    return (q.astype(np.float64) * np.repeat(s.astype(np.float64), gs)).reshape(M.shape)


def _kv8(M, hs, quantize):
    """K or V rows [T][kvd] as an int8 KV cache keeps them: Q8_0 groups of one head
    (hs values), code * scale rounded to fp32."""
    q, s = quantize(M.astype(np.float32).ravel(), hs)
    return f32(q.astype(np.float64) * np.repeat(s.astype(np.float64), hs)).reshape(M.shape)


def prefill_logits(cfg, blob, shared, tokens, q80_gs=0, quantize=None, kv8=False, wquantize=None):
    """Logits [T][V].  q80_gs: quantized weights and matvec inputs at that group size,
    the inputs (and the int8 KV rows) through `quantize`, the weights and the embedding
    table through `wquantize` (default: `quantize`; the Q4_0 weights pass their own)."""
    wquantize = wquantize or quantize
    d, h, L, H, Hkv, V, S = cfg
    hs = d // H
    rep = H // Hkv
    W = unpack(cfg, blob, shared)
    T = len(tokens)
    freqs = np.array([np.float32(10000.0 ** (-j / hs)) for j in range(0, hs, 2)], np.float32)
    theta = np.outer(np.arange(T, dtype=np.float32), freqs).astype(np.float32).astype(np.float64)
    cis = np.exp(1j * theta)  # [T][hs/2]

    def rope(X, nh):  # X [T][nh*hs]
        Z = X[:, 0::2] + 1j * X[:, 1::2]
        Z = Z.reshape(T, nh, hs // 2) * cis[:, None, :]
        out = np.empty_like(X)
        out[:, 0::2] = Z.real.reshape(T, -1)
        out[:, 1::2] = Z.imag.reshape(T, -1)
        return f32(out)

    def mm(Xin, M):
        """Rows of Xin times M^T; through Q8_0 when q80_gs is set."""
        if not q80_gs:
            return f32(Xin @ M.T)
        Xq = np.stack([_q8_fake(r, q80_gs, quantize) for r in Xin.astype(np.float32)])
        return f32(Xq @ _q8_fake(M, q80_gs, wquantize).T)

    if q80_gs:
        X = _q8_fake(W["E"], q80_gs, wquantize)[tokens]
    else:
        X = W["E"][tokens].copy()
    mask = np.triu(np.full((T, T), -np.inf), 1)
    for l in range(L):
        Xn = _rms(X, W["w_att"][l])
        Q = rope(mm(Xn, W["wq"][l]), H)
        K = rope(mm(Xn, W["wk"][l]), Hkv)
        Vv = mm(Xn, W["wv"][l])
        if kv8:
            K, Vv = _kv8(K, hs, quantize), _kv8(Vv, hs, quantize)
        Kr = np.repeat(K.reshape(T, Hkv, hs), rep, axis=1)
        Vr = np.repeat(Vv.reshape(T, Hkv, hs), rep, axis=1)
        Qh = Q.reshape(T, H, hs)
        Sc = np.einsum("thi,shi->hts", Qh, Kr) / np.sqrt(hs) + mask
        Sc = np.exp(Sc - Sc.max(-1, keepdims=True))
        A = Sc / Sc.sum(-1, keepdims=True)
        O = f32(np.einsum("hts,shi->thi", A, Vr).reshape(T, d))
        X = f32(X + mm(O, W["wo"][l]))
        Xn = _rms(X, W["w_ffn"][l])
        G = mm(Xn, W["w1"][l])
        U = mm(Xn, W["w3"][l])
        Hh = f32(G / (1 + np.exp(-G)) * U)
        X = f32(X + mm(Hh, W["w2"][l]))
    Xn = _rms(X, W["w_final"])
    return mm(Xn, W["wcls"])
