"""CPU oracle of the llama2.c decode step (ctypes binding of oracle.c).

TEST INFRASTRUCTURE ONLY.  The plain, slow restatement that the GPU library is
checked against.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import it; the GPU library never does.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_HDR = os.path.join(_HERE, "oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")

# IEEE arithmetic as written: no fast-math, no contraction into FMAs.
CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared", "-std=c99"]


def build(force: bool = False) -> str:
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("dim", "hidden_dim", "n_layers", "n_heads", "n_kv_heads", "vocab_size", "seq_len")]


_lib = None


def lib():
    global _lib
    if _lib is None:
        # ORACLE_LIB_PATH loads a differently built copy (the mutation tests plant
        # mistakes in copies of oracle.c to show that the pins catch them)
        path = os.environ.get("ORACLE_LIB_PATH") or build()
        L = ctypes.CDLL(path)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        sig = {
            "orc_set_fp32_accum": (None, [i32]),
            "orc_rmsnorm": (None, [vp, vp, vp, i32]),
            "orc_matvec": (None, [vp, vp, vp, i32, i32]),
            "orc_rope_freq": (ctypes.c_float, [i32, i32]),
            "orc_rope": (None, [vp, i32, i32, i32]),
            "orc_softmax": (None, [vp, i32]),
            "orc_attention": (None, [vp, vp, vp, vp, i32, i32, i32, i32]),
            "orc_silu": (ctypes.c_double, [ctypes.c_double]),
            "orc_swiglu": (None, [vp, vp, i32]),
            "orc_quantize": (i32, [vp, i64, i32, vp, vp]),
            "orc_quantize4": (i32, [vp, i64, i32, vp, vp]),
            "orc_dequantize": (None, [vp, vp, i64, i32, vp]),
            "orc_q80_group_dots": (None, [vp, vp, vp, i32, i32, i32]),
            "orc_matvec_q80": (None, [vp, vp, vp, vp, vp, i32, i32, i32]),
            "orc_argmax": (i32, [vp, i32]),
            "orc_sample": (i32, [vp, i32, ctypes.c_float, ctypes.c_float, ctypes.c_double]),
            "orc_blob_floats": (sz, [vp, i32]),
            "orc_create": (vp, [vp, vp, sz, i32, i32]),
            "orc_enable_q80": (i32, [vp, i32]),
            "orc_enable_q40": (i32, [vp, i32]),
            "orc_enable_kv8": (i32, [vp]),
            "orc_kv8_row": (None, [vp, i32, i32]),
            "orc_forward": (i32, [vp, i32, i32, i32, i32, vp]),
            "orc_kv_load": (i32, [vp, i32, i32, vp, vp]),
            "orc_kv_read": (i32, [vp, i32, i32, vp, vp]),
            "orc_kv_reset": (i32, [vp, i32]),
            "orc_generate": (i32, [vp, i32, i32, i32, i32, i32, vp, vp]),
            "orc_destroy": (None, [vp]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags.c_contiguous
    return a.ctypes.data


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


class fp32_accum:
    """Context manager: the pages' fp32 sequential sums instead of double."""

    def __enter__(self):
        lib().orc_set_fp32_accum(1)

    def __exit__(self, *exc):
        lib().orc_set_fp32_accum(0)


def rmsnorm(x, w):
    x, w = _f32(x), _f32(w)
    o = np.empty_like(x)
    lib().orc_rmsnorm(_p(o), _p(x), _p(w), x.size)
    return o


def matvec(W, x):
    """W [d][n] @ x [n] -> [d]."""
    W, x = _f32(W), _f32(x)
    d, n = W.shape
    o = np.empty(d, dtype=np.float32)
    lib().orc_matvec(_p(o), _p(x), _p(W), n, d)
    return o


def rope_freq(j: int, head_size: int) -> float:
    return lib().orc_rope_freq(j, head_size)


def rope(v, head_size: int, pos: int):
    v = _f32(v).copy()
    lib().orc_rope(_p(v), v.size, head_size, pos)
    return v


def softmax(x):
    x = np.ascontiguousarray(x, dtype=np.float64).copy()
    lib().orc_softmax(_p(x), x.size)
    return x


def attention(q, kc, vc, pos: int, n_heads: int, n_kv_heads: int):
    """q [H*hs]; kc, vc [>=pos+1][kv_dim] -> [H*hs]."""
    q, kc, vc = _f32(q), _f32(kc), _f32(vc)
    hs = q.size // n_heads
    assert kc.shape[-1] == n_kv_heads * hs and kc.shape[0] > pos
    o = np.empty_like(q)
    lib().orc_attention(_p(o), _p(q), _p(kc), _p(vc), pos, n_heads, n_kv_heads, hs)
    return o


def silu(z: float) -> float:
    return lib().orc_silu(z)


def swiglu(a, b):
    a, b = _f32(a).copy(), _f32(b)
    lib().orc_swiglu(_p(a), _p(b), a.size)
    return a


def quantize(x, gs: int):
    """Q8_0: (codes int8 [n], scales fp32 [n/gs])."""
    x = _f32(x).ravel()
    q = np.empty(x.size, dtype=np.int8)
    s = np.empty(x.size // gs, dtype=np.float32)
    if lib().orc_quantize(_p(x), x.size, gs, _p(q), _p(s)) != 0:
        raise ValueError("n must be a multiple of gs")
    return q, s


def quantize4(x, gs: int):
    """Q4_0: (codes int8 [n] in [-7, 7], scales fp32 [n/gs])."""
    x = _f32(x).ravel()
    q = np.empty(x.size, dtype=np.int8)
    s = np.empty(x.size // gs, dtype=np.float32)
    if lib().orc_quantize4(_p(x), x.size, gs, _p(q), _p(s)) != 0:
        raise ValueError("n must be a multiple of gs")
    return q, s


def dequantize(q, s, gs: int):
    q = np.ascontiguousarray(q, dtype=np.int8)
    s = _f32(s)
    o = np.empty(q.size, dtype=np.float32)
    lib().orc_dequantize(_p(q), _p(s), q.size, gs, _p(o))
    return o


def q80_group_dots(qw, qx, gs: int):
    """qw [d][n] int8, qx [n] int8 -> int32 [d][n/gs]."""
    qw = np.ascontiguousarray(qw, dtype=np.int8)
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    d, n = qw.shape
    o = np.empty((d, n // gs), dtype=np.int32)
    lib().orc_q80_group_dots(_p(o), _p(qx), _p(qw), n, d, gs)
    return o


def matvec_q80(qw, sw, qx, sx, gs: int):
    qw = np.ascontiguousarray(qw, dtype=np.int8)
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    sw, sx = _f32(sw), _f32(sx)
    d, n = qw.shape
    o = np.empty(d, dtype=np.float32)
    lib().orc_matvec_q80(_p(o), _p(qx), _p(sx), _p(qw), _p(sw), n, d, gs)
    return o


def kv8_row(row, gs: int) -> np.ndarray:
    """A K/V row as the int8 KV cache keeps it: quantize() per gs group, then code * scale."""
    r = _f32(row).copy()
    lib().orc_kv8_row(_p(r), r.size, int(gs))
    return r


def argmax(x) -> int:
    x = _f32(x)
    return lib().orc_argmax(_p(x), x.size)


def sample(z, temperature: float, topp: float, coin: float) -> int:
    """Temperature / top-p / multinomial draw with the given coin (orc_sample)."""
    z = _f32(z)
    return lib().orc_sample(_p(z), z.size, float(temperature), float(topp), float(coin))


def blob_floats(cfg, shared_weights: int) -> int:
    c = _Config(*cfg)
    return lib().orc_blob_floats(ctypes.byref(c), shared_weights)


class Model:
    """The whole decode step on the CPU; keeps a reference to `blob`."""

    def __init__(self, cfg, blob: np.ndarray, shared_weights: int, n_seq: int = 1):
        assert blob.dtype == np.float32 and blob.flags.c_contiguous
        self.cfg = tuple(cfg)
        self.vocab = cfg[5]
        self._blob = blob
        c = _Config(*cfg)
        self._h = lib().orc_create(ctypes.byref(c), _p(blob), blob.size, shared_weights, n_seq)
        if not self._h:
            raise ValueError("orc_create rejected the config or blob size")
        self.gs = 0
        self.gs4 = 0

    def enable_q80(self, gs: int):
        if lib().orc_enable_q80(self._h, gs) != 0:
            raise ValueError("orc_enable_q80 failed")
        self.gs = gs

    def enable_q40(self, gs: int):
        """Q4_0 weights (orc_enable_q40); their matvec inputs stay Q8_0."""
        if lib().orc_enable_q40(self._h, gs) != 0:
            raise ValueError("orc_enable_q40 failed")
        self.gs4 = gs

    def enable_kv8(self):
        """int8 KV cache: K/V rows kept as Q8_0 groups of head_size (orc_enable_kv8)."""
        if lib().orc_enable_kv8(self._h) != 0:
            raise ValueError("orc_enable_kv8 failed")

    @staticmethod
    def _wf(q80, q40):
        return 2 if q40 else int(bool(q80))

    def forward(self, token: int, pos: int, q80: bool = False, seq: int = 0, q40: bool = False) -> np.ndarray:
        out = np.empty(self.vocab, dtype=np.float32)
        if lib().orc_forward(self._h, seq, token, pos, self._wf(q80, q40), _p(out)) != 0:
            raise ValueError("orc_forward rejected its arguments")
        return out

    def kv_load(self, k, v, seq: int = 0):
        k, v = _f32(k), _f32(v)
        if lib().orc_kv_load(self._h, seq, k.shape[1], _p(k), _p(v)) != 0:
            raise ValueError("orc_kv_load failed")

    def kv_read(self, n_pos: int, seq: int = 0):
        L, kvd = self.cfg[2], self.cfg[4] * (self.cfg[0] // self.cfg[3])
        k = np.empty((L, n_pos, kvd), dtype=np.float32)
        v = np.empty_like(k)
        if lib().orc_kv_read(self._h, seq, n_pos, _p(k), _p(v)) != 0:
            raise ValueError("orc_kv_read failed")
        return k, v

    def kv_reset(self, seq: int = 0):
        lib().orc_kv_reset(self._h, seq)

    def generate(self, token0: int, steps: int, q80: bool = False, pos0: int = 0, seq: int = 0,
                 keep_logits: bool = True, q40: bool = False):
        toks = np.empty(steps, dtype=np.int32)
        lg = np.empty((steps, self.vocab), dtype=np.float32) if keep_logits else None
        rc = lib().orc_generate(self._h, seq, token0, pos0, steps, self._wf(q80, q40), _p(toks),
                                _p(lg) if lg is not None else None)
        if rc != 0:
            raise ValueError("orc_generate failed")
        return toks, lg

    def close(self):
        if self._h:
            lib().orc_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
