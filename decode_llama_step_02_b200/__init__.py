"""Python binding of libl2c.so, the B200 decode-step library (include/l2c.h).

Argument marshalling only: every step of the decode path runs in the library's
CUDA kernels.  PyTorch supplies device memory and streams.  Importing this
module does not need a GPU; creating a handle does, and there is no CPU
fallback: a missing library or device raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libl2c.so")

L2C_OK, L2C_E_ARG, L2C_E_OOM, L2C_E_CUDA, L2C_E_DEVICE, L2C_E_STATE, L2C_E_SCRATCH = 0, -1, -2, -3, -4, -5, -6

# every symbol declared in include/l2c.h
EXPORTS = (
    "l2c_blob_floats", "l2c_create", "l2c_enable_q80", "l2c_enable_q40", "l2c_forward", "l2c_forward_q80",
    "l2c_forward_q40", "l2c_argmax",
    "l2c_generate", "l2c_sample", "l2c_forward_batch", "l2c_prefill", "l2c_enable_kv8", "l2c_quantize_q80", "l2c_q80_group_dots", "l2c_kv_load",
    "l2c_kv_read", "l2c_kv_reset", "l2c_attention", "l2c_attention_noalloc", "l2c_time_kernel", "l2c_sync", "l2c_stream", "l2c_last_status", "l2c_last_error",
    "l2c_destroy",
)

# kernels of the step, as numbered by l2c_time_kernel
K_QKV, K_ATTN, K_WO, K_W13, K_W2, K_CLS = range(6)


class L2CError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"l2c error {code}: {msg}")
        self.code = code


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("dim", "hidden_dim", "n_layers", "n_heads", "n_kv_heads", "vocab_size", "seq_len")]


_lib = None


def lib():
    """Loads libl2c.so (built in-tree by __graft_entry__.build())."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; g.build()'`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        sig = {
            "l2c_blob_floats": (sz, [vp, i32]),
            "l2c_create": (i32, [vp, vp, sz, i32, i32, vp, ctypes.POINTER(vp)]),
            "l2c_enable_q80": (i32, [vp, i32]),
            "l2c_enable_q40": (i32, [vp, i32]),
            "l2c_forward": (vp, [vp, i32, i32]),
            "l2c_forward_q80": (vp, [vp, i32, i32]),
            "l2c_forward_q40": (vp, [vp, i32, i32]),
            "l2c_argmax": (i32, [vp, vp, i32, ctypes.POINTER(ctypes.c_int)]),
            "l2c_generate": (i32, [vp, i32, i32, i32, i32, vp]),
            "l2c_sample": (i32, [vp, vp, i32, ctypes.c_float, ctypes.c_float, ctypes.c_double,
                                 ctypes.POINTER(ctypes.c_int)]),
            "l2c_forward_batch": (i32, [vp, i32, vp, vp, i32, vp]),
            "l2c_prefill": (i32, [vp, i32, i32, vp, i32, i32, vp]),
            "l2c_enable_kv8": (i32, [vp, i32]),
            "l2c_quantize_q80": (i32, [vp, vp, i64, i32, vp, vp]),
            "l2c_q80_group_dots": (i32, [vp, vp, vp, i32, i32, i32, vp]),
            "l2c_kv_load": (i32, [vp, i32, i32, vp, vp]),
            "l2c_kv_read": (i32, [vp, i32, i32, vp, vp]),
            "l2c_kv_reset": (i32, [vp, i32]),
            "l2c_attention": (i32, [vp, vp, vp, vp, i32, i32, vp]),
            "l2c_attention_noalloc": (i32, [vp, vp, vp, i32, i32, i32, i32, i32, vp, vp]),
            "l2c_time_kernel": (i32, [vp, i32, i32, i32, ctypes.POINTER(ctypes.c_float)]),
            "l2c_sync": (i32, [vp]),
            "l2c_stream": (vp, [vp]),
            "l2c_last_status": (i32, [vp]),
            "l2c_last_error": (i32, [vp, ctypes.c_char_p, i32]),
            "l2c_destroy": (None, [vp]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def blob_floats(cfg, shared_weights: int) -> int:
    c = Config(*cfg)
    return int(lib().l2c_blob_floats(ctypes.byref(c), int(shared_weights)))


def _ptr(buf) -> int:
    """Address of a torch tensor (host or device) or a numpy array."""
    if isinstance(buf, np.ndarray):
        assert buf.flags.c_contiguous
        return buf.ctypes.data
    assert buf.is_contiguous()
    return buf.data_ptr()


class _DevArray:
    """Zero-copy __cuda_array_interface__ view of handle-owned device memory."""

    def __init__(self, ptr: int, shape, typestr: str, stream: int):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (ptr, False),
                                         "version": 3, "strides": None, "stream": None}


class Decoder:
    """One l2c handle: a Llama-2 decoder's weights, KV caches and step graphs on the GPU."""

    def __init__(self, cfg, blob, shared_weights: int, max_batch: int = 1, stream=None):
        import torch
        self.cfg = tuple(int(v) for v in cfg)
        self.vocab = self.cfg[5]
        if stream is None:
            stream = torch.cuda.current_stream()
        self.stream = stream
        n = blob.numel() if hasattr(blob, "numel") else blob.size
        h = ctypes.c_void_p()
        c = Config(*self.cfg)
        rc = lib().l2c_create(ctypes.byref(c), _ptr(blob), n, int(shared_weights), int(max_batch),
                              ctypes.c_void_p(stream.cuda_stream), ctypes.byref(h))
        if rc != L2C_OK:
            raise L2CError(rc, "l2c_create failed (see stderr)")
        self._h = h

    # -- errors
    def _msg(self) -> str:
        buf = ctypes.create_string_buffer(512)
        lib().l2c_last_error(self._h, buf, 512)
        return buf.value.decode(errors="replace")

    def _check(self, rc: int):
        if rc != L2C_OK:
            raise L2CError(rc, self._msg())

    def sync(self):
        self._check(lib().l2c_sync(self._h))

    # -- weights
    def enable_q80(self, gs: int):
        self._check(lib().l2c_enable_q80(self._h, int(gs)))

    def enable_q40(self, gs: int):
        """Q4_0 weights (l2c_enable_q40): 4-bit codes, scale = max|x| / 7 per group of gs."""
        self._check(lib().l2c_enable_q40(self._h, int(gs)))

    @staticmethod
    def _wf(q80, q40):
        """Weight format of the C ABI: 0 fp32, 1 Q8_0, 2 Q4_0."""
        return 2 if q40 else int(q80)

    # -- steps
    def forward_ptr(self, token: int, pos: int, q80: bool = False, q40: bool = False) -> int:
        f = (lib().l2c_forward, lib().l2c_forward_q80, lib().l2c_forward_q40)[self._wf(q80, q40)]
        p = f(self._h, int(token), int(pos))
        if not p:
            raise L2CError(lib().l2c_last_status(self._h), self._msg())
        return p

    def forward(self, token: int, pos: int, q80: bool = False, q40: bool = False):
        """Enqueues one step; returns a zero-copy torch view of the device logits."""
        import torch
        p = self.forward_ptr(token, pos, q80, q40)
        return torch.as_tensor(_DevArray(p, (self.vocab,), "<f4", 0), device="cuda")

    def argmax(self, logits) -> int:
        out = ctypes.c_int()
        self._check(lib().l2c_argmax(self._h, _ptr(logits), logits.numel(), ctypes.byref(out)))
        return out.value

    def sample(self, logits, temperature: float, topp: float, coin: float) -> int:
        """The token drawn from device logits with temperature / top-p and the given coin (l2c_sample)."""
        out = ctypes.c_int()
        self._check(lib().l2c_sample(self._h, _ptr(logits), int(logits.numel()), float(temperature), float(topp),
                                     float(coin), ctypes.byref(out)))
        return out.value

    def generate(self, token0: int, steps: int, q80: bool = False, pos0: int = 0, q40: bool = False) -> np.ndarray:
        toks = np.empty(steps, dtype=np.int32)
        self._check(lib().l2c_generate(self._h, int(token0), int(pos0), int(steps), self._wf(q80, q40),
                                       toks.ctypes.data))
        return toks

    def forward_batch(self, tokens, pos, logits_out, q80: bool = True):
        self._check(lib().l2c_forward_batch(self._h, int(tokens.numel() if hasattr(tokens, "numel") else tokens.size),
                                            _ptr(tokens), _ptr(pos), int(q80), _ptr(logits_out)))

    def prefill(self, tokens, pos0: int = 0, q80: bool = False, logits_last=None, seq: int = 0):
        """Prompt tokens (host int32) at positions pos0.. of sequence seq, as GEMMs
        (l2c_prefill); the last token's logits go to logits_last (device, optional)."""
        toks = np.ascontiguousarray(tokens, dtype=np.int32)
        self._check(lib().l2c_prefill(self._h, int(seq), int(toks.size), toks.ctypes.data, int(pos0), int(q80),
                                      _ptr(logits_last) if logits_last is not None else None))

    # -- KV cache
    def enable_kv8(self, on: bool = True):
        """The int8 KV cache (K/V rows as Q8_0 groups of one head) on or off (l2c_enable_kv8)."""
        self._check(lib().l2c_enable_kv8(self._h, int(on)))

    def kv_load(self, k, v, seq: int = 0):
        n_pos = k.shape[1]
        self._check(lib().l2c_kv_load(self._h, int(seq), int(n_pos), _ptr(k), _ptr(v)))

    def kv_read(self, n_pos: int, seq: int = 0):
        d, h, L, H, Hkv, V, S = self.cfg
        kvd = Hkv * (d // H)
        k = np.empty((L, n_pos, kvd), np.float32)
        v = np.empty_like(k)
        self._check(lib().l2c_kv_read(self._h, int(seq), int(n_pos), k.ctypes.data, v.ctypes.data))
        return k, v

    def kv_reset(self, seq: int = -1):
        self._check(lib().l2c_kv_reset(self._h, int(seq)))

    # -- standalone kernels
    def quantize_q80(self, x, gs: int, q_out, s_out):
        self._check(lib().l2c_quantize_q80(self._h, _ptr(x), int(x.numel()), int(gs), _ptr(q_out), _ptr(s_out)))

    def attention(self, q, k, v, pos: int, out, precision: int = 0):
        """One layer's GQA attention for positions 0..pos (l2c_attention)."""
        self._check(lib().l2c_attention(self._h, _ptr(q), _ptr(k), _ptr(v), int(pos), int(precision), _ptr(out)))

    def q80_group_dots(self, qw, qx, gs: int, out):
        rows, K = qw.shape
        self._check(lib().l2c_q80_group_dots(self._h, _ptr(qw), _ptr(qx), int(rows), int(K), int(gs), _ptr(out)))

    def time_kernel(self, kind: int, q80, iters: int) -> float:
        """Average ms per launch of one kernel of the step run alone (l2c_time_kernel);
        q80: 0 / False fp32, 1 / True Q8_0, 2 Q4_0."""
        ms = ctypes.c_float()
        self._check(lib().l2c_time_kernel(self._h, int(kind), int(q80), int(iters), ctypes.byref(ms)))
        return ms.value

    def set_position(self, token: int, pos: int, q80: bool = False, q40: bool = False):
        """Runs one step at (token, pos) so that the handle's state holds them."""
        self.forward_ptr(token, pos, q80, q40)

    def close(self):
        if getattr(self, "_h", None):
            lib().l2c_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
