"""Seeded synthetic inputs for the Llama-2 decode step (weights, KV prefill, token ids).

Both the CPU oracle's tests and the GPU harness draw their inputs from here, so
the two sides see the same numbers.  The module holds none of the decode step's
arithmetic: see ``synth.c`` for the generator's definition (SplitMix64 counters,
Box-Muller normals) and the weight blob layout (llama2.c checkpoint order).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")

CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared", "-std=c99"]


def build(force: bool = False) -> str:
    """Compiles libsynth.so next to its source (host C only)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        u64, i32, u32, dbl = ctypes.c_uint64, ctypes.c_int32, ctypes.c_uint32, ctypes.c_double
        vp = ctypes.c_void_p
        _lib.synth_key.restype = u64
        _lib.synth_key.argtypes = [u64, u32, u64]
        _lib.synth_u64.restype = u64
        _lib.synth_u64.argtypes = [u64, u64]
        _lib.synth_normal_f64.argtypes = [u64, u64, u64, vp]
        _lib.synth_normal_f32.argtypes = [u64, u64, u64, dbl, dbl, vp]
        _lib.synth_uniform_int.argtypes = [u64, u64, u64, u32, vp]
        _lib.synth_blob_floats.restype = u64
        _lib.synth_blob_floats.argtypes = [vp, ctypes.c_int]
        _lib.synth_blob.restype = ctypes.c_int
        _lib.synth_blob.argtypes = [vp, ctypes.c_int, u64, dbl, dbl, u64, u64, vp]
        _lib.synth_kv.argtypes = [u64, u64, i32, i32, i32, i32, dbl, vp, vp]
        _lib.synth_tokens.argtypes = [u64, u64, u64, u32, vp]
        _lib.synth_positions.argtypes = [u64, u64, u64, u32, vp]
    return _lib


@dataclass(frozen=True)
class ModelSpec:
    """A Llama-2 decoder shape plus the recipe of its synthetic weights."""
    name: str
    dim: int
    hidden_dim: int
    n_layers: int
    n_heads: int
    n_kv_heads: int
    vocab_size: int
    seq_len: int
    shared_weights: int
    seed: int
    wsigma: float = 0.02
    nsigma: float = 0.0  # RMSNorm gains are 1 + N(0, nsigma)

    @property
    def cfg(self) -> tuple:
        return (self.dim, self.hidden_dim, self.n_layers, self.n_heads, self.n_kv_heads,
                self.vocab_size, self.seq_len)

    @property
    def head_size(self) -> int:
        return self.dim // self.n_heads

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_size


# The five workloads: tiny, 15M-shape, 110M-shape, 7B-shape (MHA, untied), 7B-width GQA.
TINY = ModelSpec("tiny", 64, 172, 5, 8, 4, 512, 512, 1, seed=0)
M15 = ModelSpec("15M", 288, 768, 6, 6, 6, 32000, 256, 1, seed=1, nsigma=0.1)
M110 = ModelSpec("110M", 768, 2048, 12, 12, 12, 32000, 1024, 1, seed=2)
L7B = ModelSpec("7B", 4096, 11008, 32, 32, 32, 32000, 4096, 0, seed=3)
GQA7B = ModelSpec("GQA-7B", 4096, 11008, 32, 32, 8, 32000, 2048, 0, seed=4)
SPECS = {s.name: s for s in (TINY, M15, M110, L7B, GQA7B)}


def _cfg_arr(spec: ModelSpec):
    return (ctypes.c_int32 * 7)(*spec.cfg)


def blob_floats(spec: ModelSpec) -> int:
    return int(lib().synth_blob_floats(_cfg_arr(spec), spec.shared_weights))


def blob_into(spec: ModelSpec, out: np.ndarray, start: int = 0) -> None:
    """Writes blob elements [start, start + out.size) into the float32 array `out`."""
    assert out.dtype == np.float32 and out.flags.c_contiguous
    rc = lib().synth_blob(_cfg_arr(spec), spec.shared_weights, spec.seed, spec.wsigma, spec.nsigma,
                          start, out.size, out.ctypes.data)
    if rc != 0:
        raise ValueError("blob range out of bounds")


def blob(spec: ModelSpec) -> np.ndarray:
    out = np.empty(blob_floats(spec), dtype=np.float32)
    blob_into(spec, out)
    return out


def kv_prefill(spec: ModelSpec, seq: int, n_pos: int, seed: int | None = None, sigma: float = 1.0):
    """K and V caches [L][n_pos][kv_dim] of N(0, sigma) for positions 0..n_pos-1."""
    seed = spec.seed if seed is None else seed
    shape = (spec.n_layers, n_pos, spec.kv_dim)
    k = np.empty(shape, dtype=np.float32)
    v = np.empty(shape, dtype=np.float32)
    lib().synth_kv(seed, seq, spec.n_layers, spec.seq_len, spec.kv_dim, n_pos, sigma,
                   k.ctypes.data, v.ctypes.data)
    return k, v


def tokens(seed: int, sub: int, n: int, vocab: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    lib().synth_tokens(seed, sub, n, vocab, out.ctypes.data)
    return out


def positions(seed: int, sub: int, n: int, n_range: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    lib().synth_positions(seed, sub, n, n_range, out.ctypes.data)
    return out


def normal(seed: int, stream: int, sub: int, n: int, mu: float = 0.0, sigma: float = 1.0,
           start: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    lib().synth_normal_f32(lib().synth_key(seed, stream, sub), start, n, mu, sigma, out.ctypes.data)
    return out


def normal_f64(seed: int, stream: int, sub: int, n: int, start: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    lib().synth_normal_f64(lib().synth_key(seed, stream, sub), start, n, out.ctypes.data)
    return out
