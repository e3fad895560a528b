"""The C ABI without a GPU: the library loads, exports every symbol that
include/l2c.h declares, and rejects bad shapes on the host before any CUDA call."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def l2c():
    import __graft_entry__
    __graft_entry__.build()
    import decode_llama_step_02_b200 as m
    return m


def _declared():
    src = open(os.path.join(ROOT, "include", "l2c.h")).read()
    return sorted(set(re.findall(r"L2C_API\s+[^;(]*?\b(l2c_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(l2c):
    names = _declared()
    assert len(names) >= 17
    lib = ctypes.CDLL(l2c.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(l2c.EXPORTS) == names


def test_blob_floats_matches_generator(l2c):
    import synth
    for spec in synth.SPECS.values():
        assert l2c.blob_floats(spec.cfg, spec.shared_weights) == synth.blob_floats(spec)


@pytest.mark.parametrize("cfg,why", [
    ((64, 172, 5, 7, 1, 512, 512), "dim % n_heads"),
    ((64, 172, 5, 8, 3, 512, 512), "n_heads % n_kv_heads"),
    ((60, 172, 5, 4, 4, 512, 512), "odd head_size"),
    ((64, 170, 5, 8, 4, 512, 512), "hidden not a multiple of 4"),
    ((0, 172, 5, 8, 4, 512, 512), "zero dim"),
    ((1024, 4096, 1, 4, 4, 10, 10), "head_size 256 unsupported"),
])
def test_create_rejects_bad_shapes(l2c, cfg, why):
    c = l2c.Config(*cfg)
    blob = np.zeros(16, np.float32)
    h = ctypes.c_void_p()
    rc = l2c.lib().l2c_create(ctypes.byref(c), blob.ctypes.data, blob.size, 1, 1, None, ctypes.byref(h))
    assert rc == l2c.L2C_E_ARG, why
    assert not h.value


def test_create_rejects_wrong_blob_size(l2c):
    import synth
    spec = synth.TINY
    n = synth.blob_floats(spec)
    c = l2c.Config(*spec.cfg)
    blob = np.zeros(n + 1, np.float32)
    h = ctypes.c_void_p()
    rc = l2c.lib().l2c_create(ctypes.byref(c), blob.ctypes.data, n + 1, 1, 1, None, ctypes.byref(h))
    assert rc == l2c.L2C_E_ARG
    rc = l2c.lib().l2c_create(ctypes.byref(c), None, n, 1, 1, None, ctypes.byref(h))
    assert rc == l2c.L2C_E_ARG


def test_null_handle_calls_are_safe(l2c):
    L = l2c.lib()
    assert L.l2c_forward(None, 0, 0) is None
    assert L.l2c_sync(None) == l2c.L2C_E_ARG
    assert L.l2c_enable_q80(None, 32) == l2c.L2C_E_ARG
    L.l2c_destroy(None)
