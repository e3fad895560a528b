"""Shared helpers of the GPU parity tests: build once, seeded workloads, tolerances."""
import numpy as np
import pytest

import synth

# Tolerances: max |gpu - oracle| <= TOL * max |oracle logit|
TOL_F32 = 1e-4
TOL_Q80 = 2e-3


def need_gpu():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    import decode_llama_step_02_b200 as l2c
    return torch, l2c


def device_blob(torch, spec):
    """The spec's seeded blob as a device tensor, and the host copy."""
    b = synth.blob(spec)
    return torch.from_numpy(b).cuda(), b


def rel_err(got, ref):
    return float(np.abs(np.asarray(got, np.float64) - ref).max() / np.abs(ref).max())


def top2_gap(logits):
    s = np.sort(np.asarray(logits, np.float64))
    return s[-1] - s[-2]
