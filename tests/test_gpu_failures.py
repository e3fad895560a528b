"""Failure detection without a GPU fault.

- A bounded wait that runs out: with the test switch L2C_TEST_STALL=1 read at
  l2c_create, CTA 0 of the first Q8_0 q/k/v kernel withholds one weight copy
  once, so the warp that needs it waits for data that never comes.  With the
  wait limit shortened to 20 ms (L2C_WAIT_NS), the kernels give up, record
  DERR_TIMEOUT and return; l2c_sync reports L2C_E_DEVICE ("wait-timeout"), and
  the handle then decodes the same step correctly.
- Device allocations that fail: the switch L2C_TEST_OOM_AFTER=N makes every
  allocation after the first N fail; l2c_create and l2c_enable_q80 must return
  L2C_E_OOM and leave no device memory behind.
"""
import time

import numpy as np
import pytest

import oracle
import synth
from gpu_util import need_gpu, rel_err

pytestmark = pytest.mark.gpu

Q64 = synth.ModelSpec("q64", 256, 768, 2, 4, 2, 700, 200, 0, seed=14)


def test_bounded_wait_runs_out_and_handle_recovers(monkeypatch):
    torch, l2c = need_gpu()
    spec = Q64
    b = synth.blob(spec)
    monkeypatch.setenv("L2C_TEST_STALL", "1")
    monkeypatch.setenv("L2C_WAIT_NS", str(20_000_000))
    dec = l2c.Decoder(spec.cfg, torch.from_numpy(b).cuda(), spec.shared_weights)
    monkeypatch.delenv("L2C_TEST_STALL")
    monkeypatch.delenv("L2C_WAIT_NS")
    dec.enable_q80(64)
    orc = oracle.Model(spec.cfg, b, spec.shared_weights)
    orc.enable_q80(64)
    t0 = time.perf_counter()
    dec.forward(3, 0, q80=True)
    with pytest.raises(l2c.L2CError) as e:
        dec.sync()
    elapsed = time.perf_counter() - t0
    assert e.value.code == l2c.L2C_E_DEVICE
    assert "wait-timeout" in str(e.value)
    assert elapsed < 1.5, elapsed  # a few 20 ms limits, not the 2 s default
    # the switch fired once: the same step now matches the oracle, and so do the next ones
    for p, tok in enumerate((3, 17, 250)):
        got = dec.forward(tok, p, q80=True).cpu().numpy()
        ref = orc.forward(tok, p, q80=True)
        assert rel_err(got, ref) <= 1e-5, p
    dec.sync()
    dec.close()
    orc.close()


def _create(l2c, torch, spec, blob):
    return l2c.Decoder(spec.cfg, blob, spec.shared_weights)


def test_allocation_failures_return_oom_and_leak_nothing(monkeypatch):
    torch, l2c = need_gpu()
    spec = synth.M15
    blob = torch.from_numpy(synth.blob(spec)).cuda()
    _create(l2c, torch, spec, blob).close()  # warm-up: context, streams, module loading
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    # l2c_create: refuse the n-th allocation for a few n
    n_ok = None
    for n in range(0, 64):
        monkeypatch.setenv("L2C_TEST_OOM_AFTER", str(n))
        try:
            dec = _create(l2c, torch, spec, blob)
        except l2c.L2CError as err:
            assert err.code == l2c.L2C_E_OOM, (n, err.code)
            continue
        n_ok = n
        break
    assert n_ok is not None and n_ok > 5
    dec.close()
    # l2c_enable_q80: the handle is made, the Q8_0 set fails part-way
    monkeypatch.setenv("L2C_TEST_OOM_AFTER", str(n_ok + 2))
    dec = _create(l2c, torch, spec, blob)
    monkeypatch.delenv("L2C_TEST_OOM_AFTER")
    with pytest.raises(l2c.L2CError) as e:
        dec.enable_q80(32)
    assert e.value.code == l2c.L2C_E_OOM
    # the fp32 path still works on that handle
    got = dec.forward(1, 0).cpu().numpy()
    assert np.all(np.isfinite(got))
    dec.sync()
    dec.close()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert abs(free1 - free0) <= (1 << 20), (free0, free1)
