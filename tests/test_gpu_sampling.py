"""l2c_sample against the oracle's sampling step (orc_sample) on the same logits.

The index must be the oracle's, except where the oracle's own decision is
within rounding of a threshold: the top-p running weight within 1e-12 of
topp * sum q, or the coin's target within 1e-12 of a running weight (the GPU
sums in another order).  Coins come from the seeded generator (numpy's
seeded generator, uniform in [0, 1)); logits are seeded normals of several sizes
(ragged tails included) and the logits of a 15M-shape decode step."""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    torch, l2c = need_gpu()
    dec = l2c.Decoder(synth.TINY.cfg, synth.blob(synth.TINY), synth.TINY.shared_weights)
    yield torch, l2c, dec
    dec.close()


def _margins(z, T, topp, coin):
    """Relative distance of the oracle's two decisions from their thresholds."""
    q = np.exp((z.astype(np.float64) - float(z.max())) / T)
    Z = q.sum()
    mp = np.inf
    tau = 0.0
    if topp < 1.0:
        s = np.sort(q)[::-1]
        c = np.cumsum(s)
        k = int(np.argmax(c >= topp * Z))
        tau = s[k]
        mp = abs(c[k] - topp * Z) / Z
        if k > 0:
            mp = min(mp, abs(c[k - 1] - topp * Z) / Z)
    sel = q >= tau
    zs = q[sel].sum()
    cs = np.cumsum(q[sel])
    mc = np.abs(cs - coin * zs).min() / zs
    return min(mp, mc)


def _coins(seed, n):
    return np.random.default_rng(seed).random(n)


@pytest.mark.parametrize("n", [1, 7, 1000, 32000, 32001])
@pytest.mark.parametrize("T,topp", [(1.0, 1.0), (0.7, 0.95), (1.5, 0.5), (1.0, 0.05), (0.3, 0.9)])
def test_sample_matches_oracle(env, n, T, topp):
    torch, l2c, dec = env
    rng = np.random.default_rng(n * 7 + int(T * 10) + int(topp * 100))
    z = (rng.standard_normal(n) * 2.0).astype(np.float32)
    if n > 10:
        z[n // 3] = z[n // 5]  # a tie
    zd = torch.from_numpy(z).cuda()
    checked = 0
    for u in _coins(n + int(topp * 1000), 12):
        got = dec.sample(zd, T, topp, float(u))
        ref = oracle.sample(z, T, topp, float(u))
        if got != ref:
            assert _margins(z, T, topp, float(u)) < 1e-12, (got, ref, u)
        else:
            checked += 1
    assert checked >= 10


def test_sample_temperature_zero_is_argmax(env):
    torch, l2c, dec = env
    rng = np.random.default_rng(1)
    z = rng.standard_normal(5000).astype(np.float32)
    z[10] = z[20] = z.max() + 1
    assert dec.sample(torch.from_numpy(z).cuda(), 0.0, 0.9, 0.5) == 10


def test_sample_decode_logits(env):
    """The logits of a 15M-shape step, sampled on the device without a host round trip."""
    torch, l2c, _ = env
    spec = synth.M15
    b = synth.blob(spec)
    dec = l2c.Decoder(spec.cfg, torch.from_numpy(b).cuda(), spec.shared_weights)
    for p, tok in enumerate((1, 500, 31999)):
        lg = dec.forward(tok, p)
        z = lg.cpu().numpy()  # the same logits on both sides: the device's own
        for u in (0.1, 0.6, 0.97):
            got = dec.sample(lg, 0.8, 0.9, u)
            ref = oracle.sample(z, 0.8, 0.9, u)
            if got != ref:
                assert _margins(z, 0.8, 0.9, u) < 1e-12
    dec.close()


def test_sample_rejects_bad_arguments_and_nan(env):
    torch, l2c, dec = env
    z = torch.zeros(100, device="cuda")
    for T, topp, u in ((-1.0, 0.9, 0.5), (1.0, 0.0, 0.5), (1.0, 0.9, 1.0), (1.0, 0.9, -0.1)):
        with pytest.raises(l2c.L2CError) as e:
            dec.sample(z, T, topp, u)
        assert e.value.code == l2c.L2C_E_ARG
    z[5] = float("nan")
    with pytest.raises(l2c.L2CError) as e:
        dec.sample(z, 1.0, 0.9, 0.5)
    assert e.value.code == l2c.L2C_E_DEVICE
