"""The benchmark's algorithmic byte counts, checked on the CPU against the blob
layout (llama2.c checkpoint order): a decode step reads every stored weight once,
except that it reads one row of the embedding table and skips the two legacy RoPE
tables, plus the KV cache for positions 0..pos.  Also against the 7B figures of the
measurement plan (26.43 / 7.02 GB per token at pos 0, 28.58 / 9.17 GB at pos 2048)."""
import os
import sys

import pytest

import synth

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _fp32_weight_floats(spec):
    d, h, L, H, Hkv, V, S = spec.cfg
    hs = d // H
    legacy_rope = 2 * S * hs // 2
    n = synth.blob_floats(spec) - legacy_rope
    # the embedding table is read one row per token; tied, it is also the classifier
    return n - V * d + d if not spec.shared_weights else n + d


@pytest.mark.parametrize("spec", [synth.TINY, synth.M15, synth.M110, synth.L7B, synth.GQA7B],
                         ids=lambda s: s.name)
def test_fp32_bytes_follow_the_blob(spec):
    d, h, L, H, Hkv, V, S = spec.cfg
    kvd = Hkv * (d // H)
    for pos in (0, 7, S - 1):
        want = 4.0 * _fp32_weight_floats(spec) + 8.0 * L * (pos + 1) * kvd
        assert bench.bytes_per_token(False, pos, spec) == pytest.approx(want, rel=1e-12)


@pytest.mark.parametrize("gs", [32, 64, 128])
def test_q80_bytes_are_codes_scales_and_fp32_gains(gs):
    spec = synth.L7B
    d, h, L, H, Hkv, V, S = spec.cfg
    kvd = Hkv * (d // H)
    gains = L * 2 * d + d
    quantized = _fp32_weight_floats(spec) - gains  # matrices, classifier, one embedding row
    want = quantized * (1 + 4.0 / gs) + 4.0 * gains + 8.0 * L * 1 * kvd
    assert bench.bytes_per_token(True, 0, spec, gs) == pytest.approx(want, rel=1e-12)


def test_7b_figures_of_the_plan():
    s = synth.L7B
    assert bench.bytes_per_token(False, 0, s) / 1e9 == pytest.approx(26.43, abs=0.01)
    assert bench.bytes_per_token(True, 0, s) / 1e9 == pytest.approx(7.02, abs=0.01)
    assert bench.bytes_per_token(False, 2048, s) / 1e9 == pytest.approx(28.58, abs=0.01)
    assert bench.bytes_per_token(True, 2048, s) / 1e9 == pytest.approx(9.17, abs=0.01)
    assert bench.bytes_per_token(True, -1, synth.GQA7B) / 1e9 == pytest.approx(6.17, abs=0.01)
    # one W1/W3 launch: both matrices, gain, input and output
    assert bench.w13_bytes(False, s) / 1e6 == pytest.approx(360.8, abs=0.1)
    assert bench.w13_bytes(True, s) / 1e6 == pytest.approx(95.9, abs=0.1)


@pytest.mark.parametrize("gs", [32, 64, 128])
def test_q40_bytes_are_nibbles_scales_and_fp32_gains(gs):
    """Q4_0: every matrix and the classifier at half a byte per weight plus an fp32 scale
    per group; the embedding row in the int8-wide layout (a byte per code); gains fp32."""
    spec = synth.L7B
    d, h, L, H, Hkv, V, S = spec.cfg
    kvd = Hkv * (d // H)
    gains = L * 2 * d + d
    mats = _fp32_weight_floats(spec) - gains - d  # without the embedding row
    want = mats * (0.5 + 4.0 / gs) + d * (1 + 4.0 / gs) + 4.0 * gains + 8.0 * L * 1 * kvd
    assert bench.q40_bytes_per_token(0, spec, gs) == pytest.approx(want, rel=1e-12)
    # the kernels' weight bytes (q/k/v, wo, W1/W3, W2 per layer; the classifier) add up to
    # the step's quantized matrices
    vec = {0: 4.0 * (2 * d + d + 2 * kvd), 2: 4.0 * 3 * d, 3: 4.0 * (2 * d + h), 4: 4.0 * (h + 2 * d),
           5: 4.0 * (2 * d + V)}
    kw = L * sum(bench.kernel_bytes(k, 2, 0, spec, gs) - vec[k] for k in (0, 2, 3, 4))
    kw += bench.kernel_bytes(5, 2, 0, spec, gs) - vec[5]
    assert kw == pytest.approx(mats * (0.5 + 4.0 / gs), rel=1e-12)
