"""The seeded input generator: published SplitMix64 outputs, counter independence,
moments of the normals, and the blob layout against the page's model sizes."""
import os

import numpy as np
import pytest

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_splitmix64_published_outputs():
    # SplitMix64 seeded with 0 (Steele, Lea, Flood 2014; Vigna's splitmix64.c):
    # the first three outputs of next() are widely tabulated.
    expect = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    got = [synth.lib().synth_u64(0, i) for i in range(3)]
    assert got == expect


def test_counter_based_ranges_agree():
    a = synth.normal(5, 0, 0, 10_001)
    for start in (0, 1, 2, 777, 9_999):
        b = synth.normal(5, 0, 0, 10_001 - start, start=start)
        assert np.array_equal(a[start:], b)


def test_normal_moments():
    z = synth.normal_f64(11, 0, 3, 2_000_000)
    assert abs(z.mean()) < 3e-3
    assert abs(z.std() - 1.0) < 3e-3
    # Gaussian tail mass beyond 2 sigma is 4.55%
    assert abs((np.abs(z) > 2).mean() - 0.0455) < 2e-3


def test_uniform_ints_in_range_and_flat():
    t = synth.tokens(3, 0, 200_000, 32000)
    assert t.min() >= 0 and t.max() < 32000
    hist = np.bincount(t // 3200, minlength=10)
    assert np.all(np.abs(hist / t.size - 0.1) < 0.005)


def test_blob_regions():
    spec = synth.M15
    b = synth.blob(spec)
    d, h, L, H, Hkv, V, S = spec.cfg
    hs = d // H
    kvd = Hkv * hs
    off_watt = V * d
    w_att = b[off_watt:off_watt + L * d]
    # RMSNorm gains of the 15M workload are 1 + N(0, 0.1)
    assert abs(w_att.mean() - 1.0) < 0.03 and abs(w_att.std() - 0.1) < 0.02
    E = b[:V * d]
    assert abs(E.std() - 0.02) < 2e-4
    # the legacy freq_cis region (seq_len * hs floats) sits at the tail and is zero (tied)
    assert np.all(b[-S * hs:] == 0)
    # chunked generation matches whole-blob generation
    part = np.empty(12345, dtype=np.float32)
    synth.blob_into(spec, part, start=off_watt - 100)
    assert np.array_equal(part, b[off_watt - 100:off_watt - 100 + 12345])


def test_blob_sizes_match_page_table():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "model_sizes.txt"))
            if ln.strip() and not ln.startswith("#")]
    for name, fp32_b, q8_b, tol in rows:
        spec = synth.SPECS[name]
        n = synth.blob_floats(spec)
        d, h, L, H, Hkv, V, S = spec.cfg
        hs = d // H
        # fp32 bytes of the checkpoint and Q8_0 bytes at GS=64 (codes + fp32 scales;
        # RMSNorm gains stay fp32, the legacy RoPE tables are dropped)
        norms = (2 * L + 1) * d
        quant = n - norms - S * hs
        q8 = quant * (1 + 4 / 64) + 4 * norms
        assert abs(4 * n / float(fp32_b) - 1) < float(tol), (name, 4 * n)
        assert abs(q8 / float(q8_b) - 1) < float(tol), (name, q8)


def test_kv_prefill_prefix_consistent():
    spec = synth.TINY
    k1, v1 = synth.kv_prefill(spec, seq=2, n_pos=10)
    k2, v2 = synth.kv_prefill(spec, seq=2, n_pos=17)
    assert np.array_equal(k1, k2[:, :10]) and np.array_equal(v1, v2[:, :10])
    k3, _ = synth.kv_prefill(spec, seq=3, n_pos=10)
    assert not np.array_equal(k1, k3)
    assert not np.array_equal(k1, v1)
