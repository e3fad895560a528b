"""Pins of the oracle's sampling step (temperature, top-p, a draw with the
caller's coin).  The pages fix only that a temperature divides the logits
before the softmax ("LLM底层原理与工程实践" §3.2) and that temperature 0 is the
greedy sample_argmax ("超精简LLM部署" 智能家居控制案例); the rest is the reading
stated in oracle.c (orc_sample).  The pins are closed forms and an exact
quadrature of the draw against an independent float64 softmax."""
import math

import numpy as np
import pytest

import oracle


def test_temperature_zero_is_the_greedy_argmax():
    rng = np.random.default_rng(0)
    z = rng.standard_normal(1000).astype(np.float32)
    z[17] = z[400] = z.max() + 1.0  # tie: the lowest index
    for u in (0.0, 0.3, 0.999):
        assert oracle.sample(z, 0.0, 1.0, u) == 17 == oracle.argmax(z)


@pytest.mark.parametrize("n", [1, 7, 1000])
def test_uniform_logits_map_the_coin_to_floor_u_n(n):
    z = np.full(n, 0.25, np.float32)
    for k in range(min(n, 50)):
        u = (k + 0.5) / n
        assert oracle.sample(z, 1.0, 1.0, u) == k
    assert oracle.sample(z, 1.0, 1.0, 0.0) == 0


@pytest.mark.parametrize("T", [0.5, 1.0, 2.0])
def test_two_tokens_split_at_the_logistic_probability(T):
    a, b = np.float32(0.3), np.float32(-0.4)
    p0 = 1.0 / (1.0 + math.exp((float(b) - float(a)) / T))
    z = np.array([a, b], np.float32)
    assert oracle.sample(z, T, 1.0, p0 - 1e-9) == 0
    assert oracle.sample(z, T, 1.0, p0 + 1e-9) == 1


def test_draw_frequencies_equal_the_softmax():
    # coins on a fine grid: token i is drawn for a fraction of the coins equal to its
    # probability, to within one grid step (the draw inverts the cumulative weights)
    rng = np.random.default_rng(3)
    z = (rng.standard_normal(10) * 1.5).astype(np.float32)
    T = 0.8
    N = 20000
    counts = np.zeros(10)
    for k in range(N):
        counts[oracle.sample(z, T, 1.0, (k + 0.5) / N)] += 1
    e = np.exp((z.astype(np.float64) - z.max()) / T)
    p = e / e.sum()
    assert np.abs(counts / N - p).max() <= 1.0 / N + 1e-12


def _logits(probs):
    return np.log(np.asarray(probs, np.float64)).astype(np.float32)


def test_top_p_keeps_the_smallest_set_reaching_p():
    z = _logits([0.5, 0.3, 0.2])
    # p = 0.45: {0}
    assert {oracle.sample(z, 1.0, 0.45, u) for u in (0.0, 0.5, 0.999)} == {0}
    # p = 0.7: {0, 1}, drawn in proportion 0.5 : 0.3 (split at u = 0.625)
    assert oracle.sample(z, 1.0, 0.7, 0.62) == 0
    assert oracle.sample(z, 1.0, 0.7, 0.63) == 1
    assert oracle.sample(z, 1.0, 0.7, 0.999) == 1
    # p = 0.85: all three (split at 0.5 and 0.8 of the total)
    assert oracle.sample(z, 1.0, 0.85, 0.79) == 1
    assert oracle.sample(z, 1.0, 0.85, 0.81) == 2


def test_top_p_takes_every_token_tied_with_the_last_one():
    # 0.4 then three tokens of 0.2: the running sum reaches 0.5 on the first 0.2,
    # and the two other 0.2 tokens, tied with it, are in the set as well
    z = _logits([0.2, 0.4, 0.2, 0.2])
    assert oracle.sample(z, 1.0, 0.5, 0.999) == 3
    assert oracle.sample(z, 1.0, 0.5, 0.0) == 0
    # the set's order is the index order: token 1 (0.4) covers coins in [0.2, 0.6)
    assert oracle.sample(z, 1.0, 0.5, 0.3) == 1


def test_temperature_sharpens_and_flattens():
    z = _logits([0.6, 0.4])
    # T -> small: the larger logit takes almost every coin; T large: close to uniform
    assert oracle.sample(z, 0.05, 1.0, 0.99) == 0
    p0_hot = 1.0 / (1.0 + (0.4 / 0.6) ** (1 / 20.0))
    assert abs(p0_hot - 0.5) < 0.011
    assert oracle.sample(z, 20.0, 1.0, p0_hot - 1e-6) == 0
    assert oracle.sample(z, 20.0, 1.0, p0_hot + 1e-6) == 1
