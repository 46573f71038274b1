"""Pins of the sampling oracle (``oracle.sampler``) against the page's worked
example, closed forms and independent brute-force formulations."""
from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest

from oracle import sampler


GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "sampler_page_example.json")


def test_page_example():
    # "vLLM 基本原理", FlashInfer 采样器: logits 8.2 / 7.9 / 5.1 / 1.2 with
    # temperature 0.7, top_k 50, top_p 0.9.  The two most likely tokens already
    # hold 0.60 + 0.39 >= 0.9, so they are kept and the draw is between them
    # with probability sigmoid((8.2 - 7.9) / 0.7) for the first.
    g = json.load(open(GOLDEN))
    x = np.array(g["logits"])
    assert (g["temperature"], g["top_k"], g["top_p"]) == (0.7, 50, 0.9)
    r = sampler.distribution(x, g["temperature"], g["top_k"], g["top_p"])
    first = 1.0 / (1.0 + math.exp(-(8.2 - 7.9) / 0.7))
    assert r[0] == pytest.approx(first, abs=1e-12)
    assert r[1] == pytest.approx(1 - first, abs=1e-12)
    assert r[2] == 0 and r[3] == 0
    assert sampler.sample(x, 0.7, 50, 0.9, first - 1e-9) == 0
    assert sampler.sample(x, 0.7, 50, 0.9, first + 1e-9) == 1


def test_greedy_and_ties():
    x = np.array([1.0, 3.0, 3.0, 2.0])
    assert sampler.sample(x, 0.0, 0, 1.0, 0.99) == 1      # lowest index of the tie
    assert sampler.sample(x, -1.0, 2, 0.5, 0.0) == 1
    # top-k 1 keeps both tied maxima; the draw splits evenly between them
    r = sampler.distribution(x, 1.0, 1, 1.0)
    assert r.tolist() == [0.0, 0.5, 0.5, 0.0]


def test_plain_softmax_when_nothing_is_filtered():
    rng = np.random.default_rng(0)
    x = rng.normal(size=50) * 3
    for T in (0.5, 1.0, 2.0):
        r = sampler.distribution(x, T, 0, 1.0)
        e = np.exp(x / T - (x / T).max())
        assert np.allclose(r, e / e.sum(), rtol=0, atol=1e-15)
        assert np.array_equal(r, sampler.distribution(x, T, 50, 1.0))  # K = V
        assert np.array_equal(r, sampler.distribution(x, T, 99, 1.0))  # K > V


def brute_kept(x, T, K, P):
    """Token i survives Top-K iff fewer than K logits are strictly larger; it
    survives Top-P iff the renormalised probability of the strictly larger
    survivors of Top-K is below P."""
    x = np.asarray(x, np.float64)
    V = len(x)
    keep_k = [(K <= 0 or K >= V) or sum(x[j] > x[i] for j in range(V)) < K for i in range(V)]
    z = np.exp(x / T - (x / T).max())
    tot = sum(z[j] for j in range(V) if keep_k[j])
    keep = []
    for i in range(V):
        if not keep_k[i]:
            keep.append(False)
            continue
        above = sum(z[j] for j in range(V) if keep_k[j] and x[j] > x[i]) / tot
        keep.append(P >= 1 or above < P)
    return np.array(keep)


@pytest.mark.parametrize("seed", range(20))
def test_kept_set_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    V = int(rng.integers(1, 12))
    x = np.round(rng.normal(size=V) * 2, 1)          # rounding makes ties common
    T = float(rng.choice([0.3, 1.0, 1.7]))
    K = int(rng.integers(0, V + 2))
    P = float(rng.choice([0.05, 0.5, 0.9, 1.0]))
    mask, _ = sampler.kept_set(x, T, K, P)
    assert np.array_equal(mask, brute_kept(x, T, K, P)), (x, T, K, P)


def test_draw_frequencies_follow_the_distribution():
    # stratified uniforms: the count of each token is N * r_i to within one
    rng = np.random.default_rng(5)
    x = rng.normal(size=30) * 2
    for T, K, P in [(1.0, 0, 1.0), (0.8, 10, 1.0), (1.2, 0, 0.7), (0.9, 8, 0.8)]:
        r = sampler.distribution(x, T, K, P)
        N = 4000
        counts = np.bincount([sampler.sample(x, T, K, P, (j + 0.5) / N) for j in range(N)],
                             minlength=len(x))
        assert np.all(np.abs(counts - N * r) <= 1.0 + 1e-9), (T, K, P)
        assert np.all(counts[r == 0] == 0)


def test_draw_order_is_the_vocabulary_order():
    x = np.array([0.0, 5.0, 0.0, 5.0])
    # two kept tokens with equal probability: u below 1/2 gives the lower index
    assert sampler.sample(x, 1.0, 2, 1.0, 0.49) == 1
    assert sampler.sample(x, 1.0, 2, 1.0, 0.51) == 3
    assert sampler.sample(x, 1.0, 2, 1.0, 0.0) == 1
    assert sampler.sample(x, 1.0, 2, 1.0, 1.0 - 1e-16) == 3
