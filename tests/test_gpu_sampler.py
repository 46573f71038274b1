"""The fused sampler (``pa_sample``) against the sampling oracle.

The token for a given uniform number is a pure function of the inputs, so
each row is compared exactly -- except where float rounding decides the
answer: the kernel computes probabilities in fp32, the oracle in fp64, so a
row whose uniform number or Top-P cut sits within 1e-5 of a boundary accepts
any token the oracle draws with those inputs moved by 1e-5.  Frequencies over
stratified uniform numbers must match the oracle's distribution."""
from __future__ import annotations

import json
import os

import numpy as np
import pytest

from oracle import sampler

pytestmark = pytest.mark.gpu

EPS = 1e-5


def pa():
    import paged_kv_cache_454_b200 as m
    return m


def run(logits, T, K, P, u):
    import torch
    dev = torch.device("cuda")
    out = pa().pa_sample(torch.as_tensor(np.asarray(logits, np.float32), device=dev),
                         torch.as_tensor(np.asarray(T, np.float32), device=dev),
                         torch.as_tensor(np.asarray(K, np.int32), device=dev),
                         torch.as_tensor(np.asarray(P, np.float32), device=dev),
                         torch.as_tensor(np.asarray(u, np.float32), device=dev))
    return out.cpu().numpy()


def acceptable(x, T, K, P, u):
    x = np.asarray(x, np.float32).astype(np.float64)
    return {sampler.sample(x, T, K, min(1.0, pp), min(max(uu, 0.0), 1 - 1e-12))
            for pp in (P - EPS, P, P + EPS) for uu in (u - EPS, u, u + EPS)}


@pytest.mark.parametrize("vocab", [1, 7, 1000, 32000, 152064])
def test_rows_match_the_oracle(vocab):
    rng = np.random.default_rng(vocab)
    rows = 24 if vocab < 100000 else 6
    x = (rng.normal(size=(rows, vocab)) * rng.choice([0.5, 2, 6], size=(rows, 1))).astype(np.float32)
    T = rng.choice([0.0, 0.4, 0.7, 1.0, 1.6], size=rows).astype(np.float32)
    K = rng.choice([0, 1, 5, 50, vocab, vocab + 3], size=rows).astype(np.int32)
    P = rng.choice([0.2, 0.9, 0.99, 1.0], size=rows).astype(np.float32)
    u = rng.random(rows).astype(np.float32)
    got = run(x, T, K, P, u)
    for r in range(rows):
        ok = acceptable(x[r], float(T[r]), int(K[r]), float(P[r]), float(u[r]))
        assert int(got[r]) in ok, (r, float(T[r]), int(K[r]), float(P[r]), float(u[r]), got[r], ok)


def test_page_example_frequencies():
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                    "sampler_page_example.json")))
    N = 20000
    x = np.tile(np.array(g["logits"], np.float32), (N, 1))
    u = ((np.arange(N) + 0.5) / N).astype(np.float32)
    got = run(x, np.full(N, g["temperature"]), np.full(N, g["top_k"]), np.full(N, g["top_p"]), u)
    r = sampler.distribution(np.array(g["logits"], np.float32).astype(np.float64),
                             g["temperature"], g["top_k"], g["top_p"])
    counts = np.bincount(got, minlength=4)
    assert np.all(np.abs(counts - N * r) <= 2), (counts, N * r)
    assert counts[2] == 0 and counts[3] == 0


@pytest.mark.parametrize("T,K,P", [(1.0, 0, 1.0), (0.8, 40, 1.0), (1.2, 0, 0.8), (0.9, 100, 0.95)])
def test_stratified_frequencies(T, K, P):
    rng = np.random.default_rng(11)
    V, N = 500, 8000
    row = (rng.normal(size=V) * 2).astype(np.float32)
    x = np.tile(row, (N, 1))
    u = ((np.arange(N) + 0.5) / N).astype(np.float32)
    got = run(x, np.full(N, T), np.full(N, K), np.full(N, P), u)
    r = sampler.distribution(row.astype(np.float64), T, K, P)
    counts = np.bincount(got, minlength=V)
    assert np.all(np.abs(counts - N * r) <= 2), np.max(np.abs(counts - N * r))
    assert np.all(counts[r == 0] == 0)


def test_edges_greedy_ties_nan_and_neg_inf():
    x = np.array([[1.0, 3.0, 3.0, 2.0],          # greedy tie -> index 1
                  [np.nan, 1.0, np.nan, 0.5],    # NaN never drawn
                  [-np.inf, -np.inf, 0.0, -np.inf],
                  [5.0, 5.0, 1.0, 1.0],
                  [-0.0, 0.0, -1.0, -2.0],       # -0 and +0 are equal logits: greedy -> 0
                  [-1.0, 0.0, -0.0, -3.0]],      # top-k 1 keeps both zeros; u = 0.75 -> 2
                 np.float32)
    got = run(x, [0.0, 1.0, 1.0, 1.0, 0.0, 1.0], [0, 0, 0, 1, 0, 1], [1.0] * 6,
              [0.9, 0.5, 0.5, 0.75, 0.5, 0.75])
    assert got.tolist()[:3] == [1, 1, 2]
    assert got[3] == 1   # top-k 1 keeps both tied maxima; u = 0.75 draws the second
    assert got[4] == 0 and got[5] == 2
    for r in (4, 5):
        assert sampler.sample(x[r].astype(np.float64), [0.0, 1.0][r - 4], [0, 1][r - 4], 1.0,
                              0.5 if r == 4 else 0.75) == got[r]


@pytest.mark.parametrize("vocab", [4096, 152064])
def test_clustered_top_logits(vocab):
    # The largest logits sit next to each other in runs of 16, so a thread's
    # elements (four consecutive ones per 16-byte load) hold more than four Top-K
    # candidates: the kernel cannot take its candidates from the four it keeps
    # per thread and reads the row a second time.
    rng = np.random.default_rng(11)
    rows = 16
    x = rng.normal(size=(rows, vocab)).astype(np.float32)
    for r in range(rows):
        for start in rng.choice(vocab // 16 - 1, size=4, replace=False) * 16 + rng.integers(0, 4):
            x[r, start:start + 16] = 8 + rng.normal(size=16)
    T = rng.choice([0.5, 1.0], size=rows).astype(np.float32)
    K = rng.choice([1, 5, 20, 50, 64, 200], size=rows).astype(np.int32)
    P = rng.choice([0.5, 0.9, 1.0], size=rows).astype(np.float32)
    u = rng.random(rows).astype(np.float32)
    got = run(x, T, K, P, u)
    for r in range(rows):
        ok = acceptable(x[r], float(T[r]), int(K[r]), float(P[r]), float(u[r]))
        assert int(got[r]) in ok, (r, float(T[r]), int(K[r]), float(P[r]), float(u[r]), got[r], ok)


@pytest.mark.parametrize("vocab", [3000, 32000, 152064])
def test_top_k_across_the_threshold_paths(vocab):
    # Top-K of 2..1024 on the small-K path: up to 256 the lower bound of the
    # K-th largest logit comes from the warps' sorted maxima, above it from a
    # radix select over every thread's maximum; both must keep every survivor.
    rng = np.random.default_rng(vocab + 7)
    Ks = [2, 33, 100, 255, 256, 257, 500, 700, 1000, 1024]
    rows = len(Ks)
    x = (rng.normal(size=(rows, vocab)) * rng.choice([1.0, 4.0], size=(rows, 1))).astype(np.float32)
    T = np.full(rows, 1.0, np.float32)
    K = np.array(Ks, np.int32)
    P = rng.choice([0.9, 1.0], size=rows).astype(np.float32)
    u = rng.random(rows).astype(np.float32)
    got = run(x, T, K, P, u)
    for r in range(rows):
        ok = acceptable(x[r], float(T[r]), int(K[r]), float(P[r]), float(u[r]))
        assert int(got[r]) in ok, (r, int(K[r]), float(P[r]), float(u[r]), got[r], ok)


def test_same_inputs_same_tokens():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(64, 5000)).astype(np.float32)
    args = (x, np.full(64, 0.8), np.full(64, 50), np.full(64, 0.9), rng.random(64))
    assert np.array_equal(run(*args), run(*args))


def test_many_ties_take_the_general_path():
    # every logit equal: Top-K 50 keeps all 10000 (ties with the 50th), more
    # than the small-K path holds, so the radix path runs; the draw is uniform
    V, N = 10000, 20000
    x = np.zeros((N, V), np.float32)
    u = ((np.arange(N) + 0.5) / N).astype(np.float32)
    got = run(x, np.full(N, 1.0), np.full(N, 50), np.full(N, 1.0), u)
    counts = np.bincount(got, minlength=V)
    assert counts.min() >= 1 and counts.max() <= 3
    assert np.array_equal(got, (np.floor(u.astype(np.float64) * V)).astype(np.int64)) or \
        np.abs(got - np.floor(u.astype(np.float64) * V)).max() <= 1
