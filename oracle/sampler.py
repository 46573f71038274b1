"""Plain NumPy float64 definition of next-token sampling (TEST INFRASTRUCTURE ONLY).

Source: "vLLM 基本原理", section "FlashInfer 采样器": the model's logits go
through temperature scaling, Top-K (keep the K most probable tokens), Top-P
(keep the most probable tokens until their cumulative probability reaches P)
and a random draw from what is left; a fused kernel does these without
sorting the logits and is statistically equivalent to the sort-based sampler.

The definition, with the readings taken where the page is silent:

1. ``T <= 0`` means greedy: the token with the largest logit (the lowest index
   among equal ones).  Otherwise probabilities ``p_i ∝ exp(x_i / T)``.
2. Top-K (``0 < K < V``): keep every token whose logit is at least the K-th
   largest logit (tokens tied with it are all kept).
3. Top-P (``P < 1``): renormalise over the kept set; take the tokens in
   decreasing logit order and keep the shortest run whose probability reaches
   ``P`` -- with every token tied with the last one of that run kept too.
4. Draw: renormalise over what is kept and return the first token, in vocabulary
   order, whose cumulative probability exceeds ``u`` (the caller's uniform
   number in [0, 1)), i.e. inverse-CDF sampling in index order.  Every kept
   token is drawn with its renormalised probability.
"""
from __future__ import annotations

import numpy as np


def kept_set(logits, temperature, top_k, top_p):
    """Boolean mask of the tokens that survive Top-K and Top-P, and the
    probabilities (float64) before any renormalisation."""
    x = np.asarray(logits, np.float64)
    V = x.shape[0]
    if temperature <= 0:
        mask = np.zeros(V, bool)
        mask[int(np.argmax(x))] = True  # argmax returns the lowest index of a tie
        p = mask.astype(np.float64)
        return mask, p
    z = x / temperature
    p = np.exp(z - z.max())
    p /= p.sum()
    mask = np.ones(V, bool)
    if 0 < top_k < V:
        kth = np.sort(x)[::-1][top_k - 1]
        mask &= x >= kth
    if top_p < 1:
        q = np.where(mask, p, 0.0)
        q /= q.sum()
        order = np.argsort(-x, kind="stable")
        order = order[mask[order]]
        cum = np.cumsum(q[order])
        n = int(np.searchsorted(cum, top_p))          # first run reaching top_p
        n = min(n, len(order) - 1)
        cut = x[order[n]]
        mask &= x >= cut
    return mask, p


def sample(logits, temperature, top_k, top_p, u):
    """The token drawn for uniform ``u`` (see the module docstring)."""
    mask, p = kept_set(logits, temperature, top_k, top_p)
    if temperature <= 0:
        return int(np.flatnonzero(mask)[0])
    r = np.where(mask, p, 0.0)
    r /= r.sum()
    cdf = np.cumsum(r)
    i = int(np.searchsorted(cdf, u, side="right"))   # first index whose cdf exceeds u
    # the cdf only rises at kept tokens, so index i is kept; rounding can only
    # push u past the last one, which is then the answer
    return i if i < len(cdf) else int(np.flatnonzero(mask)[-1])


def distribution(logits, temperature, top_k, top_p):
    """The renormalised probability of each token under the definition."""
    mask, p = kept_set(logits, temperature, top_k, top_p)
    r = np.where(mask, p, 0.0)
    return r / r.sum()
