"""Definitions the oracle is pinned against, written with library routines.

These do not restate the oracle's code: top-k comes from ``numpy.lexsort``, the
softmax from ``scipy.special.softmax``, the top-p cut from its defining
property (the shortest prefix, in logit-descending order, whose renormalised
top-k mass reaches top_p) via ``numpy.cumsum``/``searchsorted``.  Under the
"joint" order the prefix mass is read from the softmax of the whole row, and
the kept prefix is then cut to the top-k.
"""
from __future__ import annotations

import numpy as np
from scipy import special, stats


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _prefix_mass(l: np.ndarray, idx: np.ndarray, temperature: float, top_k: int, order: str) -> np.ndarray:
    """Probabilities, in logit-descending order, whose running sum the top-p
    cut reads: the renormalised top-k set, or the whole row's softmax."""
    if order == "joint":
        return special.softmax(l / temperature)[idx]
    assert order == "topk_first", order
    return special.softmax(l[idx[:min(top_k, l.size)]] / temperature)


def filtered_dist(logits: np.ndarray, temperature: float, top_k: int, top_p: float,
                  order: str = "topk_first") -> np.ndarray:
    """Dense filtered distribution of one finite row (float64, sums to 1)."""
    l = np.asarray(logits, dtype=np.float64)
    n = l.size
    idx = np.lexsort((np.arange(n), -l))  # logit desc, id asc
    k = min(top_k, n)
    top = idx[:k]
    out = np.zeros(n)
    if temperature == 0:
        out[top[0]] = 1.0
        return out
    if order == "joint" and top_p < 1.0:
        c = np.cumsum(_prefix_mass(l, idx, temperature, top_k, order))
        L = min(max(int(np.searchsorted(c, top_p, side="left")) + 1, 1), k)
        top = idx[:L]
        p = special.softmax(l[top] / temperature)
        out[top] = p
        return out
    p = special.softmax(l[top] / temperature)
    if top_p < 1.0:
        c = np.cumsum(p)
        # shortest prefix whose mass reaches top_p
        L = int(np.searchsorted(c, top_p, side="left")) + 1
        L = min(max(L, 1), k)
        top, p = top[:L], p[:L]
        p = p / p.sum()
    out[top] = p
    return out


def top_p_margin(logits: np.ndarray, temperature: float, top_k: int, top_p: float,
                 order: str = "topk_first") -> float:
    """Distance of the top-p cut from flipping (min |prefix mass - top_p|)."""
    l = np.asarray(logits, dtype=np.float64)
    idx = np.lexsort((np.arange(l.size), -l))
    k = min(top_k, l.size)
    if temperature == 0 or top_p >= 1.0:
        return np.inf
    p = _prefix_mass(l, idx, temperature, top_k, order)[:k]
    c = np.cumsum(p)[:-1]
    return float(np.min(np.abs(c - top_p))) if c.size else np.inf


def chi2_pvalue(counts: np.ndarray, probs: np.ndarray, min_expected: float = 5.0) -> float:
    """Pearson chi-square goodness of fit, pooling cells with small expectation."""
    counts = np.asarray(counts, dtype=np.float64).ravel()
    probs = np.asarray(probs, dtype=np.float64).ravel()
    n = counts.sum()
    assert abs(probs.sum() - 1.0) < 1e-9, probs.sum()
    # any observation in a zero-probability cell is an outright failure
    if np.any((probs == 0) & (counts > 0)):
        return 0.0
    exp = probs * n
    big = exp >= min_expected
    obs_b, exp_b = counts[big], exp[big]
    small_obs, small_exp = counts[~big & (probs > 0)].sum(), exp[~big & (probs > 0)].sum()
    if small_exp > 0:
        obs_b = np.append(obs_b, small_obs)
        exp_b = np.append(exp_b, small_exp)
    if obs_b.size < 2:
        return 1.0
    return float(stats.chisquare(obs_b, exp_b).pvalue)
