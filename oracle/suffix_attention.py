"""Oracle for tree-suffix attention with the log-sum-exp (LSE) merge.

TEST INFRASTRUCTURE ONLY, like the rest of this package: only the tests, the
package smoke check and the benchmark's CPU legs may use it.  Plain numpy in
float64, written for a reader to check by eye; no blocking or fusion.

Source.  "sgl-project/sglang pull request 37667: UNO", section
"Modifications": tree mode verifies its V nodes with EAGLE's cascade
attention, and UNO adds a fused kernel for the tree-suffix attention and the
LSE merge (the existing attention and state-merge path stays as fallback);
the shared attention backend uses the fused merge only for eligible UNO tree
verification.  The page prints no formula; the reading taken is the standard
cascade split:

* Each request's V tree nodes carry queries q_j and keys/values k_j, v_j.
  A node attends to the request's shared prefix (the context already in the
  KV cache) and, within the tree, to its ancestors and itself.
* The prefix part is computed elsewhere and arrives as a partial state: the
  normalised output o_p and its LSE l_p = log sum_i exp(s_i) over the prefix
  scores s_i = scale * <q, k_i>.
* The suffix part is the same over the tree keys the node may see:
  o_s, l_s.
* The merge weighs the partial outputs by exp(l): o = (e^l_p o_p + e^l_s o_s)
  / (e^l_p + e^l_s), l = log(e^l_p + e^l_s).  That equals attention over the
  union of the two key sets, which is what the pins check.

Shapes: q [V, H, d], k and v [V, Hkv, d] with H a multiple of Hkv (query head
h reads key/value head h // (H / Hkv)); parent [V] with parent[0] = -1 (the
root) and parent[j] < j; prefix state o_p [V, H, d], l_p [V, H] (l_p = -inf
for an empty prefix).  Natural logarithms throughout.
"""
from __future__ import annotations

import numpy as np


def tree_mask(parent) -> np.ndarray:
    """mask[j, i] is True when node i is node j or one of its ancestors."""
    parent = np.asarray(parent, dtype=np.int64)
    V = parent.size
    if V == 0 or parent[0] != -1 or np.any(parent[1:] < 0) or np.any(parent[1:] >= np.arange(1, V)):
        raise ValueError("parent must give node 0 as the root and a smaller index for every other node")
    mask = np.zeros((V, V), dtype=bool)
    for j in range(V):
        i = j
        while i >= 0:
            mask[j, i] = True
            i = parent[i]
    return mask


def _kv_head(H, Hkv):
    if Hkv < 1 or H % Hkv:
        raise ValueError("the query heads must be a multiple of the key/value heads")
    return np.arange(H) // (H // Hkv)


def suffix_attention(q, k, v, parent, scale):
    """Attention of each node over the tree keys it may see.  Returns
    (o_s [V, H, d], l_s [V, H]), float64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    V, H, d = q.shape
    kvh = _kv_head(H, k.shape[1])
    mask = tree_mask(parent)
    o = np.zeros((V, H, d))
    lse = np.zeros((V, H))
    for j in range(V):
        seen = np.nonzero(mask[j])[0]
        for h in range(H):
            s = scale * (k[seen, kvh[h], :] @ q[j, h, :])
            m = s.max()
            w = np.exp(s - m)
            total = w.sum()
            o[j, h] = (w @ v[seen, kvh[h], :]) / total
            lse[j, h] = m + np.log(total)
    return o, lse


def lse_merge(o1, l1, o2, l2):
    """Merge two partial attention states by their LSEs.  An LSE of -inf
    marks an empty part, which then carries no weight."""
    o1, o2 = np.asarray(o1, dtype=np.float64), np.asarray(o2, dtype=np.float64)
    l1, l2 = np.asarray(l1, dtype=np.float64), np.asarray(l2, dtype=np.float64)
    m = np.maximum(l1, l2)
    if np.any(np.isneginf(m)):
        raise ValueError("both parts empty")
    w1, w2 = np.exp(l1 - m), np.exp(l2 - m)
    o = (w1[..., None] * o1 + w2[..., None] * o2) / (w1 + w2)[..., None]
    return o, m + np.log(w1 + w2)


def suffix_attention_merge(q, k, v, parent, o_prefix, lse_prefix, scale):
    """The fused operation: tree-suffix attention, then the LSE merge with the
    prefix state.  Returns (o [V, H, d], lse [V, H])."""
    o_s, l_s = suffix_attention(q, k, v, parent, scale)
    return lse_merge(o_prefix, lse_prefix, o_s, l_s)


def prefix_attention(q, k_prefix, v_prefix, scale):
    """The prefix state a separate attention kernel would hand over: every
    node attends to all L prefix keys.  k_prefix, v_prefix [L, Hkv, d].
    Returns (o_p [V, H, d], l_p [V, H]); l_p = -inf and o_p = 0 when L = 0."""
    q = np.asarray(q, dtype=np.float64)
    kp = np.asarray(k_prefix, dtype=np.float64)
    vp = np.asarray(v_prefix, dtype=np.float64)
    V, H, d = q.shape
    if kp.shape[0] == 0:
        return np.zeros((V, H, d)), np.full((V, H), -np.inf)
    kvh = _kv_head(H, kp.shape[1])
    o = np.zeros((V, H, d))
    lse = np.zeros((V, H))
    for j in range(V):
        for h in range(H):
            s = scale * (kp[:, kvh[h], :] @ q[j, h, :])
            m = s.max()
            w = np.exp(s - m)
            o[j, h] = (w @ vp[:, kvh[h], :]) / w.sum()
            lse[j, h] = m + np.log(w.sum())
    return o, lse
