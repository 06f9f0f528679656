"""CPU models of two pieces of kernel arithmetic, checked against their plain
definitions on random inputs (host-side checks of the design; the GPU parity
tests check the kernels themselves).

- The finisher's top-k cut (csrc/uno_filter.cu, warp_select_topk): the keys'
  high halves are counted into 64 buckets of 2^shift values below the
  largest, the bucket holding the k-th key is found with a scan over lanes
  that each hold two buckets, and every key at or above that bucket's floor
  is kept.  It must keep the best k keys and whole buckets only.
- The suffix attention's ancestor masks (csrc/uno_suffix_attention.cu,
  build_ancestor_masks): each node walks up its parent links.  It must equal
  the definition in node order (a node's mask is its parent's mask plus
  itself; a node whose link does not point to an earlier node keeps itself
  alone and flags the tree).
"""
import random


def _clz32(x):
    return 32 - x.bit_length()


def _histogram_cut(keys, k):
    hi = [x >> 32 for x in keys]
    top, bot = max(hi), min(hi)
    span = top - bot
    shift = 0 if span < 64 else 26 - _clz32(span)
    assert span >> shift < 64
    hist = [0] * 64
    for h in hi:
        hist[(top - h) >> shift] += 1
    incl, acc = [], 0
    for lane in range(32):
        acc += hist[2 * lane] + hist[2 * lane + 1]
        incl.append(acc)
    first = next(lane for lane in range(32) if incl[lane] >= k)
    bstar = 2 * first + (0 if incl[first] - hist[2 * first + 1] >= k else 1)
    floor = max(0, top - ((bstar + 1) << shift) + 1)
    return [x for x in keys if x >= floor << 32]


def test_histogram_cut_keeps_the_best_k_in_whole_buckets():
    rng = random.Random(11)
    checked = 0
    for t in range(4000):
        k = rng.randint(1, 64)
        n = rng.randint(k + 9, 256)
        base = rng.randint(0x3F000000, 0xC0000000)
        mode = t % 4
        if mode == 0:  # a span under 64: one value per bucket
            his = [base + rng.randint(0, 63) for _ in range(n)]
        elif mode == 1:  # wide spans
            his = [base + rng.randint(0, 1 << rng.randint(6, 30)) for _ in range(n)]
        elif mode == 2:  # one value: everything in bucket 0
            his = [base] * n
        else:  # bf16-like values (low 16 bits zero)
            his = [base + (rng.randint(0, 300) << 16) for _ in range(n)]
        keys = list({(h << 32) | rng.getrandbits(32) for h in his})
        if len(keys) <= k + 8:
            continue
        kept = _histogram_cut(keys, k)
        assert len(kept) >= k
        assert set(sorted(keys, reverse=True)[:k]) <= set(kept)
        assert all(x in kept for x in keys if x >= min(kept))
        checked += 1
    assert checked > 3000


def _masks_in_node_order(parent, n):
    anc, bad = [], False
    for j in range(n):
        p = parent[j]
        ok = p == -1 if j == 0 else 0 <= p < j
        anc.append((anc[p] if ok and j > 0 else 0) | 1 << j)
        bad |= not ok
    return anc, bad


def _masks_by_walk(parent, n):
    anc, bad = [], False
    for j in range(n):
        mask, cur = 1 << j, j
        for _ in range(n):
            p = parent[cur]
            ok = p == -1 if cur == 0 else 0 <= p < cur
            if not ok and cur == j:
                bad = True
            if not ok or cur == 0:
                break
            mask |= 1 << p
            cur = p
        anc.append(mask)
    return anc, bad


def test_ancestor_walk_equals_the_node_order_definition():
    rng = random.Random(12)
    for _ in range(3000):
        n = rng.randint(1, 128)
        parent = [(rng.randint(-2, j + 2) if rng.random() < 0.05 else (rng.randint(0, j - 1) if j else -1))
                  for j in range(n)]
        assert _masks_by_walk(parent, n) == _masks_in_node_order(parent, n)
