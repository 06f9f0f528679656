"""The seeded input generator follows its stated recipe (CPU).

Both the CUDA path and the oracle read what this module writes, so its layout
and its rounding are checked against independent routines: torch's binary32
to bfloat16 conversion (round to nearest even), regeneration of single rows,
and the statistics the recipe names (row standard deviation, planted peaks,
the second peak on about half the rows of the bimodal tree workload).
"""
import numpy as np
import torch

from speculative_decoding_verification_filter_b200.inputs import (WORKLOADS, base_row, fresh_row, linear_draft,
                                                                 linear_target, noise_row, to_bf16_bits,
                                                                 tree_target)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(200_000) * rng.choice([1e-3, 1.0, 1e3], 200_000)).astype(np.float32)
    # exact halfway cases between two bfloat16 values, both parities of the kept bit
    halves = (np.arange(1, 2000, dtype=np.uint32) << 16 | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, halves, -halves, np.array([0.0, -0.0, 1.0, -1.0], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(to_bf16_bits(x), ref)


def test_rows_regenerate_on_their_own_and_layout():
    w = WORKLOADS[0]  # tiny linear, fp32
    q, p = linear_draft(w), linear_target(w)
    assert q.shape == (w.R * w.B, w.vocab) and p.shape == (w.R * (w.B + 1), w.vocab)
    for r in range(w.R):
        for i in range(w.B):
            assert np.array_equal(q[r * w.B + i], base_row(w, r, i))
        for i in range(w.B + 1):
            assert np.array_equal(p[r * (w.B + 1) + i], base_row(w, r, i) + noise_row(w, r, i))
    # a subset of requests gives the same rows as the whole batch
    assert np.array_equal(linear_draft(w, [2]), q[2 * w.B:3 * w.B])
    assert np.array_equal(linear_target(w, [3, 1]),
                          np.concatenate([p[3 * (w.B + 1):4 * (w.B + 1)], p[1 * (w.B + 1):2 * (w.B + 1)]]))
    # distinct streams and indices give distinct rows
    assert not np.array_equal(base_row(w, 0, 0), base_row(w, 0, 1))
    assert not np.array_equal(base_row(w, 0, 0), noise_row(w, 0, 0) / w.noise * w.sigma)


def test_linear_workload_statistics():
    w = WORKLOADS[1]  # linear 8/1/8 bf16: sigma 1, peak +8, noise 0.7
    flat = w.with_(peak=0.0)
    for r in range(4):
        for i in range(3):
            x, y = base_row(w, r, i), base_row(flat, r, i)
            # one planted peak: the same Gaussian row with one element raised by the peak height
            diff = np.nonzero(x != y)[0]
            assert diff.size == 1 and abs(float(x[diff[0]] - y[diff[0]]) - w.peak) < 1e-5
            assert abs(y.std() - w.sigma) < 0.01 and abs(y.mean()) < 0.01
    n = noise_row(w, 0, 0)
    assert abs(n.std() - w.noise) < 0.01
    # bf16 storage of the target rows rounds base + noise
    t = linear_target(w, [0])
    assert t.dtype == np.uint16
    assert np.array_equal(t[0], to_bf16_bits(base_row(w, 0, 0) + noise_row(w, 0, 0)))


def test_bimodal_tree_workload_has_a_second_peak_on_about_half_the_rows():
    w = WORKLOADS[3]  # tree 8/16/8 bimodal: peak +8, second peak +6 on half the rows
    high = [int(np.sum(base_row(w, r, 0) > 4.5)) for r in range(w.R)]
    two = np.mean([h >= 2 for h in high])
    assert all(h >= 1 for h in high)
    assert 0.3 < two < 0.7


def test_tree_target_rows_follow_node_depths():
    w = WORKLOADS[3].with_(vocab=512, R=2)
    depth = np.array([[0, 1, 1, 2, 8, 3, -1, -1], [0, 1, 2, 3, 4, 5, 6, 7]])
    nn = np.array([6, 8])
    t = tree_target(w, depth, nn)
    for k in range(2):
        for j in range(w.V):
            d = int(depth[k, j]) if j < nn[k] else w.B
            base = base_row(w, k, d) if d < w.B else fresh_row(w, k, j)
            assert np.array_equal(t[k * w.V + j], to_bf16_bits(base + noise_row(w, k, j)))
