"""Helpers shared by the GPU parity tests: move seeded inputs to the device,
run the CUDA path, and compare it with the oracle element by element.

Bar (stated, not from the pages): token ids, counts, accept lengths and tree
nodes bit-exact; filtered probabilities within PROB_ATOL; a decision may differ
only where the oracle reports it within oracle.BOUNDARY_EPS of its flip point
(a boundary event), and such events must stay below 1e-5 of the decisions.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

PROB_ATOL = 1e-6  # tighter than the 1e-5 (fp32) / 2e-3 (bf16) bar the task states


def to_device(arr: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).cuda()


def np_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


# (name, decisions, boundary events) of every named check in this session;
# conftest prints them after the run and, when UNO_PARITY_EVENTS names a
# file, writes them there as JSON
RECORDS: list = []


class Events:
    """Counts decisions and excused boundary events."""

    def __init__(self, name=None):
        self.name = name
        self.decisions = 0
        self.boundary = 0

    def check(self, max_rate=1e-5):
        if self.name is not None:
            RECORDS.append(dict(check=self.name, decisions=self.decisions, boundary_events=self.boundary))
        if self.decisions:
            assert self.boundary <= max(0, int(max_rate * self.decisions)), (self.boundary, self.decisions)


def compare_filter(gpu: dict, ref: dict, events: Events, rows=None, sample=False):
    """Compare compact filter outputs row by row (rows: oracle row -> gpu row)."""
    g = {k: np_of(v) for k, v in gpu.items()}
    n = ref["count"].shape[0]
    idx = np.arange(n) if rows is None else np.asarray(rows)
    for i in range(n):
        gi = idx[i]
        events.decisions += 1
        near = ref["margin"][i] < oracle.BOUNDARY_EPS
        same = (g["count"][gi] == ref["count"][i]
                and np.array_equal(g["ids"][gi, :ref["count"][i]], ref["ids"][i, :ref["count"][i]]))
        if not same:
            assert near, f"row {i}: count/ids differ away from a boundary"
            events.boundary += 1
            continue
        c = ref["count"][i]
        assert np.max(np.abs(g["probs"][gi, :c] - ref["probs"][i, :c]), initial=0.0) <= PROB_ATOL, i
        assert np.all(g["ids"][gi, c:] == -1), i
        assert int(g["flags"][gi]) == int(ref["flags"][i]), i
        if sample:
            if g["sample"][gi] != ref["sample"][i]:
                assert near, f"row {i}: sample differs away from a boundary"
                events.boundary += 1


def compare_requests(gpu: dict, ref: dict, events: Events, keys, reqs=None):
    g = {k: np_of(v) for k, v in gpu.items()}
    n = ref["margin"].shape[0]
    idx = np.arange(n) if reqs is None else np.asarray(reqs)
    for i in range(n):
        gi = idx[i]
        events.decisions += 1
        same = all(np.array_equal(np.asarray(g[k][gi]).astype(np.int64), np.asarray(ref[k][i]).astype(np.int64))
                   for k in keys)
        if not same:
            assert ref["margin"][i] < oracle.BOUNDARY_EPS, (
                f"request {i} differs away from a boundary: " +
                "; ".join(f"{k}: gpu {g[k][gi]} ref {ref[k][i]}" for k in keys))
            events.boundary += 1
