"""Seeded synthetic logits shaped like the UNO workloads.

This module only draws random numbers; it holds none of the method's
arithmetic (no filtering, softmax, sampling or tree logic).  Both the CUDA
path and the oracle consume what it produces.

The UNO PR page ("Validation": H200 math evaluation) runs Qwen3-8B (vocabulary
151,936) at temperature 1, top-k 50, top-p 0.95, seed 42, with linear 8/1/8 at
64 concurrent requests and tree 16/32/32 at one request; the smoke table adds
tree 8/16/8.  No model weights or datasets are used here: each row is
independent Gaussian noise with planted peaks, which stands in for the model's
logits.

Every row comes from its own numpy ``Philox`` bit generator keyed by
(config seed, stream, request, index), so any row can be regenerated on its
own (the tests check sampled requests of the full-size workloads that way).

Layout: a linear request r owns base rows g[r][0..B]; its draft marginals are
q_i = g[r][i] (i < B) and its target rows are p_i = g[r][i] + n[r][i]
(i <= B).  A tree request owns draft marginals q_d = g[r][d] (d < B); the target
row of tree node j at depth t is g[r][t] + n[r][j] when t < B (the marginal
that proposes j's children) and a fresh row f[r][j] + n[r][j] at depth B.
"""
from __future__ import annotations

import concurrent.futures as _cf
import os
from dataclasses import dataclass, field, replace

import numpy as np

STREAM_BASE, STREAM_NOISE, STREAM_FRESH = 1, 2, 3


@dataclass(frozen=True)
class Workload:
    name: str
    mode: str  # "linear" or "tree"
    R: int
    B: int
    vocab: int
    dtype: str  # "f32" or "bf16"
    sigma: float  # std of the base rows
    noise: float  # std of the target-minus-draft noise
    peak: float = 0.0  # height of the planted peak (0: none)
    second_peak: float = 0.0  # second peak on half the rows (0: none)
    temperature: float = 1.0
    top_k: int = 50
    top_p: float = 0.95
    seed: int = 42
    K: int = 1
    V: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def q_rows(self) -> int:
        return self.R * self.B

    @property
    def p_rows(self) -> int:
        return self.R * (self.B + 1) if self.mode == "linear" else self.R * self.V

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def logit_bytes(self) -> int:
        """Bytes of draft plus target logits one cycle reads once."""
        return (self.q_rows + self.p_rows) * self.vocab * self.elem_bytes

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads, in order: tiny linear; linear 8/1/8 at 64 requests;
# tree 16/32/32 at one request; tree 8/16/8 at 64 requests (bimodal rows);
# linear stress at 512 requests with B = 16, fp32, T = 0.7.
WORKLOADS = [
    Workload("tiny linear 4/1/4 fp32 vocab 1024", "linear", R=4, B=4, vocab=1024, dtype="f32",
             sigma=2.0, noise=0.5, seed=42),
    Workload("linear 8/1/8 bf16 x64", "linear", R=64, B=8, vocab=151936, dtype="bf16",
             sigma=1.0, noise=0.7, peak=8.0, seed=42),
    Workload("tree 16/32/32 bf16 x1", "tree", R=1, B=16, K=32, V=32, vocab=151936, dtype="bf16",
             sigma=1.0, noise=0.7, peak=8.0, seed=42),
    Workload("tree 8/16/8 bf16 x64 bimodal", "tree", R=64, B=8, K=16, V=8, vocab=151936, dtype="bf16",
             sigma=1.0, noise=0.7, peak=8.0, second_peak=6.0, seed=7),
    Workload("linear 16/1/16 fp32 x512 stress", "linear", R=512, B=16, vocab=151936, dtype="f32",
             sigma=1.5, noise=1.0, temperature=0.7, seed=123),
]


def _gen(w: Workload, stream: int, request: int, index: int) -> np.random.Generator:
    key = np.array([w.seed & 0xFFFFFFFFFFFFFFFF,
                    (stream << 56) | (request << 20) | index], dtype=np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def base_row(w: Workload, request: int, index: int) -> np.ndarray:
    g = _gen(w, STREAM_BASE, request, index)
    x = g.standard_normal(w.vocab, dtype=np.float32)
    x *= np.float32(w.sigma)
    if w.peak:
        x[int(g.integers(w.vocab))] += np.float32(w.peak)
    if w.second_peak and int(g.integers(2)) == 0:
        x[int(g.integers(w.vocab))] += np.float32(w.second_peak)
    return x


def fresh_row(w: Workload, request: int, node: int) -> np.ndarray:
    g = _gen(w, STREAM_FRESH, request, node)
    x = g.standard_normal(w.vocab, dtype=np.float32)
    x *= np.float32(w.sigma)
    if w.peak:
        x[int(g.integers(w.vocab))] += np.float32(w.peak)
    return x


def noise_row(w: Workload, request: int, index: int) -> np.ndarray:
    g = _gen(w, STREAM_NOISE, request, index)
    x = g.standard_normal(w.vocab, dtype=np.float32)
    x *= np.float32(w.noise)
    return x


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """binary32 -> bfloat16 bit patterns, round to nearest even (inputs are finite)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def encode(w: Workload, x: np.ndarray) -> np.ndarray:
    return to_bf16_bits(x) if w.dtype == "bf16" else np.ascontiguousarray(x, dtype=np.float32)


def _storage_dtype(w: Workload):
    return np.uint16 if w.dtype == "bf16" else np.float32


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def _fill(out: np.ndarray, jobs) -> np.ndarray:
    """Run jobs (row index, zero-arg row maker) on a thread pool into out."""
    def run(job):
        i, make = job
        out[i] = make()
    with _cf.ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(run, jobs))
    return out


def linear_draft(w: Workload, requests=None) -> np.ndarray:
    """Draft marginal logits [len(requests) * B, vocab] (storage dtype)."""
    reqs = list(range(w.R)) if requests is None else list(requests)
    out = np.empty((len(reqs) * w.B, w.vocab), dtype=_storage_dtype(w))
    jobs = [(k * w.B + i, (lambda r=r, i=i: encode(w, base_row(w, r, i))))
            for k, r in enumerate(reqs) for i in range(w.B)]
    return _fill(out, jobs)


def linear_target(w: Workload, requests=None) -> np.ndarray:
    """Target logits [len(requests) * (B+1), vocab] (storage dtype)."""
    reqs = list(range(w.R)) if requests is None else list(requests)
    out = np.empty((len(reqs) * (w.B + 1), w.vocab), dtype=_storage_dtype(w))
    jobs = [(k * (w.B + 1) + i, (lambda r=r, i=i: encode(w, base_row(w, r, i) + noise_row(w, r, i))))
            for k, r in enumerate(reqs) for i in range(w.B + 1)]
    return _fill(out, jobs)


def tree_draft(w: Workload, requests=None) -> np.ndarray:
    return linear_draft(w, requests)


def tree_target(w: Workload, node_depth: np.ndarray, num_nodes: np.ndarray, requests=None) -> np.ndarray:
    """Target logits [len(requests) * V, vocab], one row per tree node.

    node_depth / num_nodes are per request (rows of the given requests, in the
    same order).  Rows of absent nodes (index >= num_nodes) are fresh rows."""
    reqs = list(range(w.R)) if requests is None else list(requests)
    node_depth = np.asarray(node_depth).reshape(len(reqs), w.V)
    num_nodes = np.asarray(num_nodes).reshape(len(reqs))
    out = np.empty((len(reqs) * w.V, w.vocab), dtype=_storage_dtype(w))

    def make(r, j, t):
        if 0 <= t < w.B:
            return encode(w, base_row(w, r, t) + noise_row(w, r, j))
        return encode(w, fresh_row(w, r, j) + noise_row(w, r, j))

    jobs = []
    for k, r in enumerate(reqs):
        for j in range(w.V):
            t = int(node_depth[k, j]) if j < int(num_nodes[k]) else w.B
            jobs.append((k * w.V + j, (lambda r=r, j=j, t=t: make(r, j, t))))
    return _fill(out, jobs)
