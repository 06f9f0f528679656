"""The oracle's side of the full-size parity tests, one request per job, run
in a pool of spawned worker processes (spawned, not forked: the parent has
already used the GPU).  Each job regenerates its request's seeded rows itself,
so only small arrays cross between processes."""
from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np

import oracle
from speculative_decoding_verification_filter_b200.inputs import (WORKLOADS, linear_draft, linear_target,
                                                                 tree_draft, tree_target)


def pool_map(fn, jobs):
    """fn over jobs in spawned workers (results in job order)."""
    jobs = list(jobs)
    n = max(1, min(len(jobs), 32, os.cpu_count() or 1))
    if n == 1:
        return [fn(j) for j in jobs]
    with ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn")) as ex:
        return list(ex.map(fn, jobs, chunksize=1))


def linear_request(job):
    """Oracle results of one linear request: the draft filter and proposal
    draw, the verification of the B + 1 target rows (generic layout) and, if
    asked, the two-pass cycle over the first B target rows."""
    cfg, r, cycle, two_pass = job
    w = WORKLOADS[cfg]
    rng = (w.seed, cycle, r)
    q = linear_draft(w, [r])
    p = linear_target(w, [r])
    rq = oracle.filter_softmax(q, w.dtype, w.temperature, w.top_k, w.top_p, rows_per_request=w.B, rng=rng)
    ro = oracle.linear_verify(p, w.dtype, 1, w.B, w.temperature, w.top_k, w.top_p, rq["sample"].reshape(1, w.B),
                              rq["ids"], rq["probs"], rq["count"], rng=rng)
    out = dict(rq=rq, ro=ro)
    if two_pass:
        p2 = np.ascontiguousarray(p.reshape(w.B + 1, -1)[:w.B])
        out["rc"] = oracle.linear_cycle(q, p2, w.dtype, 1, w.B, w.temperature, w.top_k, w.top_p, rng)
    return out


def tree_request_tree(job):
    """The oracle's filtered marginals and V-node tree of one tree request."""
    cfg, r = job
    w = WORKLOADS[cfg]
    q = tree_draft(w, [r])
    rq = oracle.filter_softmax(q, w.dtype, w.temperature, w.top_k, w.top_p, rows_per_request=w.B)
    rt = oracle.tree_topk_expand(rq["ids"], rq["probs"], rq["count"], 1, w.B, w.K, w.V)
    return dict(rq=rq, rt=rt)


def tree_request_verify(job):
    """Target-only verification of one tree request over its node rows."""
    cfg, r, cycle, node_token, node_parent, node_depth, num_nodes = job
    w = WORKLOADS[cfg]
    p = tree_target(w, node_depth, num_nodes, requests=[r])
    return oracle.tree_verify(p, w.dtype, 1, w.B, w.V, w.temperature, w.top_k, w.top_p, node_token, node_parent,
                              num_nodes, rng=(w.seed, cycle, r))
