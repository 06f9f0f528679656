"""Two ranks over gloo on the CPU: request sharding and the max-over-ranks
timing reduction that bench.py uses.  Each rank runs the oracle on its own
shard with its global request offset; together they must reproduce the single
batch exactly (same filtered rows, draws and verified tokens)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from speculative_decoding_verification_filter_b200.inputs import WORKLOADS, linear_draft, linear_target

CYCLE = 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cycle(w, reqs, first):
    q = linear_draft(w, reqs)
    p = linear_target(w, reqs)
    sp = (w.temperature, w.top_k, w.top_p)
    rq = oracle.filter_softmax(q, w.dtype, *sp, rows_per_request=w.B, rng=(w.seed, CYCLE, first))
    ro = oracle.linear_verify(p, w.dtype, len(reqs), w.B, *sp, rq["sample"].reshape(len(reqs), w.B), rq["ids"],
                              rq["probs"], rq["count"], rng=(w.seed, CYCLE, first))
    return rq, ro


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    os.environ["RANK"], os.environ["WORLD_SIZE"] = str(rank), str(world)
    import bench
    dist = bench.init_dist(world, backend="gloo")
    try:
        w = WORKLOADS[0]
        first, reqs = bench.shard(rank, w.R)
        rq, ro = _cycle(w, reqs, first)
        parts = {}
        for name, arr in (("sample", rq["sample"]), ("tokens", ro["tokens"]), ("accept", ro["accept_len"])):
            t = torch.from_numpy(np.ascontiguousarray(arr).astype(np.int64))
            got = [torch.zeros_like(t) for _ in range(world)]
            dist.all_gather(got, t)
            parts[name] = torch.cat(got).numpy()
        slowest = bench.max_over_ranks([10.0 + rank, -rank], world, torch.device("cpu"))
        if rank == 0:
            out.put((parts, slowest))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reproduce_one_batch():
    oracle.build()
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    parts, slowest = out.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = WORKLOADS[0]
    rq, ro = _cycle(w, range(world * w.R), 0)
    assert np.array_equal(parts["sample"], rq["sample"].astype(np.int64))
    assert np.array_equal(parts["tokens"], ro["tokens"].astype(np.int64))
    assert np.array_equal(parts["accept"], ro["accept_len"].astype(np.int64))
    assert slowest == [11.0, 0.0]


def test_shard_offsets():
    import bench
    assert bench.shard(0, 64) == (0, range(0, 64))
    assert bench.shard(3, 64) == (192, range(192, 256))
