"""A cycle captured once in a CUDA graph and replayed with a device cycle
word: each replay must draw that cycle's uniforms, i.e. equal the eager call
for the same cycle and the oracle, for cycles 0..3 (no repeated draws).

Tree chain: uno_filter_softmax -> uno_tree_topk_expand -> uno_tree_verify.
Linear chain: uno_linear_cycle (both layouts)."""
import numpy as np
import pytest
import torch

import oracle
from _parity import Events, compare_requests, np_of, to_device
from speculative_decoding_verification_filter_b200 import (LAYOUT_GENERIC, LAYOUT_TWO_PASS, uno_filter_softmax,
                                                          uno_linear_cycle, uno_tree_topk_expand, uno_tree_verify)
from speculative_decoding_verification_filter_b200.inputs import (Workload, linear_draft, linear_target,
                                                                 tree_draft, tree_target)

pytestmark = pytest.mark.gpu

CYCLES = (0, 1, 2, 3)


def _capture(fn, stream):
    """fn() warmed up on `stream`, then captured; returns (graph, outputs)."""
    with torch.cuda.stream(stream):
        for _ in range(2):
            fn()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        out = fn()
    return g, out


def _replay(g, cyc, c, stream):
    with torch.cuda.stream(stream):
        cyc.fill_(c)
        g.replay()
    stream.synchronize()


TREE_CASES = [
    Workload("graph tree 16/32/32 shape", "tree", R=1, B=16, K=32, V=32, vocab=8192, dtype="bf16", sigma=1.0,
             noise=0.7, peak=8.0, seed=42),
    Workload("graph tree 8/16/8 x6 bimodal", "tree", R=6, B=8, K=16, V=8, vocab=3001, dtype="bf16", sigma=1.0,
             noise=0.7, peak=8.0, second_peak=6.0, seed=7),
]


@pytest.mark.parametrize("w", TREE_CASES, ids=lambda w: w.name)
def test_tree_chain_graph_replays_draw_each_cycle(w):
    sp = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)
    q_np = tree_draft(w)
    rq = oracle.filter_softmax(q_np, w.dtype, w.temperature, w.top_k, w.top_p, rows_per_request=w.B)
    rt = oracle.tree_topk_expand(rq["ids"], rq["probs"], rq["count"], w.R, w.B, w.K, w.V)
    p_np = tree_target(w, rt["node_depth"], rt["num_nodes"])
    q, p = to_device(q_np, w.dtype), to_device(p_np, w.dtype)
    cyc = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.Stream()

    def chain():
        f = uno_filter_softmax(q, rows_per_request=w.B, **sp)
        t = uno_tree_topk_expand(f["ids"], f["probs"], f["count"], R=w.R, B=w.B, K=w.K, V=w.V)
        v = uno_tree_verify(p, t["node_token"], t["node_parent"], t["num_nodes"], R=w.R, B=w.B, V=w.V,
                            rng=(w.seed, cyc, 0), **sp)
        return t, v

    g, (gt, gv) = _capture(chain, stream)
    keys = ("tokens", "accept_len", "num_tokens", "path_nodes", "flags")
    seen = set()
    ev = Events(f"{w.name}: graph replays, cycles 0..3")
    for c in CYCLES:
        _replay(g, cyc, c, stream)
        for key in ("node_token", "node_parent", "num_nodes"):
            assert np.array_equal(np_of(gt[key]), rt[key]), key
        ref = oracle.tree_verify(p_np, w.dtype, w.R, w.B, w.V, w.temperature, w.top_k, w.top_p, rt["node_token"],
                                 rt["node_parent"], rt["num_nodes"], rng=(w.seed, c, 0))
        compare_requests(gv, ref, ev, keys)
        eager = uno_tree_verify(p, gt["node_token"], gt["node_parent"], gt["num_nodes"], R=w.R, B=w.B, V=w.V,
                                rng=(w.seed, c, 0), **sp)
        for key in keys:
            assert torch.equal(eager[key], gv[key]), (c, key)
        seen.add(np_of(gv["tokens"]).tobytes())
    ev.check()
    assert len(seen) > 1  # the replays did not repeat one cycle's draws
    del g


@pytest.mark.parametrize("layout", [LAYOUT_GENERIC, LAYOUT_TWO_PASS])
def test_linear_cycle_graph_replays_draw_each_cycle(layout):
    w = Workload("graph linear", "linear", R=16, B=6, vocab=6007, dtype="bf16", sigma=1.0, noise=0.7, peak=5.0,
                 seed=11)
    sp = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)
    q_np = linear_draft(w)
    p_full = linear_target(w)
    p_np = p_full if layout == LAYOUT_GENERIC else \
        np.ascontiguousarray(p_full.reshape(w.R, w.B + 1, -1)[:, :w.B]).reshape(w.R * w.B, -1)
    q, p = to_device(q_np, w.dtype), to_device(p_np, w.dtype)
    cyc = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.Stream()
    g, out = _capture(lambda: uno_linear_cycle(q, p, R=w.R, B=w.B, rng=(w.seed, cyc, 0), layout=layout, **sp),
                      stream)
    keys = ("drafts", "tokens", "num_accepted", "num_tokens", "flags")
    seen = set()
    ev = Events(f"{w.name} layout {layout}: graph replays, cycles 0..3")
    for c in CYCLES:
        _replay(g, cyc, c, stream)
        eager = uno_linear_cycle(q, p, R=w.R, B=w.B, rng=(w.seed, c, 0), layout=layout, **sp)
        for key in keys:
            assert torch.equal(eager[key], out[key]), (c, key)
        if layout == LAYOUT_TWO_PASS:
            r = oracle.linear_cycle(q_np, p_np, w.dtype, w.R, w.B, w.temperature, w.top_k, w.top_p, (w.seed, c, 0))
            ref = dict(tokens=r["tokens"], num_accepted=r["num_correct_drafts"], num_tokens=r["accept_len"],
                       flags=r["flags"], margin=r["margin"])
            compare_requests(out, ref, ev, ("tokens", "num_accepted", "num_tokens", "flags"))
        else:
            rq = oracle.filter_softmax(q_np, w.dtype, w.temperature, w.top_k, w.top_p, rows_per_request=w.B,
                                       rng=(w.seed, c, 0))
            r = oracle.linear_verify(p_np, w.dtype, w.R, w.B, w.temperature, w.top_k, w.top_p,
                                     rq["sample"].reshape(w.R, w.B), rq["ids"], rq["probs"], rq["count"],
                                     rng=(w.seed, c, 0))
            ref = dict(drafts=rq["sample"].reshape(w.R, w.B), tokens=r["tokens"], num_accepted=r["accept_len"],
                       num_tokens=r["num_tokens"],
                       flags=r["flags"] | np.bitwise_or.reduce(rq["flags"].reshape(w.R, w.B), axis=1),
                       margin=np.minimum(r["margin"], rq["margin"].reshape(w.R, w.B).min(axis=1)))
            compare_requests(out, ref, ev, keys)
        seen.add(np_of(out["tokens"]).tobytes())
    ev.check()
    assert len(seen) > 1
    del g
