"""The five workloads at full size, in the launch configuration the benchmark
times (one call over the whole batch), checked against the oracle: every
request of the small workloads, sampled requests of the large ones."""
import numpy as np
import pytest
import torch

import oracle
from _parity import Events, compare_filter, compare_requests, np_of, to_device
from speculative_decoding_verification_filter_b200 import (uno_filter_softmax, uno_linear_verify,
                                                          uno_tree_topk_expand, uno_tree_verify)
from speculative_decoding_verification_filter_b200.inputs import (WORKLOADS, linear_draft, linear_target,
                                                                 tree_draft, tree_target)

pytestmark = pytest.mark.gpu

CYCLE = 3


def _upload(w, maker, nrows_per_req, chunk=32):
    """Generate a workload's rows request-chunk by request-chunk into one
    device tensor (keeps host memory small for the 10 GB workload)."""
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    out = torch.empty((w.R * nrows_per_req, w.vocab), dtype=tdt, device="cuda")
    for c0 in range(0, w.R, chunk):
        reqs = range(c0, min(w.R, c0 + chunk))
        rows = maker(w, reqs)
        out[c0 * nrows_per_req:(c0 + len(reqs)) * nrows_per_req] = to_device(rows, w.dtype)
    return out


def _sampled(R, seed):
    rng = np.random.default_rng(seed)
    return sorted(set([0, 1, R // 2, R - 1] + rng.integers(0, R, 2).tolist()))


@pytest.mark.parametrize("cfg", [0, 1, 4])
def test_linear_workload(cfg):
    w = WORKLOADS[cfg]
    sp = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)
    rng = (w.seed, CYCLE)
    q = _upload(w, linear_draft, w.B)
    gq = uno_filter_softmax(q, rows_per_request=w.B, rng=rng, **sp)
    del q
    p = _upload(w, linear_target, w.B + 1)
    g = uno_linear_verify(p, gq["sample"].reshape(w.R, w.B), gq["ids"], gq["probs"], gq["count"], R=w.R, B=w.B,
                          rng=rng, **sp)
    del p
    torch.cuda.synchronize()
    ev = Events()
    reqs = range(w.R) if w.R <= 8 else _sampled(w.R, cfg)
    for r in reqs:
        q_np = linear_draft(w, [r])
        rq = oracle.filter_softmax(q_np, w.dtype, w.temperature, w.top_k, w.top_p, rows_per_request=w.B,
                                   rng=(w.seed, CYCLE, r))
        compare_filter(gq, rq, ev, rows=range(r * w.B, (r + 1) * w.B), sample=True)
        p_np = linear_target(w, [r])
        ro = oracle.linear_verify(p_np, w.dtype, 1, w.B, w.temperature, w.top_k, w.top_p,
                                  rq["sample"].reshape(1, w.B), rq["ids"], rq["probs"], rq["count"],
                                  rng=(w.seed, CYCLE, r))
        compare_requests(g, ro, ev, ("tokens", "accept_len", "num_tokens", "flags"), reqs=[r])
    ev.check()
    acc = np_of(g["accept_len"])
    assert np.all((acc >= 0) & (acc <= w.B)) and np.all(np_of(g["num_tokens"]) == acc + 1)


@pytest.mark.parametrize("cfg", [2, 3])
def test_tree_workload(cfg):
    w = WORKLOADS[cfg]
    sp = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)
    rng = (w.seed, CYCLE)
    q_np = tree_draft(w)
    gq = uno_filter_softmax(to_device(q_np, w.dtype), rows_per_request=w.B, **sp)
    gt = uno_tree_topk_expand(gq["ids"], gq["probs"], gq["count"], R=w.R, B=w.B, K=w.K, V=w.V)
    # the oracle builds its own trees from its own filtered marginals; the
    # target rows (one per node) come from the oracle's trees
    rq = oracle.filter_softmax(q_np, w.dtype, w.temperature, w.top_k, w.top_p, rows_per_request=w.B)
    ev = Events()
    compare_filter(gq, rq, ev)
    rt = oracle.tree_topk_expand(rq["ids"], rq["probs"], rq["count"], w.R, w.B, w.K, w.V)
    for key in ("node_token", "node_parent", "node_depth", "node_score", "num_nodes"):
        assert np.array_equal(np_of(gt[key]), rt[key]), key
    p_np = tree_target(w, rt["node_depth"], rt["num_nodes"])
    g = uno_tree_verify(to_device(p_np, w.dtype), gt["node_token"], gt["node_parent"], gt["num_nodes"], R=w.R,
                        B=w.B, V=w.V, rng=rng, **sp)
    torch.cuda.synchronize()
    reqs = range(w.R) if w.R <= 8 else _sampled(w.R, cfg)
    for r in reqs:
        ro = oracle.tree_verify(p_np[r * w.V:(r + 1) * w.V], w.dtype, 1, w.B, w.V, w.temperature, w.top_k, w.top_p,
                                rt["node_token"][r:r + 1], rt["node_parent"][r:r + 1], rt["num_nodes"][r:r + 1],
                                rng=(w.seed, CYCLE, r))
        compare_requests(g, ro, ev, ("tokens", "accept_len", "num_tokens", "path_nodes", "flags"), reqs=[r])
    ev.check()
