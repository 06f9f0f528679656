"""The five workloads at full size, in the launch configuration the benchmark
times (one call over the whole batch), checked against the oracle request by
request: every request of the tiny, linear 8/1/8, tree 16/32/32 and tree
8/16/8 workloads, and 65 requests spread over the 512 of the stress workload.
The linear workloads run three ways: uno_filter_softmax then
uno_linear_verify, uno_linear_cycle in the generic layout, and
uno_linear_cycle in the two-pass layout.  Decision and boundary-event counts
of every check are printed after the run (and written to the file that
UNO_PARITY_EVENTS names)."""
import numpy as np
import pytest
import torch

import _oracle_jobs as jobs
from _parity import Events, compare_filter, compare_requests, np_of, to_device
from speculative_decoding_verification_filter_b200 import (LAYOUT_GENERIC, LAYOUT_TWO_PASS, uno_filter_softmax,
                                                          uno_linear_cycle, uno_linear_verify, uno_tree_topk_expand,
                                                          uno_tree_verify)
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


def _checked_requests(w):
    """Every request, or (above 64 requests) every eighth one and the last."""
    if w.R <= 64:
        return list(range(w.R))
    return sorted(set(range(0, w.R, 8)) | {w.R - 1})


@pytest.mark.parametrize("cfg", [0, 1, 4])
def test_linear_workload(cfg):
    w = WORKLOADS[cfg]
    sp = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)
    rng = (w.seed, CYCLE)
    q = _upload(w, linear_draft, w.B)
    p = _upload(w, linear_target, w.B + 1)
    gq = uno_filter_softmax(q, rows_per_request=w.B, rng=rng, **sp)
    g = uno_linear_verify(p, gq["sample"].reshape(w.R, w.B), gq["ids"], gq["probs"], gq["count"], R=w.R, B=w.B,
                          rng=rng, **sp)
    gc = uno_linear_cycle(q, p, R=w.R, B=w.B, rng=rng, layout=LAYOUT_GENERIC, **sp)
    # the two-pass layout reads B target rows per request: the first B of each
    p2 = p.view(w.R, w.B + 1, w.vocab)[:, :w.B].contiguous().view(w.R * w.B, w.vocab)
    del p
    g2 = uno_linear_cycle(q, p2, R=w.R, B=w.B, rng=rng, layout=LAYOUT_TWO_PASS, **sp)
    del q, p2
    torch.cuda.synchronize()
    reqs = _checked_requests(w)
    refs = jobs.pool_map(jobs.linear_request, [(cfg, r, CYCLE, True) for r in reqs])
    ev_f, ev_v = Events(f"{w.name}: filter rows"), Events(f"{w.name}: uno_linear_verify requests")
    ev_c, ev_2 = Events(f"{w.name}: uno_linear_cycle generic"), Events(f"{w.name}: uno_linear_cycle two-pass")
    for r, ref in zip(reqs, refs):
        rq, ro, rc = ref["rq"], ref["ro"], ref["rc"]
        compare_filter(gq, rq, ev_f, rows=range(r * w.B, (r + 1) * w.B), sample=True)
        compare_requests(g, ro, ev_v, ("tokens", "accept_len", "num_tokens", "flags"), reqs=[r])
        gen = dict(tokens=ro["tokens"], num_accepted=ro["accept_len"], num_tokens=ro["num_tokens"],
                   flags=ro["flags"] | np.bitwise_or.reduce(rq["flags"]).reshape(1),
                   drafts=rq["sample"].reshape(1, w.B), margin=np.minimum(ro["margin"], rq["margin"].min()))
        compare_requests(gc, gen, ev_c, ("drafts", "tokens", "num_accepted", "num_tokens", "flags"), reqs=[r])
        two = dict(tokens=rc["tokens"], num_accepted=rc["num_correct_drafts"], num_tokens=rc["accept_len"],
                   flags=rc["flags"], margin=rc["margin"])
        compare_requests(g2, two, ev_2, ("tokens", "num_accepted", "num_tokens", "flags"), reqs=[r])
    for ev in (ev_f, ev_v, ev_c, ev_2):
        ev.check()
    acc = np_of(g["accept_len"])
    assert np.all((acc >= 0) & (acc <= w.B)) and np.all(np_of(g["num_tokens"]) == acc + 1)


@pytest.mark.parametrize("cfg", [2, 3])
def test_tree_workload(cfg):
    w = WORKLOADS[cfg]
    sp = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)
    rng = (w.seed, CYCLE)
    q = _upload(w, tree_draft, w.B)
    gq = uno_filter_softmax(q, rows_per_request=w.B, **sp)
    del q
    gt = uno_tree_topk_expand(gq["ids"], gq["probs"], gq["count"], R=w.R, B=w.B, K=w.K, V=w.V)
    torch.cuda.synchronize()
    # the oracle builds its own trees from its own filtered marginals; the
    # target rows (one per node) come from the oracle's trees
    trees = jobs.pool_map(jobs.tree_request_tree, [(cfg, r) for r in range(w.R)])
    ev_f, ev_v = Events(f"{w.name}: filter rows"), Events(f"{w.name}: uno_tree_verify requests")
    for r, t in enumerate(trees):
        compare_filter(gq, t["rq"], ev_f, rows=range(r * w.B, (r + 1) * w.B))
    rt = {key: np.concatenate([t["rt"][key] for t in trees])
          for key in ("node_token", "node_parent", "node_depth", "node_score", "num_nodes")}
    for key in rt:
        assert np.array_equal(np_of(gt[key]), rt[key]), key
    p = _upload(w, lambda w_, reqs: tree_target(w_, rt["node_depth"][list(reqs)], rt["num_nodes"][list(reqs)],
                                                requests=reqs), w.V)
    g = uno_tree_verify(p, gt["node_token"], gt["node_parent"], gt["num_nodes"], R=w.R, B=w.B, V=w.V, rng=rng, **sp)
    torch.cuda.synchronize()
    del p
    vjobs = [(cfg, r, CYCLE, rt["node_token"][r:r + 1], rt["node_parent"][r:r + 1], rt["node_depth"][r:r + 1],
              rt["num_nodes"][r:r + 1]) for r in range(w.R)]
    for r, ro in enumerate(jobs.pool_map(jobs.tree_request_verify, vjobs)):
        compare_requests(g, ro, ev_v, ("tokens", "accept_len", "num_tokens", "path_nodes", "flags"), reqs=[r])
    ev_f.check()
    ev_v.check()
