"""GPU parity of the per-request parameter entry points (uno_*_params) and of
the joint filter order against the oracle's per-request calls.

Each request draws its own temperature (greedy included), top_k and top_p;
both filter orders run; top_k bounds at or below 64 take the pipelined row
kernel, larger ones the general row kernel.  Out-of-range entries flag their
request's rows and leave the other requests unchanged."""
import numpy as np
import pytest
import torch

import oracle
from _parity import Events, compare_filter, compare_requests, np_of, to_device
from speculative_decoding_verification_filter_b200 import (FLAG_BAD_PARAMS, LAYOUT_GENERIC, LAYOUT_TWO_PASS,
                                                          uno_filter_softmax, uno_linear_cycle, uno_linear_verify,
                                                          uno_tree_topk_expand, uno_tree_verify)
from speculative_decoding_verification_filter_b200.inputs import (Workload, linear_draft, linear_target,
                                                                 tree_draft, tree_target)

pytestmark = pytest.mark.gpu

ORDERS = ("topk_first", "joint")


def _params(R, seed, k_hi):
    """Mixed per-request parameters: greedy, cool, neutral and hot
    temperatures; top_k from 1 to k_hi; top_p from 0.5 to 1."""
    g = np.random.default_rng(seed)
    T = g.choice(np.array([0.0, 0.6, 1.0, 1.4], dtype=np.float32), R)
    k = g.integers(1, k_hi + 1, R).astype(np.int32)
    k[g.random(R) < 0.3] = k_hi
    p = g.choice(np.array([0.5, 0.8, 0.95, 1.0], dtype=np.float32), R)
    return T, k, p


LINEAR = [
    (Workload("params bf16 8/1/8 full vocab", "linear", R=12, B=8, vocab=151936, dtype="bf16", sigma=1.0, noise=0.7,
              peak=8.0, seed=21), 50),
    (Workload("params f32 ragged", "linear", R=20, B=4, vocab=3001, dtype="f32", sigma=1.5, noise=1.0, seed=22), 64),
    (Workload("params bf16 top_k above 64", "linear", R=10, B=3, vocab=20000, dtype="bf16", sigma=1.0, noise=0.7,
              peak=5.0, seed=23), 120),
    (Workload("params f32 flat rows", "linear", R=9, B=5, vocab=4096, dtype="f32", sigma=0.3, noise=0.2, seed=24),
     40),
]


@pytest.mark.parametrize("order", ORDERS)
@pytest.mark.parametrize("w,k_hi", LINEAR, ids=lambda x: getattr(x, "name", str(x)))
def test_filter_and_linear_verify_per_request(w, k_hi, order):
    T, k, p = _params(w.R, w.seed, k_hi)
    q_np, p_np = linear_draft(w), linear_target(w)
    rng = (w.seed, 2, 5)
    dev_T, dev_k, dev_p = (torch.from_numpy(a).cuda() for a in (T, k, p))
    gq = uno_filter_softmax(to_device(q_np, w.dtype), temperature=dev_T, top_k=dev_k, top_p=dev_p,
                            rows_per_request=w.B, rng=rng, order=order, top_k_max=k_hi)
    rq = oracle.filter_softmax(q_np, w.dtype, T, k, p, rows_per_request=w.B, cap=min(k_hi, w.vocab), rng=rng,
                               order=order)
    ev = Events(f"{w.name} {order}: filter rows")
    compare_filter(gq, rq, ev, sample=True)
    ev.check()
    g = uno_linear_verify(to_device(p_np, w.dtype), gq["sample"].reshape(w.R, w.B), gq["ids"], gq["probs"],
                          gq["count"], R=w.R, B=w.B, temperature=dev_T, top_k=dev_k, top_p=dev_p, rng=rng,
                          order=order, top_k_max=k_hi)
    r = oracle.linear_verify(p_np, w.dtype, w.R, w.B, T, k, p, rq["sample"].reshape(w.R, w.B), rq["ids"],
                             rq["probs"], rq["count"], rng=rng, order=order)
    ev = Events(f"{w.name} {order}: uno_linear_verify_params requests")
    compare_requests(g, r, ev, ("tokens", "accept_len", "num_tokens", "flags"))
    ev.check()


@pytest.mark.parametrize("order", ORDERS)
@pytest.mark.parametrize("layout", [LAYOUT_GENERIC, LAYOUT_TWO_PASS])
def test_linear_cycle_per_request(layout, order):
    w = Workload("params cycle", "linear", R=16, B=6, vocab=151936, dtype="bf16", sigma=1.0, noise=0.7, peak=8.0,
                 seed=31)
    T, k, p = _params(w.R, 31 + layout, 50)
    q_np = linear_draft(w)
    p_full = linear_target(w)
    p_np = p_full if layout == LAYOUT_GENERIC else \
        np.ascontiguousarray(p_full.reshape(w.R, w.B + 1, -1)[:, :w.B]).reshape(w.R * w.B, -1)
    rng = (w.seed, 4, 0)
    g = uno_linear_cycle(to_device(q_np, w.dtype), to_device(p_np, w.dtype), R=w.R, B=w.B,
                         temperature=torch.from_numpy(T).cuda(), top_k=torch.from_numpy(k).cuda(),
                         top_p=torch.from_numpy(p).cuda(), rng=rng, layout=layout, order=order, top_k_max=50)
    ev = Events(f"params cycle layout {layout} {order}")
    if layout == LAYOUT_TWO_PASS:
        r = oracle.linear_cycle(q_np, p_np, w.dtype, w.R, w.B, T, k, p, rng, order=order)
        ref = dict(tokens=r["tokens"], num_accepted=r["num_correct_drafts"], num_tokens=r["accept_len"],
                   flags=r["flags"], margin=r["margin"])
        compare_requests(g, ref, ev, ("tokens", "num_accepted", "num_tokens", "flags"))
    else:
        rq = oracle.filter_softmax(q_np, w.dtype, T, k, p, rows_per_request=w.B, cap=50, rng=rng, order=order)
        r = oracle.linear_verify(p_np, w.dtype, w.R, w.B, T, k, p, rq["sample"].reshape(w.R, w.B), rq["ids"],
                                 rq["probs"], rq["count"], rng=rng, order=order)
        ref = dict(drafts=rq["sample"].reshape(w.R, w.B), tokens=r["tokens"], num_accepted=r["accept_len"],
                   num_tokens=r["num_tokens"],
                   flags=r["flags"] | np.bitwise_or.reduce(rq["flags"].reshape(w.R, w.B), axis=1),
                   margin=np.minimum(r["margin"], rq["margin"].reshape(w.R, w.B).min(axis=1)))
        compare_requests(g, ref, ev, ("drafts", "tokens", "num_accepted", "num_tokens", "flags"))
    ev.check()


@pytest.mark.parametrize("order", ORDERS)
def test_tree_verify_per_request(order):
    w = Workload("params tree", "tree", R=6, B=5, K=4, V=10, vocab=30011, dtype="bf16", sigma=1.0, noise=0.7,
                 peak=6.0, second_peak=4.0, seed=41)
    T, k, p = _params(w.R, 41, 50)
    q_np = tree_draft(w)
    rq = oracle.filter_softmax(q_np, w.dtype, w.temperature, w.top_k, w.top_p, rows_per_request=w.B)
    rt = oracle.tree_topk_expand(rq["ids"], rq["probs"], rq["count"], w.R, w.B, w.K, w.V)
    p_np = tree_target(w, rt["node_depth"], rt["num_nodes"])
    rng = (w.seed, 1, 0)
    nt, npa, nn = (torch.from_numpy(rt[key]).cuda() for key in ("node_token", "node_parent", "num_nodes"))
    g = uno_tree_verify(to_device(p_np, w.dtype), nt, npa, nn, R=w.R, B=w.B, V=w.V,
                        temperature=torch.from_numpy(T).cuda(), top_k=torch.from_numpy(k).cuda(),
                        top_p=torch.from_numpy(p).cuda(), rng=rng, order=order, top_k_max=50)
    r = oracle.tree_verify(p_np, w.dtype, w.R, w.B, w.V, T, k, p, rt["node_token"], rt["node_parent"],
                           rt["num_nodes"], rng=rng, order=order)
    ev = Events(f"params tree {order}")
    compare_requests(g, r, ev, ("tokens", "accept_len", "num_tokens", "path_nodes", "flags"))
    ev.check()


def test_scalar_arrays_equal_the_scalar_entry_points():
    """Arrays that repeat one value in the top-k-first order give exactly the
    results of the scalar entry points."""
    w = Workload("params scalar", "linear", R=8, B=4, vocab=70000, dtype="bf16", sigma=1.0, noise=0.7, peak=6.0,
                 seed=51)
    q, p = to_device(linear_draft(w), w.dtype), to_device(linear_target(w), w.dtype)
    rng = (w.seed, 0, 0)
    a = uno_linear_cycle(q, p, R=w.R, B=w.B, temperature=0.8, top_k=30, top_p=0.9, rng=rng)
    T = torch.full((w.R,), 0.8, device="cuda")
    k = torch.full((w.R,), 30, dtype=torch.int32, device="cuda")
    pp = torch.full((w.R,), 0.9, device="cuda")
    b = uno_linear_cycle(q, p, R=w.R, B=w.B, temperature=T, top_k=k, top_p=pp, rng=rng, top_k_max=30)
    for key in a:
        assert torch.equal(a[key], b[key]), key


def test_out_of_range_entries_flag_their_request_only():
    w = Workload("params bad", "linear", R=6, B=3, vocab=5000, dtype="f32", sigma=1.0, noise=0.5, seed=61)
    q_np = linear_draft(w)
    T = np.full(w.R, 1.0, np.float32)
    k = np.full(w.R, 20, np.int32)
    p = np.full(w.R, 0.9, np.float32)
    T[1] = -1.0        # negative temperature
    p[2] = 0.0         # top_p outside (0, 1]
    k[3] = 40          # above the call's bound of 20
    T[4] = np.nan
    rng = (w.seed, 0, 0)
    g = uno_filter_softmax(to_device(q_np, w.dtype), temperature=torch.from_numpy(T).cuda(),
                           top_k=torch.from_numpy(k).cuda(), top_p=torch.from_numpy(p).cuda(), rows_per_request=w.B,
                           rng=rng, top_k_max=20)
    flags, count = np_of(g["flags"]).reshape(w.R, w.B), np_of(g["count"]).reshape(w.R, w.B)
    for r in (1, 2, 3, 4):
        assert np.all(flags[r] & FLAG_BAD_PARAMS) and np.all(count[r] == 0), r
        assert np.all(np_of(g["sample"]).reshape(w.R, w.B)[r] == -1)
    good = [0, 5]
    rq = oracle.filter_softmax(q_np, w.dtype, 1.0, 20, 0.9, rows_per_request=w.B, rng=rng)
    ev = Events()
    rows = [r * w.B + i for r in good for i in range(w.B)]
    sub = {key: val[rows] for key, val in rq.items()}
    compare_filter(g, sub, ev, rows=rows, sample=True)
    ev.check()
