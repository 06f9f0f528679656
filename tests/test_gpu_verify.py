"""GPU parity of the linear and tree paths (filter -> verify, filter -> expand
-> verify) against the oracle, on seeded inputs of moderate size."""
import numpy as np
import pytest
import torch

import oracle
from _parity import Events, compare_filter, compare_requests, np_of, to_device
from speculative_decoding_verification_filter_b200 import (LAYOUT_TWO_PASS, uno_filter_softmax, uno_linear_cycle,
                                                          uno_linear_verify, uno_tree_topk_expand, uno_tree_verify)
from speculative_decoding_verification_filter_b200.inputs import (Workload, linear_draft, linear_target,
                                                                 tree_draft, tree_target)

pytestmark = pytest.mark.gpu

LINEAR_KEYS = ("tokens", "accept_len", "num_tokens", "flags")
TREE_KEYS = ("tokens", "accept_len", "num_tokens", "path_nodes", "flags")
TREE_NODE_KEYS = ("node_token", "node_parent", "node_depth", "node_score", "num_nodes")


def run_linear(w: Workload, q_np, p_np, rng, *, drafts_edit=None, ev=None):
    """Both sides from the same logits; each side uses its own filtered q."""
    ev = ev or Events()
    sp = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)
    gq = uno_filter_softmax(to_device(q_np, w.dtype), rows_per_request=w.B, rng=rng, **sp)
    rq = oracle.filter_softmax(q_np, w.dtype, w.temperature, w.top_k, w.top_p, rows_per_request=w.B, rng=rng)
    compare_filter(gq, rq, ev, sample=True)
    gd = gq["sample"].reshape(w.R, w.B).clone()
    rd = rq["sample"].reshape(w.R, w.B).copy()
    if drafts_edit is not None:
        drafts_edit(gd, rd)
    g = uno_linear_verify(to_device(p_np, w.dtype), gd, gq["ids"], gq["probs"], gq["count"], R=w.R, B=w.B,
                          rng=rng, **sp)
    r = oracle.linear_verify(p_np, w.dtype, w.R, w.B, w.temperature, w.top_k, w.top_p, rd, rq["ids"],
                             rq["probs"], rq["count"], rng=rng)
    compare_requests(g, r, ev, LINEAR_KEYS)
    ev.check()
    return g, r


def run_tree(w: Workload, rng, ev=None, target_edit=None):
    ev = ev or Events()
    sp = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)
    q_np = tree_draft(w)
    gq = uno_filter_softmax(to_device(q_np, w.dtype), rows_per_request=w.B, **sp)
    rq = oracle.filter_softmax(q_np, w.dtype, w.temperature, w.top_k, w.top_p, rows_per_request=w.B)
    compare_filter(gq, rq, ev)
    gt = uno_tree_topk_expand(gq["ids"], gq["probs"], gq["count"], R=w.R, B=w.B, K=w.K, V=w.V)
    rt = oracle.tree_topk_expand(rq["ids"], rq["probs"], rq["count"], w.R, w.B, w.K, w.V)
    for key in TREE_NODE_KEYS:
        assert np.array_equal(np_of(gt[key]), rt[key]), key
    p_np = tree_target(w, rt["node_depth"], rt["num_nodes"])
    if target_edit is not None:
        target_edit(p_np)
    g = uno_tree_verify(to_device(p_np, w.dtype), gt["node_token"], gt["node_parent"], gt["num_nodes"], R=w.R,
                        B=w.B, V=w.V, rng=rng, **sp)
    r = oracle.tree_verify(p_np, w.dtype, w.R, w.B, w.V, w.temperature, w.top_k, w.top_p, rt["node_token"],
                           rt["node_parent"], rt["num_nodes"], rng=rng)
    compare_requests(g, r, ev, TREE_KEYS)
    ev.check()
    return g, r, rt


LINEAR_CASES = [
    Workload("lin f32 small", "linear", R=4, B=4, vocab=1024, dtype="f32", sigma=2.0, noise=0.5, seed=42),
    Workload("lin bf16 ragged", "linear", R=24, B=5, vocab=3001, dtype="bf16", sigma=1.0, noise=0.7, peak=5.0,
             seed=3),
    Workload("lin bf16 many rows", "linear", R=130, B=8, vocab=2048, dtype="bf16", sigma=1.0, noise=0.7, peak=8.0,
             seed=4),
    Workload("lin f32 low acceptance", "linear", R=40, B=16, vocab=999, dtype="f32", sigma=1.5, noise=1.0,
             temperature=0.7, seed=5),
    Workload("lin f32 greedy", "linear", R=16, B=6, vocab=500, dtype="f32", sigma=1.0, noise=0.3, temperature=0.0,
             seed=6),
    Workload("lin bf16 top-k 1", "linear", R=16, B=6, vocab=500, dtype="bf16", sigma=1.0, noise=0.3, top_k=1,
             seed=7),
    Workload("lin f32 no top-p", "linear", R=16, B=3, vocab=700, dtype="f32", sigma=1.0, noise=0.5, top_p=1.0,
             seed=8),
    Workload("lin bf16 full vocab few requests", "linear", R=2, B=3, vocab=151936, dtype="bf16", sigma=1.0,
             noise=0.7, peak=8.0, seed=9),
    # more than 32 draft positions (token slots beyond one warp)
    Workload("lin f32 B=40", "linear", R=3, B=40, vocab=600, dtype="f32", sigma=1.0, noise=0.05, top_k=10, seed=10),
    Workload("lin bf16 B=40 top-k 50", "linear", R=3, B=40, vocab=600, dtype="bf16", sigma=1.0, noise=0.05, seed=13),
    # rows handed out at run time, each only head and tail scalars
    Workload("lin bf16 tiny vocab many rows", "linear", R=100, B=6, vocab=6, dtype="bf16", sigma=1.0, noise=0.5,
             seed=14),
]


@pytest.mark.parametrize("w", LINEAR_CASES, ids=lambda w: w.name)
def test_linear_path_matches_oracle(w):
    g, r = run_linear(w, linear_draft(w), linear_target(w), rng=(w.seed, 2))
    acc = np_of(g["accept_len"])
    assert np.all((acc >= 0) & (acc <= w.B))


def test_linear_draft_errors_and_nonfinite_targets():
    w = Workload("lin edge", "linear", R=8, B=4, vocab=600, dtype="f32", sigma=1.0, noise=0.2, top_k=5, seed=11)
    q_np, p_np = linear_draft(w), linear_target(w)
    p_np = p_np.copy()
    p_np[1 * (w.B + 1) + 2, 10] = np.nan      # request 1, target row 2
    p_np[2 * (w.B + 1) + 0, :] = -np.inf     # request 2, target row 0: no support
    p_np[3 * (w.B + 1) + w.B, 7] = np.inf    # request 3, bonus row

    def edit(gd, rd):
        for d in (gd, rd):
            d[4, 0] = -1         # below the vocabulary
            d[5, 1] = w.vocab    # above it
            d[6, 2] = 599        # in the vocabulary, almost surely outside supp q (top_k 5)
    g, r = run_linear(w, q_np, p_np, rng=(77, 0), drafts_edit=edit)
    flags = np_of(g["flags"])
    assert flags[2] & oracle.FLAG_NONFINITE_ROW and np_of(g["num_tokens"])[2] == 0
    assert flags[4] & oracle.FLAG_DRAFT_NOT_IN_SUPPORT and np_of(g["accept_len"])[4] == 0


def test_linear_cycles_and_first_request_offset():
    w = Workload("lin offset", "linear", R=12, B=3, vocab=1500, dtype="bf16", sigma=1.0, noise=0.7, peak=4.0, seed=12)
    q_np, p_np = linear_draft(w), linear_target(w)
    for cycle in (0, 1, 99):
        run_linear(w, q_np, p_np, rng=(w.seed, cycle, 1000))
    # the second half of the batch alone, with first_request = 6, equals the
    # second half of the whole batch
    whole, _ = run_linear(w, q_np, p_np, rng=(w.seed, 5, 0))
    half = Workload("half", "linear", R=6, B=3, vocab=1500, dtype="bf16", sigma=1.0, noise=0.7, peak=4.0, seed=12)
    gh, _ = run_linear(half, q_np[6 * 3:], p_np[6 * 4:], rng=(w.seed, 5, 6))
    for key in LINEAR_KEYS:
        assert torch.equal(gh[key], whole[key][6:]), key


TREE_CASES = [
    Workload("tree f32 small", "tree", R=3, B=4, K=3, V=10, vocab=1000, dtype="f32", sigma=2.0, noise=0.5, seed=21),
    Workload("tree bf16 8/16/8 shape", "tree", R=20, B=8, K=16, V=8, vocab=3001, dtype="bf16", sigma=1.0, noise=0.7,
             peak=8.0, second_peak=6.0, seed=7),
    Workload("tree bf16 16/32/32 shape", "tree", R=2, B=16, K=32, V=32, vocab=4099, dtype="bf16", sigma=1.0,
             noise=0.7, peak=8.0, seed=42),
    Workload("tree f32 wide", "tree", R=5, B=3, K=20, V=100, vocab=800, dtype="f32", sigma=1.0, noise=0.5, seed=22),
    Workload("tree small tree (K=1)", "tree", R=6, B=3, K=1, V=8, vocab=500, dtype="f32", sigma=1.0, noise=0.5,
             seed=23),
    Workload("tree greedy", "tree", R=6, B=5, K=4, V=12, vocab=500, dtype="bf16", sigma=1.0, noise=0.3,
             temperature=0.0, seed=24),
    Workload("tree max shape", "tree", R=2, B=16, K=16, V=128, vocab=2000, dtype="bf16", sigma=1.0, noise=0.7,
             peak=3.0, seed=25),
    # a chain longer than 32 nodes (token slots beyond one warp)
    Workload("tree deep chain", "tree", R=2, B=40, K=1, V=48, vocab=600, dtype="f32", sigma=1.0, noise=0.02,
             top_k=10, seed=26),
]


@pytest.mark.parametrize("w", TREE_CASES, ids=lambda w: w.name)
def test_tree_path_matches_oracle(w):
    g, r, rt = run_tree(w, rng=(w.seed, 1))
    acc = np_of(g["accept_len"])
    assert np.all((acc >= 0) & (acc <= w.B))


def test_tree_nonfinite_node_rows():
    w = Workload("tree edge", "tree", R=4, B=3, K=2, V=6, vocab=400, dtype="f32", sigma=1.0, noise=0.2, seed=31)

    def edit(p):
        p[0 * w.V + 0, 3] = np.nan   # request 0: root row
        p[1 * w.V + 1, :] = -np.inf  # request 1: node 1
    g, r, rt = run_tree(w, rng=(5, 0), target_edit=edit)
    assert np_of(g["flags"])[0] & oracle.FLAG_NONFINITE_ROW
    assert np_of(g["num_tokens"])[0] == 0


@pytest.mark.parametrize("layout", ["wide rows", "offset start"])
def test_linear_draft_row_layouts(layout):
    """The draft rows as the verifier receives them: a row stride above 64 entries
    (cap 100 for top-k 50), or arrays that start 4 bytes past a 16-byte boundary.
    Both must give the same verification as the oracle."""
    w = Workload("lin bf16 layouts", "linear", R=12, B=6, vocab=4099, dtype="bf16", sigma=1.0, noise=0.7, peak=6.0,
                 seed=21)
    rng = (77, 2)
    sp = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)
    q_np, p_np = linear_draft(w), linear_target(w)
    ev = Events()
    cap = 100 if layout == "wide rows" else w.top_k
    gq = uno_filter_softmax(to_device(q_np, w.dtype), rows_per_request=w.B, rng=rng, cap=cap, **sp)
    rq = oracle.filter_softmax(q_np, w.dtype, w.temperature, w.top_k, w.top_p, rows_per_request=w.B, rng=rng)
    compare_filter(gq, rq, ev, sample=True)
    q_ids, q_probs = gq["ids"], gq["probs"]
    if layout == "offset start":
        n = q_ids.numel()
        flat_i = torch.empty(n + 1, dtype=q_ids.dtype, device=q_ids.device)
        flat_p = torch.empty(n + 1, dtype=q_probs.dtype, device=q_probs.device)
        flat_i[1:].copy_(q_ids.reshape(-1))
        flat_p[1:].copy_(q_probs.reshape(-1))
        q_ids, q_probs = flat_i[1:].view(q_ids.shape), flat_p[1:].view(q_probs.shape)
        assert q_ids.data_ptr() % 16 == 4
    g = uno_linear_verify(to_device(p_np, w.dtype), gq["sample"].reshape(w.R, w.B), q_ids, q_probs, gq["count"],
                          R=w.R, B=w.B, rng=rng, **sp)
    r = oracle.linear_verify(p_np, w.dtype, w.R, w.B, w.temperature, w.top_k, w.top_p,
                             rq["sample"].reshape(w.R, w.B), rq["ids"], rq["probs"], rq["count"], rng=rng)
    compare_requests(g, r, ev, LINEAR_KEYS)
    ev.check()


def test_cycle_with_tiny_vocabulary_and_many_rows():
    """uno_linear_cycle in the two-pass layout over 1,200 rows of 6 logits:
    rows handed out at run time, none holding a whole 16-byte unit."""
    w = Workload("cycle tiny vocab", "linear", R=100, B=6, vocab=6, dtype="bf16", sigma=1.0, noise=0.5, seed=15)
    q_np = linear_draft(w)
    p_np = np.ascontiguousarray(linear_target(w).reshape(w.R, w.B + 1, -1)[:, :w.B]).reshape(w.R * w.B, -1)
    rng = (w.seed, 3, 1)
    sp = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)
    g = uno_linear_cycle(to_device(q_np, w.dtype), to_device(p_np, w.dtype), R=w.R, B=w.B, rng=rng,
                         layout=LAYOUT_TWO_PASS, **sp)
    r = oracle.linear_cycle(q_np, p_np, w.dtype, w.R, w.B, w.temperature, w.top_k, w.top_p, rng)
    ref = dict(tokens=r["tokens"], num_accepted=r["num_correct_drafts"], num_tokens=r["accept_len"],
               flags=r["flags"], margin=r["margin"])
    ev = Events("tiny vocabulary cycle, two-pass layout")
    compare_requests(g, ref, ev, ("tokens", "num_accepted", "num_tokens", "flags"))
    ev.check()
