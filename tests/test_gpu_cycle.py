"""GPU parity of uno_linear_cycle (one launch over a cycle's draft and target
rows) against the oracle, in both layouts: the generic one (every proposal
tested, B + 1 target rows; the oracle's filter_softmax then linear_verify) and
the pages' two-pass layout (x_0 untested, target row i - 1 tests x_i; the
oracle's linear_cycle)."""
import numpy as np
import pytest

import oracle
from _parity import Events, compare_requests, np_of, to_device
from speculative_decoding_verification_filter_b200 import LAYOUT_GENERIC, LAYOUT_TWO_PASS, uno_linear_cycle
from speculative_decoding_verification_filter_b200.inputs import Workload, linear_draft, linear_target

pytestmark = pytest.mark.gpu

CASES = [
    Workload("cyc f32 small", "linear", R=4, B=4, vocab=1024, dtype="f32", sigma=2.0, noise=0.5, seed=42),
    Workload("cyc bf16 ragged", "linear", R=24, B=5, vocab=3001, dtype="bf16", sigma=1.0, noise=0.7, peak=5.0,
             seed=3),
    Workload("cyc bf16 many rows", "linear", R=130, B=8, vocab=2048, dtype="bf16", sigma=1.0, noise=0.7, peak=8.0,
             seed=4),
    Workload("cyc f32 low acceptance", "linear", R=40, B=16, vocab=999, dtype="f32", sigma=1.5, noise=1.0,
             temperature=0.7, seed=5),
    Workload("cyc bf16 full vocab", "linear", R=6, B=8, vocab=151936, dtype="bf16", sigma=1.0, noise=0.7, peak=8.0,
             seed=9),
    Workload("cyc f32 top-k 100", "linear", R=8, B=4, vocab=2000, dtype="f32", sigma=1.0, noise=0.5, top_k=100,
             seed=12),
    Workload("cyc bf16 B=1", "linear", R=9, B=1, vocab=4000, dtype="bf16", sigma=1.0, noise=0.7, seed=14),
    Workload("cyc f32 greedy", "linear", R=16, B=6, vocab=500, dtype="f32", sigma=1.0, noise=0.3, temperature=0.0,
             seed=6),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_generic_cycle_matches_filter_then_verify(w):
    q_np, p_np = linear_draft(w), linear_target(w)
    rng = (w.seed, 5, 3)
    sp = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)
    g = uno_linear_cycle(to_device(q_np, w.dtype), to_device(p_np, w.dtype), R=w.R, B=w.B, rng=rng,
                         layout=LAYOUT_GENERIC, **sp)
    rq = oracle.filter_softmax(q_np, w.dtype, w.temperature, w.top_k, w.top_p, rows_per_request=w.B, rng=rng)
    r = oracle.linear_verify(p_np, w.dtype, w.R, w.B, w.temperature, w.top_k, w.top_p,
                             rq["sample"].reshape(w.R, w.B), rq["ids"], rq["probs"], rq["count"], rng=rng)
    ref = dict(tokens=r["tokens"], num_accepted=r["accept_len"], num_tokens=r["num_tokens"],
               flags=r["flags"] | np.bitwise_or.reduce(rq["flags"].reshape(w.R, w.B), axis=1),
               drafts=rq["sample"].reshape(w.R, w.B),
               margin=np.minimum(r["margin"], rq["margin"].reshape(w.R, w.B).min(axis=1)))
    ev = Events()
    compare_requests(g, ref, ev, ("drafts", "tokens", "num_accepted", "num_tokens", "flags"))
    ev.check()


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_two_pass_cycle_matches_oracle(w):
    q_np = linear_draft(w)
    # B target rows per request: the generator's first B target rows
    p_full = linear_target(w).reshape(w.R, w.B + 1, -1)
    p_np = np.ascontiguousarray(p_full[:, :w.B]).reshape(w.R * w.B, -1)
    rng = (w.seed, 6, 0)
    sp = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)
    g = uno_linear_cycle(to_device(q_np, w.dtype), to_device(p_np, w.dtype), R=w.R, B=w.B, rng=rng,
                         layout=LAYOUT_TWO_PASS, **sp)
    r = oracle.linear_cycle(q_np, p_np, w.dtype, w.R, w.B, w.temperature, w.top_k, w.top_p, rng)
    ref = dict(tokens=r["tokens"], num_accepted=r["num_correct_drafts"], num_tokens=r["accept_len"],
               flags=r["flags"], margin=r["margin"])
    ev = Events()
    compare_requests(g, ref, ev, ("tokens", "num_accepted", "num_tokens", "flags"))
    ev.check()
    # the pages' counters: num_correct_drafts = accept_len - 2 on finite rows
    nt, na = np_of(g["num_tokens"]), np_of(g["num_accepted"])
    fin = np_of(g["flags"]) == 0
    assert np.all(na[fin] == np.maximum(nt[fin] - 2, 0) + (nt[fin] < 2) * 0)


def test_cycle_repeated_calls_carry_predictions():
    """Back-to-back calls on the same workspace (the later ones start from the
    earlier ones' predictions) give the same results as the first."""
    w = Workload("cyc repeat", "linear", R=64, B=8, vocab=151936, dtype="bf16", sigma=1.0, noise=0.7, peak=8.0,
                 seed=42)
    q = to_device(linear_draft(w), w.dtype)
    p = to_device(linear_target(w), w.dtype)
    outs = [uno_linear_cycle(q, p, R=w.R, B=w.B, rng=(42, 0), temperature=1.0, top_k=50, top_p=0.95)
            for _ in range(3)]
    for o in outs[1:]:
        for key in ("tokens", "num_accepted", "num_tokens", "flags", "drafts"):
            assert np.array_equal(np_of(o[key]), np_of(outs[0][key])), key
