"""GPU parity of uno_filter_softmax against the oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle
from _parity import Events, compare_filter, np_of, to_device
from speculative_decoding_verification_filter_b200 import uno_filter_softmax
from speculative_decoding_verification_filter_b200.inputs import to_bf16_bits

pytestmark = pytest.mark.gpu


def _rows(rng, rows, vocab, scale=2.0, peak=0.0):
    x = (rng.standard_normal((rows, vocab)) * scale).astype(np.float32)
    if peak:
        x[np.arange(rows), rng.integers(0, vocab, rows)] += peak
    return x


def _encode(x, dtype):
    return to_bf16_bits(x) if dtype == "bf16" else x


def _run(x_enc, dtype, T, k, p, *, rpr=1, cap=None, rng=None, dense=False, dev=None):
    dev = to_device(x_enc, dtype) if dev is None else dev
    g = uno_filter_softmax(dev, temperature=T, top_k=k, top_p=p, rows_per_request=rpr, cap=cap, rng=rng,
                           dense=dense)
    r = oracle.filter_softmax(x_enc, dtype, T, k, p, rows_per_request=rpr, cap=cap, rng=rng, dense=dense)
    return g, r


CASES = [
    # (dtype, rows, vocab, T, k, p) -- rows spanning one CTA per row and split rows,
    # ragged vocabularies (not a multiple of the 16-byte vector), tiny ones
    ("f32", 37, 1003, 1.0, 50, 0.95),
    ("bf16", 37, 1003, 1.0, 50, 0.95),
    ("bf16", 700, 4099, 0.8, 50, 0.9),
    ("f32", 700, 4099, 1.3, 20, 0.99),
    ("bf16", 6, 151936, 1.0, 50, 0.95),
    ("f32", 5, 151936, 0.7, 50, 0.95),
    ("bf16", 3, 65537, 1.0, 300, 0.999),
    ("bf16", 2, 1000003, 1.0, 50, 0.95),  # long rows: about six pieces each, merged across CTAs
    ("f32", 64, 300, 1.0, 1024, 1.0),
    ("bf16", 9, 7, 1.0, 50, 0.95),
    ("f32", 9, 1, 1.0, 50, 0.95),
    # enough rows for run-time row hand-out, on rows of head and tail scalars
    # only (no whole 16-byte unit) and on barely longer ones
    ("bf16", 700, 7, 1.0, 50, 0.95),
    ("f32", 650, 3, 1.0, 50, 0.95),
    ("bf16", 640, 9, 0.8, 4, 0.9),
    ("f32", 33, 2000, 0.0, 50, 0.95),
    ("bf16", 33, 2000, 1.0, 1, 0.95),
    ("f32", 33, 2000, 1.0, 50, 1.0),
]


@pytest.mark.parametrize("dtype,rows,vocab,T,k,p", CASES)
def test_filter_and_sample_match_oracle(dtype, rows, vocab, T, k, p):
    rng = np.random.default_rng(rows * 7919 + vocab)
    x = _encode(_rows(rng, rows, vocab, peak=6.0 if vocab > 100 else 0.0), dtype)
    ev = Events()
    g, r = _run(x, dtype, T, k, p, rpr=4, rng=(1234, 7, 11))
    compare_filter(g, r, ev, sample=True)
    ev.check()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_unaligned_and_strided_rows(dtype):
    rng = np.random.default_rng(5)
    rows, vocab = 40, 5001
    full = _encode(_rows(rng, rows, vocab + 3, peak=5.0), dtype)
    ev = Events()
    for off in (1, 2, 3):
        x = np.ascontiguousarray(full[:, off:off + vocab])
        dev = to_device(full, dtype)[:, off:off + vocab]  # row stride vocab+3, base not 16-byte aligned
        assert dev.stride(0) == vocab + 3
        g, r = _run(x, dtype, 1.0, 50, 0.95, rng=(9, 0), dev=dev)
        compare_filter(g, r, ev, sample=True)
    ev.check()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ties_negative_zero_and_masks(dtype):
    rng = np.random.default_rng(6)
    rows, vocab = 64, 3000
    x = rng.integers(-4, 3, size=(rows, vocab)).astype(np.float32)  # heavy ties
    x[0, :] = 0.0
    x[0, ::2] = -0.0  # -0 and +0 tie; order by id
    x[1, :] = -np.inf
    x[1, 17] = 1.0
    x[2, :] = -np.inf
    x[2, [5, 2999, 1500]] = [2.0, 2.0, 1.0]
    x[3, 100:] = -np.inf
    ev = Events()
    for T, k, p in [(1.0, 50, 0.95), (1.0, 1000, 1.0), (0.5, 7, 0.5), (0.0, 50, 0.9)]:
        g, r = _run(_encode(x, dtype), dtype, T, k, p, rng=(3, 1), dense=True)
        compare_filter(g, r, ev, sample=True)
        assert np.max(np.abs(np_of(g["dense"]) - r["dense"])) <= 1e-6
    ev.check()


def test_non_finite_rows_are_flagged_not_trapped():
    rng = np.random.default_rng(7)
    x = _rows(rng, 12, 4000)
    x[0, 5] = np.nan
    x[1, 3999] = np.inf
    x[2, :] = -np.inf
    x[3, 0] = np.nan
    x[3, 1] = -np.inf
    for dtype in ("f32", "bf16"):
        g, r = _run(_encode(x, dtype), dtype, 1.0, 50, 0.95, rng=(1, 1))
        ev = Events()
        compare_filter(g, r, ev, sample=True)
        flags = np_of(g["flags"])
        assert list(flags[:4]) == [oracle.FLAG_NONFINITE_ROW] * 4
        assert list(np_of(g["count"])[:4]) == [0] * 4
        assert list(np_of(g["sample"])[:4]) == [-1] * 4
        assert np.all(flags[4:] == 0)


def test_split_rows_and_single_cta_rows_agree():
    """The same rows filtered alone (fp32 rows of 151,936 logits: each split
    across two CTAs) and in a large batch (one CTA per row, rows handed out
    at run time) give identical results."""
    rng = np.random.default_rng(8)
    x = _rows(rng, 4, 151936, scale=1.0, peak=8.0)
    few = uno_filter_softmax(to_device(x, "f32"), temperature=1.0, top_k=50, top_p=0.95, rng=(5, 0))
    many_x = np.concatenate([x] * 150)
    many = uno_filter_softmax(to_device(many_x, "f32"), temperature=1.0, top_k=50, top_p=0.95, rng=(5, 0))
    for key in ("ids", "probs", "count"):
        assert torch.equal(few[key], many[key][:4]), key
    assert torch.equal(few["sample"], many["sample"][:4])


def test_repeated_calls_reuse_the_workspace():
    rng = np.random.default_rng(9)
    x = to_device(to_bf16_bits(_rows(rng, 3, 151936, peak=8.0)), "bf16")
    outs = [uno_filter_softmax(x, temperature=1.0, top_k=50, top_p=0.95, rng=(5, c)) for c in range(4)]
    for o in outs[1:]:
        assert torch.equal(o["ids"], outs[0]["ids"]) and torch.equal(o["probs"], outs[0]["probs"])
    r = oracle.filter_softmax(np_of(x.view(torch.int16)).view(np.uint16), "bf16", 1.0, 50, 0.95, rng=(5, 3))
    assert np.array_equal(np_of(outs[3]["sample"]), r["sample"])


@pytest.mark.parametrize("dtype,rows,vocab,k,p,pattern", [
    ("bf16", 600, 20000, 8, 0.9, (1.0, 20.0)),
    ("f32", 600, 20000, 8, 0.9, (1.0, 1.0, 1.0, 20.0, 20.0, 20.0)),
    ("bf16", 400, 70001, 16, 0.95, (30.0, 1.0, 1.0)),
    ("f32", 450, 40000, 50, 0.95, (1.0, 25.0)),
])
def test_rows_of_changing_scale_match_oracle(dtype, rows, vocab, k, p, pattern):
    """Consecutive rows of very different scale: a threshold predicted from
    one row is far too high or far too low for the next, so rows are re-read
    in the redo pass or flood the candidate buffers.  Results must still
    equal the oracle's."""
    rng = np.random.default_rng(rows + vocab + k)
    scale = np.resize(np.asarray(pattern, dtype=np.float32), rows)[:, None]
    x = _encode(_rows(rng, rows, vocab, scale=1.0, peak=4.0) * scale, dtype)
    ev = Events()
    g, r = _run(x, dtype, 1.0, k, p, rpr=3, rng=(77, 2))
    compare_filter(g, r, ev, sample=True)
    ev.check()
