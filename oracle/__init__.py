"""The oracle: a plain CPU restatement of UNO's per-cycle sampling and
verification step, in double precision (``uno_ref.c``), with a numpy wrapper.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  It shares no code with the CUDA library and the library never calls
it.

What pins each function (the tests under ``tests/test_oracle_*.py``):

* ``philox`` / ``uniform``: the published Philox4x32-10 known-answer vectors
  (``tests/golden/philox4x32_10_kat.txt``) and the counter layout checked on a
  known-answer counter.
* ``filter_softmax``: reduces to ``numpy.argmax`` for T = 0 or top_k = 1, to
  ``scipy.special.softmax`` for top_p = 1 with top_k >= vocab, to a softmax
  over a ``numpy.lexsort`` top-k for top_p = 1; the top-p cut is checked
  against its defining property (the shortest prefix whose mass reaches
  top_p); the draw is checked by a chi-square test against the filtered
  probabilities.
* ``linear_verify``: the emitted sequence is distributed exactly as the
  target-only autoregressive process (chi-square on a tiny vocabulary with a
  prefix-dependent target table); the mean accept length equals its closed
  form; the invariants named by the method (counts in [0, B], equal p and q
  accept all, disjoint one-hot p and q reject at the first position, top_k 1
  is greedy speculative decoding).
* ``tree_topk_expand``: brute-force enumeration of every path of the depth-B
  trie, ranked by score; K = 1, V = B + 1 gives the argmax chain.
* ``tree_verify``: emitted sequence distributed as the target-only process
  (chi-square), mean accept length equals the sum over tree nodes of the
  target path probability, one-hot targets equal greedy decoding.
* the joint filter order (``order="joint"``, top-p read from the softmax of
  the whole row): a worked example derived by hand (weights 4 : 2 : 1 : 1),
  the closed form of a geometric row, its definition written with
  ``scipy.special.softmax`` over the whole row, the nesting of its support
  over the top-k-first one, reduction to the top-k-first order when
  top_p = 1 or top_k >= vocab, and linear verification under it distributed
  as the joint-filtered target process (chi-square).
* per-request sampling parameters (arrays of temperature, top_k, top_p):
  every call equals the same requests run one at a time.
* ``linear_cycle`` (the two-pass layout: base-weights first token, B - 1
  proposals, B + 1 output slots): it emits exactly what ``linear_verify``
  emits when the first draft row is also the first target row; its counters
  satisfy num_correct_drafts = accept_len - 2 and sum to the generated-token
  count; its output is distributed as the target-only process (chi-square).
* ``suffix_attention`` (a module of its own, numpy float64): the LSE merge of
  the prefix state with the tree-suffix attention equals attention over the
  union of the key sets (``scipy.special.softmax``); a chain tree equals
  causal attention (torch ``scaled_dot_product_attention``); grouped
  key/value heads equal repeated heads.

Parity unpinned: the boundary-event margin below which a GPU/oracle decision
difference is excused (``BOUNDARY_EPS``) is a stated tolerance, not a value the
pages fix.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "uno_ref.c"
_LIB_PATH = _HERE / "_build" / "libuno_ref.so"

F32, BF16 = 0, 1
DRAW_PROPOSAL, DRAW_ACCEPT, DRAW_RESIDUAL, DRAW_TARGET = 0, 1, 2, 3
FLAG_NONFINITE_ROW, FLAG_DRAFT_NOT_IN_SUPPORT, FLAG_RESIDUAL_EMPTY = 1, 2, 4

# A decision whose distance from its flip point is below this is a boundary
# event: the GPU may take the other branch there, and such cases are counted.
BOUNDARY_EPS = 1e-6

_lib = None


def build(force: bool = False) -> Path:
    """Compile ``uno_ref.c`` into ``oracle/_build/libuno_ref.so`` with gcc."""
    _LIB_PATH.parent.mkdir(parents=True, exist_ok=True)
    if force or not _LIB_PATH.exists() or _LIB_PATH.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB_PATH.with_suffix(".so.tmp%d" % os.getpid())
        cmd = ["gcc", "-std=c11", "-O2", "-Wall", "-Wextra", "-fPIC", "-shared",
               "-o", str(tmp), str(_SRC), "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(lib):
    P = ctypes.c_void_p
    i32, i64, u32, u64, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_float
    lib.uno_ref_philox4x32_10.argtypes = [P, P, P]
    lib.uno_ref_philox4x32_10.restype = None
    lib.uno_ref_uniform.argtypes = [u64, u32, u32, u32, u32]
    lib.uno_ref_uniform.restype = ctypes.c_double
    lib.uno_ref_set_uniforms.argtypes = [P, i64, i32]
    lib.uno_ref_set_uniforms.restype = None
    lib.uno_ref_filter_softmax.argtypes = [P, ctypes.c_int, i64, i64, i64, i32, f32, i32, f32, i32,
                                           P, P, P, P, ctypes.c_int, u64, u32, u32, P, P, P]
    lib.uno_ref_filter_softmax.restype = ctypes.c_int
    lib.uno_ref_linear_verify.argtypes = [P, ctypes.c_int, i32, i32, i64, f32, i32, f32, P, P, P, P, i32,
                                          u64, u32, u32, P, P, P, P, P]
    lib.uno_ref_linear_verify.restype = ctypes.c_int
    lib.uno_ref_tree_topk_expand.argtypes = [P, P, P, i32, i32, i32, i32, i32, P, P, P, P, P]
    lib.uno_ref_tree_topk_expand.restype = ctypes.c_int
    lib.uno_ref_tree_verify.argtypes = [P, ctypes.c_int, i32, i32, i32, i64, f32, i32, f32, P, P, P,
                                        u64, u32, u32, P, P, P, P, P, P]
    lib.uno_ref_tree_verify.restype = ctypes.c_int
    lib.uno_ref_filter_softmax_params.argtypes = [P, ctypes.c_int, i64, i64, i64, i32, P, P, P, ctypes.c_int,
                                                  i32, P, P, P, P, ctypes.c_int, u64, u32, u32, P, P, P]
    lib.uno_ref_filter_softmax_params.restype = ctypes.c_int
    lib.uno_ref_linear_verify_params.argtypes = [P, ctypes.c_int, i32, i32, i64, P, P, P, ctypes.c_int, P, P, P,
                                                 P, i32, u64, u32, u32, P, P, P, P, P]
    lib.uno_ref_linear_verify_params.restype = ctypes.c_int
    lib.uno_ref_tree_verify_params.argtypes = [P, ctypes.c_int, i32, i32, i32, i64, P, P, P, ctypes.c_int, P, P,
                                               P, u64, u32, u32, P, P, P, P, P, P]
    lib.uno_ref_tree_verify_params.restype = ctypes.c_int
    lib.uno_ref_linear_cycle.argtypes = [P, P, ctypes.c_int, i32, i32, i64, P, P, P, ctypes.c_int, u64, u32, u32,
                                         P, P, P, P, P]
    lib.uno_ref_linear_cycle.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(str(build())))
    return _lib


class use_library:
    """Context manager: route the functions of this module to another build of
    the oracle source (the tests use it to check that planted mistakes fail
    the pins)."""

    def __init__(self, so_path):
        self._new = _bind(ctypes.CDLL(str(so_path)))

    def __enter__(self):
        global _lib
        self._old = _load()
        _lib = self._new
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self._old
        return False


def _ptr(a):
    return None if a is None else a.ctypes.data


def _rng(rng):
    """rng = (seed, cycle) or (seed, cycle, first_request) -> three ints."""
    if rng is None:
        return 0, 0, 0
    return int(rng[0]), int(rng[1]), int(rng[2]) if len(rng) > 2 else 0


def _logits(arr, dtype):
    """Return (contiguous array, dtype code).  bf16 rows travel as uint16 bits."""
    if dtype == "bf16":
        a = np.ascontiguousarray(arr, dtype=np.uint16)
        return a, BF16
    if dtype == "f32":
        a = np.ascontiguousarray(arr, dtype=np.float32)
        return a, F32
    raise ValueError("dtype must be 'f32' or 'bf16'")


class OracleError(RuntimeError):
    pass


# Filter orders: "topk_first" renormalises the top-k set before the top-p
# cut; "joint" takes the top-p cut on the full-vocabulary softmax.
ORDERS = {"topk_first": 0, "joint": 1}


def _order_code(order):
    if order not in ORDERS:
        raise ValueError("order must be one of %s" % sorted(ORDERS))
    return ORDERS[order]


def _param_arrays(temperature, top_k, top_p, nreq):
    """One temperature, top_k and top_p per request (scalars broadcast)."""
    T = np.ascontiguousarray(np.broadcast_to(np.asarray(temperature, dtype=np.float32), (nreq,)))
    K = np.ascontiguousarray(np.broadcast_to(np.asarray(top_k, dtype=np.int32), (nreq,)))
    P = np.ascontiguousarray(np.broadcast_to(np.asarray(top_p, dtype=np.float32), (nreq,)))
    return T, K, P


def _per_request(temperature, top_k, top_p, order, nreq):
    """None when the call is the scalar top-k-first form; otherwise the
    three per-request arrays and the order code."""
    code = _order_code(order)
    if order == "topk_first" and all(np.ndim(v) == 0 for v in (temperature, top_k, top_p)):
        return None
    return _param_arrays(temperature, top_k, top_p, nreq) + (code,)


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what}: oracle status {rc}")


def philox(ctr, key):
    """Philox4x32-10 of a 4-word counter under a 2-word key."""
    lib = _load()
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, dtype=np.uint32)
    lib.uno_ref_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def uniform(seed, request, position, draw, cycle=0):
    return _load().uno_ref_uniform(int(seed), int(request), int(position), int(draw), int(cycle))


class injected_uniforms:
    """Context manager: while active, the oracle's decisions take their
    uniforms from ``table[request, position, draw]`` (shape [nreq, npos, 4],
    float64 in [0, 1)) instead of Philox; requests or positions outside the
    table still draw from Philox.  Used by the exact-enumeration pins, which
    run the oracle's own decision code at chosen uniforms."""

    def __init__(self, table):
        self.table = np.ascontiguousarray(table, dtype=np.float64)
        assert self.table.ndim == 3 and self.table.shape[2] == 4

    def __enter__(self):
        _load().uno_ref_set_uniforms(_ptr(self.table), self.table.shape[0], self.table.shape[1])
        return self

    def __exit__(self, *exc):
        _load().uno_ref_set_uniforms(None, 0, 0)
        return False


def filter_softmax(logits, dtype, temperature, top_k, top_p, *, rows_per_request=1, cap=None,
                   rng=None, dense=False, order="topk_first"):
    """Filter each row of ``logits`` ([rows, vocab]); returns a dict with
    ids [rows, cap], probs [rows, cap], count, flags, margin, and, on request,
    sample (rng = (seed, cycle)) and dense [rows, vocab].  temperature, top_k
    and top_p are scalars or one value per request."""
    a, code = _logits(logits, dtype)
    rows, vocab = a.shape
    nreq = -(-rows // rows_per_request)
    per = _per_request(temperature, top_k, top_p, order, nreq)
    if cap is None:
        cap = max(1, min(int(np.max(top_k)), vocab))
    ids = np.empty((rows, cap), dtype=np.int32)
    probs = np.empty((rows, cap), dtype=np.float32)
    count = np.empty(rows, dtype=np.int32)
    flags = np.empty(rows, dtype=np.uint32)
    margin = np.empty(rows, dtype=np.float64)
    dn = np.empty((rows, vocab), dtype=np.float32) if dense else None
    sample = np.empty(rows, dtype=np.int32) if rng is not None else None
    seed, cycle, first = _rng(rng)
    tail = (cap, _ptr(ids), _ptr(probs), _ptr(count), _ptr(dn), 1 if rng is not None else 0, seed, cycle,
            first, _ptr(sample), _ptr(flags), _ptr(margin))
    if per is None:
        rc = _load().uno_ref_filter_softmax(_ptr(a), code, rows, vocab, vocab, rows_per_request,
                                            float(temperature), int(top_k), float(top_p), *tail)
    else:
        T, K, P, oc = per
        rc = _load().uno_ref_filter_softmax_params(_ptr(a), code, rows, vocab, vocab, rows_per_request,
                                                   _ptr(T), _ptr(K), _ptr(P), oc, *tail)
    _check(rc, "filter_softmax")
    out = dict(ids=ids, probs=probs, count=count, flags=flags, margin=margin)
    if dense:
        out["dense"] = dn
    if rng is not None:
        out["sample"] = sample
    return out


def linear_verify(target_logits, dtype, R, B, temperature, top_k, top_p, draft_ids, q_ids, q_probs,
                  q_count, rng, order="topk_first"):
    """Linear rejection sampling; target_logits [R*(B+1), vocab]."""
    per = _per_request(temperature, top_k, top_p, order, R)
    a, code = _logits(target_logits, dtype)
    vocab = a.shape[-1]
    assert a.size == R * (B + 1) * vocab
    d = np.ascontiguousarray(draft_ids, dtype=np.int32).reshape(R, B)
    qi = np.ascontiguousarray(q_ids, dtype=np.int32)
    qp = np.ascontiguousarray(q_probs, dtype=np.float32)
    qc = np.ascontiguousarray(q_count, dtype=np.int32)
    q_cap = qi.shape[-1]
    toks = np.empty((R, B + 1), dtype=np.int32)
    acc = np.empty(R, dtype=np.int32)
    ntok = np.empty(R, dtype=np.int32)
    flags = np.empty(R, dtype=np.uint32)
    margin = np.empty(R, dtype=np.float64)
    seed, cycle, first = _rng(rng)
    tail = (_ptr(d), _ptr(qi), _ptr(qp), _ptr(qc), q_cap, seed, cycle, first, _ptr(toks), _ptr(acc),
            _ptr(ntok), _ptr(flags), _ptr(margin))
    if per is None:
        rc = _load().uno_ref_linear_verify(_ptr(a), code, R, B, vocab, float(temperature), int(top_k),
                                           float(top_p), *tail)
    else:
        T, K, P, oc = per
        rc = _load().uno_ref_linear_verify_params(_ptr(a), code, R, B, vocab, _ptr(T), _ptr(K), _ptr(P), oc,
                                                  *tail)
    _check(rc, "linear_verify")
    return dict(tokens=toks, accept_len=acc, num_tokens=ntok, flags=flags, margin=margin)


def tree_topk_expand(q_ids, q_probs, q_count, R, B, K, V):
    qi = np.ascontiguousarray(q_ids, dtype=np.int32)
    qp = np.ascontiguousarray(q_probs, dtype=np.float32)
    qc = np.ascontiguousarray(q_count, dtype=np.int32)
    q_cap = qi.shape[-1]
    tok = np.empty((R, V), dtype=np.int32)
    par = np.empty((R, V), dtype=np.int32)
    dep = np.empty((R, V), dtype=np.int32)
    sco = np.empty((R, V), dtype=np.float32)
    nn = np.empty(R, dtype=np.int32)
    rc = _load().uno_ref_tree_topk_expand(_ptr(qi), _ptr(qp), _ptr(qc), q_cap, R, B, K, V,
                                          _ptr(tok), _ptr(par), _ptr(dep), _ptr(sco), _ptr(nn))
    _check(rc, "tree_topk_expand")
    return dict(node_token=tok, node_parent=par, node_depth=dep, node_score=sco, num_nodes=nn)


def tree_verify(target_logits, dtype, R, B, V, temperature, top_k, top_p, node_token, node_parent,
                num_nodes, rng, order="topk_first"):
    """Target-only tree verification; target_logits [R*V, vocab]."""
    per = _per_request(temperature, top_k, top_p, order, R)
    a, code = _logits(target_logits, dtype)
    vocab = a.shape[-1]
    assert a.size == R * V * vocab
    tk = np.ascontiguousarray(node_token, dtype=np.int32)
    pa = np.ascontiguousarray(node_parent, dtype=np.int32)
    nn = np.ascontiguousarray(num_nodes, dtype=np.int32)
    toks = np.empty((R, B + 1), dtype=np.int32)
    path = np.empty((R, B + 1), dtype=np.int32)
    acc = np.empty(R, dtype=np.int32)
    ntok = np.empty(R, dtype=np.int32)
    flags = np.empty(R, dtype=np.uint32)
    margin = np.empty(R, dtype=np.float64)
    seed, cycle, first = _rng(rng)
    tail = (_ptr(tk), _ptr(pa), _ptr(nn), seed, cycle, first, _ptr(toks), _ptr(acc), _ptr(ntok), _ptr(path),
            _ptr(flags), _ptr(margin))
    if per is None:
        rc = _load().uno_ref_tree_verify(_ptr(a), code, R, B, V, vocab, float(temperature), int(top_k),
                                         float(top_p), *tail)
    else:
        T, K, P, oc = per
        rc = _load().uno_ref_tree_verify_params(_ptr(a), code, R, B, V, vocab, _ptr(T), _ptr(K), _ptr(P), oc,
                                                *tail)
    _check(rc, "tree_verify")
    return dict(tokens=toks, accept_len=acc, num_tokens=ntok, path_nodes=path, flags=flags,
                margin=margin)


def linear_cycle(draft_logits, target_logits, dtype, R, B, temperature, top_k, top_p, rng,
                 order="topk_first"):
    """One linear cycle in the two-pass layout: draft_logits and target_logits
    [R*B, vocab] each (draft row 0 of a request is the base-weights row);
    returns tokens [R, B+1], accept_len (tokens emitted), num_correct_drafts,
    flags and margin."""
    d, code = _logits(draft_logits, dtype)
    t, code_t = _logits(target_logits, dtype)
    vocab = d.shape[-1]
    assert code == code_t and d.size == R * B * vocab and t.size == R * B * vocab
    oc = _order_code(order)
    T, K, P = _param_arrays(temperature, top_k, top_p, R)
    toks = np.empty((R, B + 1), dtype=np.int32)
    acc = np.empty(R, dtype=np.int32)
    ncd = np.empty(R, dtype=np.int32)
    flags = np.empty(R, dtype=np.uint32)
    margin = np.empty(R, dtype=np.float64)
    seed, cycle, first = _rng(rng)
    rc = _load().uno_ref_linear_cycle(_ptr(d), _ptr(t), code, R, B, vocab, _ptr(T), _ptr(K), _ptr(P), oc,
                                      seed, cycle, first, _ptr(toks), _ptr(acc), _ptr(ncd), _ptr(flags),
                                      _ptr(margin))
    _check(rc, "linear_cycle")
    return dict(tokens=toks, accept_len=acc, num_correct_drafts=ncd, flags=flags, margin=margin)
