"""Thin Python binding of libuno_filter.so (include/uno_filter.h).

The functions carry the C entry points' names and only marshal arguments:
they check shapes, allocate output tensors and a zero-filled workspace with
PyTorch, pass raw device pointers and the current CUDA stream, and raise when
the library returns an error.  Every step of the computation runs in the
library's CUDA kernels.  Host (CPU) input tensors are copied to the current
CUDA device first and results are copied back, which is what the end-to-end
benchmark measures.
"""
from __future__ import annotations

import ctypes
import threading
from pathlib import Path

import numpy as np
import torch

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libuno_filter.so"

UNO_F32, UNO_BF16 = 0, 1
FLAG_NONFINITE_ROW, FLAG_DRAFT_NOT_IN_SUPPORT, FLAG_RESIDUAL_EMPTY = 1, 2, 4
FLAG_BAD_TREE = 16
FLAG_BAD_PARAMS = 32
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported argument", 3: "CUDA launch error",
          4: "workspace missing or too small"}

EXPORTED = (
    "uno_filter_softmax_workspace_bytes", "uno_filter_softmax",
    "uno_linear_verify_workspace_bytes", "uno_linear_verify",
    "uno_linear_cycle_workspace_bytes", "uno_linear_cycle",
    "uno_tree_topk_expand",
    "uno_tree_verify_workspace_bytes", "uno_tree_verify",
    "uno_filter_softmax_params", "uno_linear_verify_params", "uno_linear_cycle_params", "uno_tree_verify_params",
    "uno_linear_verify_noalloc",
    "uno_tree_suffix_attention_merge",
    "uno_status_string",
)


class UnoError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn}: {STATUS.get(status, 'status %d' % status)}")
        self.status = status


class _Params(ctypes.Structure):
    _fields_ = [("temperature", ctypes.c_float), ("top_k", ctypes.c_int32), ("top_p", ctypes.c_float)]


class _Rng(ctypes.Structure):
    _fields_ = [("seed", ctypes.c_uint64), ("cycle", ctypes.c_uint32), ("first_request", ctypes.c_uint32),
                ("cycle_word", ctypes.c_void_p)]


class _ReqParams(ctypes.Structure):
    _fields_ = [("temperature", ctypes.c_void_p), ("top_k", ctypes.c_void_p), ("top_p", ctypes.c_void_p),
                ("top_k_max", ctypes.c_int32), ("order", ctypes.c_int32)]


ORDERS = {"topk_first": 0, "joint": 1}


class _PerRequest:
    """Per-request parameter arrays on the device (kept alive for the call)
    and the struct that points at them."""

    def __init__(self, temperature, top_k, top_p, order, nreq, device, top_k_max):
        _need(order in ORDERS, f"order must be one of {sorted(ORDERS)}")

        def arr(x, dt):
            t = torch.as_tensor(x, dtype=dt)
            t = t.reshape(-1) if t.dim() else t.reshape(1).expand(nreq)
            _need(t.numel() == nreq, f"per-request parameters need {nreq} entries")
            return t.to(device, non_blocking=True).contiguous()

        self.T = arr(temperature, torch.float32)
        self.k = arr(top_k, torch.int32)
        self.p = arr(top_p, torch.float32)
        if top_k_max is None:
            # the bound from the values themselves (a device array is read back)
            top_k_max = int(torch.as_tensor(top_k).max().item())
        self.top_k_max = max(1, int(top_k_max))
        self.c = _ReqParams(ctypes.c_void_p(self.T.data_ptr()), ctypes.c_void_p(self.k.data_ptr()),
                            ctypes.c_void_p(self.p.data_ptr()), self.top_k_max, ORDERS[order])


def _per_request(temperature, top_k, top_p, order, nreq, device, top_k_max, force=False):
    """None for scalar parameters in the top-k-first order (the plain entry
    points) unless `force`, else a _PerRequest for the *_params entry points."""
    scalar = not force and all(isinstance(x, (int, float, np.generic)) or (isinstance(x, (torch.Tensor, np.ndarray)) and x.ndim == 0)
                 for x in (temperature, top_k, top_p))
    if scalar and order == "topk_first":
        return None
    return _PerRequest(temperature, top_k, top_p, order, nreq, device, top_k_max)


def _rng(rng):
    """(seed, cycle) or (seed, cycle, first_request) -> _Rng.  cycle is an
    int, or a one-element int32 CUDA tensor whose value the kernels read when
    they run (what a captured graph needs to draw a new cycle per replay)."""
    seed, cycle = int(rng[0]), rng[1]
    first = int(rng[2]) if len(rng) > 2 else 0
    if isinstance(cycle, torch.Tensor):
        _need(cycle.is_cuda and cycle.dtype == torch.int32 and cycle.numel() == 1,
              "a device cycle word must be a one-element int32 CUDA tensor")
        return _Rng(seed, 0, first, ctypes.c_void_p(cycle.data_ptr()))
    return _Rng(seed, int(cycle), first, None)


_lib = None
_lock = threading.Lock()


def load_library():
    """Load libuno_filter.so; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not LIB_PATH.exists():
            raise RuntimeError(f"{LIB_PATH.name} is not built: run `python -m "
                               "speculative_decoding_verification_filter_b200.build` (needs nvcc)")
        lib = ctypes.CDLL(str(LIB_PATH))
        P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        lib.uno_filter_softmax_workspace_bytes.argtypes = [i64, i64, i32]
        lib.uno_filter_softmax_workspace_bytes.restype = sz
        lib.uno_filter_softmax.argtypes = [P, ctypes.c_int, i64, i64, i64, i32, _Params, i32, P, P, P, P,
                                           ctypes.POINTER(_Rng), P, P, P, sz, P]
        lib.uno_filter_softmax.restype = ctypes.c_int
        lib.uno_linear_verify_workspace_bytes.argtypes = [i32, i32, i64, i32]
        lib.uno_linear_verify_workspace_bytes.restype = sz
        lib.uno_linear_verify.argtypes = [P, ctypes.c_int, i32, i32, i64, _Params, P, P, P, P, i32, _Rng,
                                          P, P, P, P, P, sz, P]
        lib.uno_linear_verify.restype = ctypes.c_int
        lib.uno_linear_cycle_workspace_bytes.argtypes = [i32, i32, i64, i32, i32]
        lib.uno_linear_cycle_workspace_bytes.restype = sz
        lib.uno_linear_cycle.argtypes = [P, P, ctypes.c_int, i32, i32, i64, i32, _Params, _Rng, P, P, P, P, P, P, sz,
                                         P]
        lib.uno_linear_cycle.restype = ctypes.c_int
        lib.uno_tree_topk_expand.argtypes = [P, P, P, i32, i32, i32, i32, i32, P, P, P, P, P, P]
        lib.uno_tree_topk_expand.restype = ctypes.c_int
        lib.uno_tree_verify_workspace_bytes.argtypes = [i32, i32, i64, i32]
        lib.uno_tree_verify_workspace_bytes.restype = sz
        lib.uno_tree_verify.argtypes = [P, ctypes.c_int, i32, i32, i32, i64, _Params, P, P, P, _Rng,
                                        P, P, P, P, P, P, sz, P]
        lib.uno_tree_verify.restype = ctypes.c_int
        RP = ctypes.POINTER(_ReqParams)
        lib.uno_filter_softmax_params.argtypes = [P, ctypes.c_int, i64, i64, i64, i32, RP, i32, P, P, P, P,
                                                  ctypes.POINTER(_Rng), P, P, P, sz, P]
        lib.uno_filter_softmax_params.restype = ctypes.c_int
        lib.uno_linear_verify_params.argtypes = [P, ctypes.c_int, i32, i32, i64, RP, P, P, P, P, i32, _Rng,
                                                 P, P, P, P, P, sz, P]
        lib.uno_linear_verify_params.restype = ctypes.c_int
        lib.uno_linear_cycle_params.argtypes = [P, P, ctypes.c_int, i32, i32, i64, i32, RP, _Rng, P, P, P, P, P, P,
                                                sz, P]
        lib.uno_linear_cycle_params.restype = ctypes.c_int
        lib.uno_tree_verify_params.argtypes = [P, ctypes.c_int, i32, i32, i32, i64, RP, P, P, P, _Rng,
                                               P, P, P, P, P, P, sz, P]
        lib.uno_tree_verify_params.restype = ctypes.c_int
        lib.uno_linear_verify_noalloc.argtypes = [P, ctypes.c_int, i32, i32, i64, _Params, P, P, P, P, i32, _Rng,
                                                  P, P, P, P, P]
        lib.uno_linear_verify_noalloc.restype = ctypes.c_int
        lib.uno_tree_suffix_attention_merge.argtypes = [P, P, P, ctypes.c_int, i32, i32, i32, i32, i32,
                                                         ctypes.c_float, P, P, P, P, P, P, P, P]
        lib.uno_tree_suffix_attention_merge.restype = ctypes.c_int
        lib.uno_status_string.argtypes = [ctypes.c_int]
        lib.uno_status_string.restype = ctypes.c_char_p
        _lib = lib
        return lib


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------
_ws_cache: dict = {}


def workspace(nbytes: int, device: torch.device, stream: torch.cuda.Stream) -> torch.Tensor:
    """A zero-filled workspace of at least nbytes for this device and stream.

    The library leaves its counters at zero after each call, so the buffer is
    zero-filled once, when it is created or grown."""
    key = (device.index, stream.cuda_stream)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return UNO_F32
    if t.dtype == torch.bfloat16:
        return UNO_BF16
    raise TypeError(f"logits must be float32 or bfloat16, got {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(fn, status):
    if status != 0:
        raise UnoError(fn, status)


# Shape checks run before anything touches a device: the kernels index these
# arrays by the sizes passed alongside them, so a short array would be read
# past its end.
def _need(cond, msg):
    if not cond:
        raise ValueError(msg)


def _check_compact(q_ids, q_probs, q_count, rows):
    """q_ids and q_probs [rows, cap] of the same shape; q_count [rows]."""
    _need(q_ids.dim() == 2 and q_ids.shape[0] == rows and q_ids.shape[1] >= 1,
          f"q_ids must be [{rows}, cap] (one compact row per draft position)")
    _need(tuple(q_probs.shape) == tuple(q_ids.shape), "q_probs must have the shape of q_ids")
    _need(q_count.numel() == rows, f"q_count must hold {rows} entries")


def _check_linear(target_logits, draft_ids, q_ids, q_probs, q_count, R, B):
    _need(R >= 1 and B >= 1, "R and B must be positive")
    _need(target_logits.dim() >= 1 and target_logits.numel() == R * (B + 1) * target_logits.shape[-1],
          "target_logits must hold R*(B+1) rows")
    _need(draft_ids.numel() == R * B, "draft_ids must hold R*B tokens")
    _check_compact(q_ids, q_probs, q_count, R * B)


def _dev(t: torch.Tensor, device) -> torch.Tensor:
    return t if t.device == device else t.to(device, non_blocking=True)


def _device_of(*ts):
    for t in ts:
        if isinstance(t, torch.Tensor) and t.is_cuda:
            return t.device
    return torch.device("cuda", torch.cuda.current_device())


def _host_back(out: dict, host: bool) -> dict:
    if not host:
        return out
    return {k: v.to("cpu", non_blocking=False) for k, v in out.items()}


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------
def uno_filter_softmax(logits, *, temperature, top_k, top_p, rows_per_request=1, cap=None, rng=None,
                       dense=False, order="topk_first", top_k_max=None, per_request=False):
    """Filter each row of logits [rows, vocab] (top-k, then top-p, softmax).

    Returns dict(ids [rows, cap] int32, probs [rows, cap] float32, count [rows],
    flags [rows] uint32 as int32, and sample [rows] when rng=(seed, cycle),
    dense [rows, vocab] when dense=True)."""
    lib = load_library()
    _need(logits.dim() == 2 and logits.stride(1) == 1, "logits must be [rows, vocab] with unit inner stride")
    host = not logits.is_cuda
    device = _device_of(logits)
    x = _dev(logits, device)
    rows, vocab = x.shape
    rpr = int(rows_per_request)
    pr = _per_request(temperature, top_k, top_p, order, (rows + rpr - 1) // max(rpr, 1), device, top_k_max,
                      per_request)
    kb = pr.top_k_max if pr is not None else int(top_k)
    if cap is None:
        cap = min(kb, vocab)
    stream = torch.cuda.current_stream(device)
    kw = dict(dtype=torch.int32, device=device)
    ids = torch.empty((rows, cap), **kw)
    probs = torch.empty((rows, cap), dtype=torch.float32, device=device)
    count = torch.empty(rows, **kw)
    flags = torch.empty(rows, **kw)
    dn = torch.empty((rows, vocab), dtype=torch.float32, device=device) if dense else None
    sample = torch.empty(rows, **kw) if rng is not None else None
    rng_c = ctypes.byref(_rng(rng)) if rng is not None else None
    nbytes = lib.uno_filter_softmax_workspace_bytes(rows, vocab, kb)
    ws = workspace(nbytes, device, stream)
    if pr is None:
        st = lib.uno_filter_softmax(_ptr(x), _dtype_code(x), rows, vocab, x.stride(0), rpr,
                                    _Params(float(temperature), int(top_k), float(top_p)), int(cap), _ptr(ids),
                                    _ptr(probs), _ptr(count), _ptr(dn), rng_c, _ptr(sample), _ptr(flags),
                                    _ptr(ws), ws.numel(), ctypes.c_void_p(stream.cuda_stream))
        _check("uno_filter_softmax", st)
    else:
        st = lib.uno_filter_softmax_params(_ptr(x), _dtype_code(x), rows, vocab, x.stride(0), rpr,
                                           ctypes.byref(pr.c), int(cap), _ptr(ids), _ptr(probs), _ptr(count),
                                           _ptr(dn), rng_c, _ptr(sample), _ptr(flags), _ptr(ws), ws.numel(),
                                           ctypes.c_void_p(stream.cuda_stream))
        _check("uno_filter_softmax_params", st)
    out = dict(ids=ids, probs=probs, count=count, flags=flags)
    if dense:
        out["dense"] = dn
    if rng is not None:
        out["sample"] = sample
    return _host_back(out, host)


def uno_linear_verify(target_logits, draft_ids, q_ids, q_probs, q_count, *, R, B, temperature, top_k, top_p,
                      rng, order="topk_first", top_k_max=None, per_request=False):
    """Linear rejection sampling.  target_logits [R*(B+1), vocab] (or
    [R, B+1, vocab]); draft_ids [R, B]; q_* as returned by uno_filter_softmax
    for the R*B draft rows.  Returns dict(tokens [R, B+1], accept_len,
    num_tokens, flags)."""
    lib = load_library()
    _check_linear(target_logits, draft_ids, q_ids, q_probs, q_count, R, B)
    host = not target_logits.is_cuda
    device = _device_of(target_logits, draft_ids, q_ids)
    x = _dev(target_logits, device).contiguous()
    vocab = x.shape[-1]
    d = _dev(draft_ids, device).to(torch.int32).contiguous()
    qi = _dev(q_ids, device).to(torch.int32).contiguous()
    qp = _dev(q_probs, device).to(torch.float32).contiguous()
    qc = _dev(q_count, device).to(torch.int32).contiguous()
    stream = torch.cuda.current_stream(device)
    kw = dict(dtype=torch.int32, device=device)
    toks = torch.empty((R, B + 1), **kw)
    acc = torch.empty(R, **kw)
    ntok = torch.empty(R, **kw)
    flags = torch.empty(R, **kw)
    pr = _per_request(temperature, top_k, top_p, order, R, device, top_k_max, per_request)
    kb = pr.top_k_max if pr is not None else int(top_k)
    nbytes = lib.uno_linear_verify_workspace_bytes(R, B, vocab, kb)
    ws = workspace(nbytes, device, stream)
    if pr is None:
        st = lib.uno_linear_verify(_ptr(x), _dtype_code(x), R, B, vocab,
                                   _Params(float(temperature), int(top_k), float(top_p)), _ptr(d), _ptr(qi),
                                   _ptr(qp), _ptr(qc), qi.shape[1], _rng(rng), _ptr(toks),
                                   _ptr(acc), _ptr(ntok), _ptr(flags), _ptr(ws), ws.numel(),
                                   ctypes.c_void_p(stream.cuda_stream))
        _check("uno_linear_verify", st)
    else:
        st = lib.uno_linear_verify_params(_ptr(x), _dtype_code(x), R, B, vocab, ctypes.byref(pr.c), _ptr(d),
                                          _ptr(qi), _ptr(qp), _ptr(qc), qi.shape[1], _rng(rng), _ptr(toks),
                                          _ptr(acc), _ptr(ntok), _ptr(flags), _ptr(ws), ws.numel(),
                                          ctypes.c_void_p(stream.cuda_stream))
        _check("uno_linear_verify_params", st)
    return _host_back(dict(tokens=toks, accept_len=acc, num_tokens=ntok, flags=flags), host)


LAYOUT_GENERIC, LAYOUT_TWO_PASS = 0, 1


def uno_linear_cycle(draft_logits, target_logits, *, R, B, temperature, top_k, top_p, rng, layout=LAYOUT_GENERIC,
                     order="topk_first", top_k_max=None, per_request=False):
    """One linear cycle in one call: draft_logits [R*B, vocab] (or [R, B,
    vocab]); target_logits [R*(B+1), vocab] for layout LAYOUT_GENERIC, [R*B,
    vocab] for LAYOUT_TWO_PASS (x_0 untested, target row i-1 tests x_i).
    Returns dict(tokens [R, B+1], num_accepted [R], num_tokens [R], flags [R],
    drafts [R, B])."""
    lib = load_library()
    _need(R >= 1 and B >= 1 and layout in (LAYOUT_GENERIC, LAYOUT_TWO_PASS), "R, B >= 1 and a known layout")
    host = not draft_logits.is_cuda
    device = _device_of(draft_logits, target_logits)
    d = _dev(draft_logits, device).contiguous()
    t = _dev(target_logits, device).contiguous()
    vocab = d.shape[-1]
    _need(t.shape[-1] == vocab and d.dtype == t.dtype, "draft and target logits share vocab and dtype")
    _need(d.numel() == R * B * vocab, "draft_logits must hold R*B rows")
    _need(t.numel() == R * (B + 1 - layout) * vocab, "target_logits must hold R*(B+1) rows (R*B two-pass)")
    stream = torch.cuda.current_stream(device)
    kw = dict(dtype=torch.int32, device=device)
    toks = torch.empty((R, B + 1), **kw)
    nacc = torch.empty(R, **kw)
    ntok = torch.empty(R, **kw)
    flags = torch.empty(R, **kw)
    drafts = torch.empty((R, B), **kw)
    pr = _per_request(temperature, top_k, top_p, order, R, device, top_k_max, per_request)
    kb = pr.top_k_max if pr is not None else int(top_k)
    nbytes = lib.uno_linear_cycle_workspace_bytes(R, B, vocab, kb, int(layout))
    ws = workspace(nbytes, device, stream)
    if pr is None:
        st = lib.uno_linear_cycle(_ptr(d), _ptr(t), _dtype_code(d), R, B, vocab, int(layout),
                                  _Params(float(temperature), int(top_k), float(top_p)), _rng(rng), _ptr(toks),
                                  _ptr(nacc), _ptr(ntok), _ptr(flags), _ptr(drafts), _ptr(ws), ws.numel(),
                                  ctypes.c_void_p(stream.cuda_stream))
        _check("uno_linear_cycle", st)
    else:
        st = lib.uno_linear_cycle_params(_ptr(d), _ptr(t), _dtype_code(d), R, B, vocab, int(layout),
                                         ctypes.byref(pr.c), _rng(rng), _ptr(toks), _ptr(nacc), _ptr(ntok),
                                         _ptr(flags), _ptr(drafts), _ptr(ws), ws.numel(),
                                         ctypes.c_void_p(stream.cuda_stream))
        _check("uno_linear_cycle_params", st)
    return _host_back(dict(tokens=toks, num_accepted=nacc, num_tokens=ntok, flags=flags, drafts=drafts), host)


def uno_tree_topk_expand(q_ids, q_probs, q_count, *, R, B, K, V):
    """Top-K candidates per marginal and best-first V-node trees.  Returns
    dict(node_token, node_parent, node_depth [R, V] int32, node_score [R, V]
    float32, num_nodes [R])."""
    lib = load_library()
    _need(R >= 1 and B >= 1, "R and B must be positive")
    _check_compact(q_ids, q_probs, q_count, R * B)
    host = not q_ids.is_cuda
    device = _device_of(q_ids)
    qi = _dev(q_ids, device).to(torch.int32).contiguous()
    qp = _dev(q_probs, device).to(torch.float32).contiguous()
    qc = _dev(q_count, device).to(torch.int32).contiguous()
    stream = torch.cuda.current_stream(device)
    kw = dict(dtype=torch.int32, device=device)
    tok = torch.empty((R, V), **kw)
    par = torch.empty((R, V), **kw)
    dep = torch.empty((R, V), **kw)
    sco = torch.empty((R, V), dtype=torch.float32, device=device)
    nn = torch.empty(R, **kw)
    st = lib.uno_tree_topk_expand(_ptr(qi), _ptr(qp), _ptr(qc), qi.shape[1], R, B, K, V, _ptr(tok), _ptr(par),
                                  _ptr(dep), _ptr(sco), _ptr(nn), ctypes.c_void_p(stream.cuda_stream))
    _check("uno_tree_topk_expand", st)
    return _host_back(dict(node_token=tok, node_parent=par, node_depth=dep, node_score=sco, num_nodes=nn), host)


def uno_tree_verify(target_logits, node_token, node_parent, num_nodes, *, R, B, V, temperature, top_k, top_p,
                    rng, order="topk_first", top_k_max=None, per_request=False):
    """Target-only tree verification.  target_logits [R*V, vocab] (one row
    per node).  Returns dict(tokens [R, B+1], accept_len, num_tokens,
    path_nodes [R, B+1], flags)."""
    lib = load_library()
    _need(R >= 1 and V >= 1, "R and V must be positive")
    _need(target_logits.dim() >= 1 and target_logits.numel() == R * V * target_logits.shape[-1],
          "target_logits must hold R*V rows")
    _need(node_token.numel() == R * V and node_parent.numel() == R * V,
          "node_token and node_parent must hold R*V entries")
    _need(num_nodes.numel() == R, "num_nodes must hold R entries")
    host = not target_logits.is_cuda
    device = _device_of(target_logits, node_token)
    x = _dev(target_logits, device).contiguous()
    vocab = x.shape[-1]
    tk = _dev(node_token, device).to(torch.int32).contiguous()
    pa = _dev(node_parent, device).to(torch.int32).contiguous()
    nn = _dev(num_nodes, device).to(torch.int32).contiguous()
    stream = torch.cuda.current_stream(device)
    kw = dict(dtype=torch.int32, device=device)
    toks = torch.empty((R, B + 1), **kw)
    path = torch.empty((R, B + 1), **kw)
    acc = torch.empty(R, **kw)
    ntok = torch.empty(R, **kw)
    flags = torch.empty(R, **kw)
    pr = _per_request(temperature, top_k, top_p, order, R, device, top_k_max, per_request)
    kb = pr.top_k_max if pr is not None else int(top_k)
    nbytes = lib.uno_tree_verify_workspace_bytes(R, V, vocab, kb)
    ws = workspace(nbytes, device, stream)
    if pr is None:
        st = lib.uno_tree_verify(_ptr(x), _dtype_code(x), R, B, V, vocab,
                                 _Params(float(temperature), int(top_k), float(top_p)), _ptr(tk), _ptr(pa),
                                 _ptr(nn), _rng(rng), _ptr(toks), _ptr(acc), _ptr(ntok), _ptr(path),
                                 _ptr(flags), _ptr(ws), ws.numel(), ctypes.c_void_p(stream.cuda_stream))
        _check("uno_tree_verify", st)
    else:
        st = lib.uno_tree_verify_params(_ptr(x), _dtype_code(x), R, B, V, vocab, ctypes.byref(pr.c), _ptr(tk),
                                        _ptr(pa), _ptr(nn), _rng(rng), _ptr(toks), _ptr(acc), _ptr(ntok),
                                        _ptr(path), _ptr(flags), _ptr(ws), ws.numel(),
                                        ctypes.c_void_p(stream.cuda_stream))
        _check("uno_tree_verify_params", st)
    return _host_back(dict(tokens=toks, accept_len=acc, num_tokens=ntok, path_nodes=path, flags=flags), host)


def uno_filter_softmax_params(logits, *, temperature, top_k, top_p, order="topk_first", top_k_max=None, **kw):
    """uno_filter_softmax through the per-request entry point: temperature,
    top_k and top_p hold one entry per request (scalars are repeated)."""
    return uno_filter_softmax(logits, temperature=temperature, top_k=top_k, top_p=top_p, order=order,
                              top_k_max=top_k_max, per_request=True, **kw)


def uno_linear_verify_params(*args, temperature, top_k, top_p, order="topk_first", top_k_max=None, **kw):
    """uno_linear_verify through the per-request entry point."""
    return uno_linear_verify(*args, temperature=temperature, top_k=top_k, top_p=top_p, order=order,
                             top_k_max=top_k_max, per_request=True, **kw)


def uno_linear_cycle_params(*args, temperature, top_k, top_p, order="topk_first", top_k_max=None, **kw):
    """uno_linear_cycle through the per-request entry point."""
    return uno_linear_cycle(*args, temperature=temperature, top_k=top_k, top_p=top_p, order=order,
                            top_k_max=top_k_max, per_request=True, **kw)


def uno_tree_verify_params(*args, temperature, top_k, top_p, order="topk_first", top_k_max=None, **kw):
    """uno_tree_verify through the per-request entry point."""
    return uno_tree_verify(*args, temperature=temperature, top_k=top_k, top_p=top_p, order=order,
                           top_k_max=top_k_max, per_request=True, **kw)


def uno_linear_verify_noalloc(target_logits, draft_ids, q_ids, q_probs, q_count, *, R, B, temperature, top_k,
                              top_p, rng):
    """uno_linear_verify for callers that cannot give the library a workspace
    (for instance a serving loop whose free device memory all belongs to its
    KV-cache pool): the scratch is a fixed 8 MiB device array owned by the
    library.  Same arguments and results as uno_linear_verify; only the output
    tensors are allocated here, by PyTorch, as for every entry point."""
    lib = load_library()
    _check_linear(target_logits, draft_ids, q_ids, q_probs, q_count, R, B)
    host = not target_logits.is_cuda
    device = _device_of(target_logits, draft_ids, q_ids)
    x = _dev(target_logits, device).contiguous()
    vocab = x.shape[-1]
    d = _dev(draft_ids, device).to(torch.int32).contiguous()
    qi = _dev(q_ids, device).to(torch.int32).contiguous()
    qp = _dev(q_probs, device).to(torch.float32).contiguous()
    qc = _dev(q_count, device).to(torch.int32).contiguous()
    stream = torch.cuda.current_stream(device)
    kw = dict(dtype=torch.int32, device=device)
    toks = torch.empty((R, B + 1), **kw)
    acc = torch.empty(R, **kw)
    ntok = torch.empty(R, **kw)
    flags = torch.empty(R, **kw)
    st = lib.uno_linear_verify_noalloc(_ptr(x), _dtype_code(x), R, B, vocab,
                                       _Params(float(temperature), int(top_k), float(top_p)), _ptr(d), _ptr(qi),
                                       _ptr(qp), _ptr(qc), qi.shape[1], _rng(rng), _ptr(toks), _ptr(acc), _ptr(ntok),
                                       _ptr(flags), ctypes.c_void_p(stream.cuda_stream))
    _check("uno_linear_verify_noalloc", st)
    return _host_back(dict(tokens=toks, accept_len=acc, num_tokens=ntok, flags=flags), host)


def uno_tree_suffix_attention_merge(q, k, v, node_parent, num_nodes, o_prefix, lse_prefix, *, scale):
    """Tree-suffix attention merged with the prefix state by log-sum-exp.

    q [R, V, H, d], k and v [R, V, Hkv, d] (float32 or bfloat16, one dtype);
    node_parent [R, V], num_nodes [R]; o_prefix [R, V, H, d] and lse_prefix
    [R, V, H] float32 (lse -inf: empty prefix).  Returns dict(o [R, V, H, d],
    lse [R, V, H] float32, flags [R])."""
    lib = load_library()
    _need(q.dim() == 4 and k.dim() == 4 and v.dim() == 4, "q, k and v must be [R, V, heads, d]")
    R, V, H, d = q.shape
    Hkv = k.shape[2]
    _need(tuple(k.shape) == (R, V, Hkv, d) and tuple(v.shape) == tuple(k.shape),
          "k and v must be [R, V, Hkv, d] with q's R, V and d")
    _need(k.dtype == q.dtype and v.dtype == q.dtype, "q, k and v must share one dtype")
    _need(node_parent.numel() == R * V and num_nodes.numel() == R, "node_parent [R, V] and num_nodes [R]")
    _need(tuple(o_prefix.shape) == (R, V, H, d) and tuple(lse_prefix.shape) == (R, V, H),
          "o_prefix must be [R, V, H, d] and lse_prefix [R, V, H]")
    host = not q.is_cuda
    device = _device_of(q, k, v)
    code = _dtype_code(q)
    qd, kd, vd = (_dev(t, device).contiguous() for t in (q, k, v))
    pa = _dev(node_parent, device).to(torch.int32).contiguous()
    nn = _dev(num_nodes, device).to(torch.int32).contiguous()
    op = _dev(o_prefix, device).to(torch.float32).contiguous()
    lp = _dev(lse_prefix, device).to(torch.float32).contiguous()
    stream = torch.cuda.current_stream(device)
    o = torch.empty((R, V, H, d), dtype=torch.float32, device=device)
    lse = torch.empty((R, V, H), dtype=torch.float32, device=device)
    flags = torch.empty(R, dtype=torch.int32, device=device)
    st = lib.uno_tree_suffix_attention_merge(_ptr(qd), _ptr(kd), _ptr(vd), code, R, V, H, Hkv, d, float(scale),
                                             _ptr(pa), _ptr(nn), _ptr(op), _ptr(lp), _ptr(o), _ptr(lse),
                                             _ptr(flags), ctypes.c_void_p(stream.cuda_stream))
    _check("uno_tree_suffix_attention_merge", st)
    return _host_back(dict(o=o, lse=lse, flags=flags), host)
