"""The C-ABI library loads without a GPU and exports every function that
include/uno_filter.h declares; argument errors are caught on the host."""
import ctypes
import re
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent
HEADER = ROOT / "include" / "uno_filter.h"


def _declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(uno_[a-z0-9_]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def _lib():
    from speculative_decoding_verification_filter_b200 import build
    build.build()
    return ctypes.CDLL(str(build.LIB))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for n in ("uno_filter_softmax", "uno_linear_verify", "uno_tree_topk_expand", "uno_tree_verify",
              "uno_status_string"):
        assert n in names


def test_library_exports_every_declared_function():
    lib = _lib()
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_names_match_the_header():
    import speculative_decoding_verification_filter_b200 as pkg
    for n in _declared_functions():
        if n.endswith("_workspace_bytes") or n == "uno_status_string":
            continue
        assert hasattr(pkg, n), n


def test_status_strings_and_workspace_sizes_without_gpu():
    lib = _lib()
    lib.uno_status_string.restype = ctypes.c_char_p
    assert lib.uno_status_string(0) == b"ok"
    assert lib.uno_status_string(1) == b"invalid argument"
    lib.uno_linear_verify_workspace_bytes.restype = ctypes.c_size_t
    lib.uno_linear_verify_workspace_bytes.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32]
    a = lib.uno_linear_verify_workspace_bytes(64, 8, 151936, 50)
    b = lib.uno_linear_verify_workspace_bytes(64, 8, 151936, 51)
    assert 0 < a <= b
    assert lib.uno_linear_verify_workspace_bytes(0, 8, 151936, 50) == 0


@pytest.mark.parametrize("bad", [
    dict(rows=0), dict(vocab=0), dict(top_k=0), dict(top_p=0.0), dict(top_p=1.5), dict(temperature=-1.0),
    dict(temperature=float("inf")), dict(stride=5), dict(null_logits=True),
])
def test_filter_rejects_bad_arguments_on_the_host(bad):
    """Invalid arguments return an error before anything touches a device, so
    these calls are safe without a GPU (the pointers are never dereferenced)."""
    from speculative_decoding_verification_filter_b200 import _binding as b
    lib = b.load_library()
    rows, vocab = bad.get("rows", 4), bad.get("vocab", 10)
    sp = b._Params(bad.get("temperature", 1.0), bad.get("top_k", 5), bad.get("top_p", 0.9))
    fake = ctypes.c_void_p(0x1000)
    logits = None if bad.get("null_logits") else fake
    st = lib.uno_filter_softmax(logits, 0, rows, vocab, bad.get("stride", vocab), 1, sp, 8, fake, fake, fake, None,
                                None, None, fake, fake, 1 << 20, None)
    assert st == 1


def test_tree_shapes_rejected_on_the_host():
    from speculative_decoding_verification_filter_b200 import _binding as b
    lib = b.load_library()
    fake = ctypes.c_void_p(0x1000)
    for B, K, V in [(8, 2, 7), (4, 2, 129), (4, 64, 64)]:
        st = lib.uno_tree_topk_expand(fake, fake, fake, 50, 1, B, K, V, fake, fake, fake, fake, fake, None)
        assert st == 1
    # short workspace
    sp = b._Params(1.0, 50, 0.95)
    st = lib.uno_tree_verify(fake, 1, 1, 4, 8, 1000, sp, fake, fake, fake, b._Rng(1, 0), fake, fake, fake, fake,
                             fake, fake, 16, None)
    assert st == 4


@pytest.mark.parametrize("bad,status", [
    (dict(V=129), 1), (dict(V=0), 1), (dict(H=6, Hkv=4), 1), (dict(d=0), 1), (dict(dt=7), 1),
    (dict(scale=float("nan")), 1), (dict(null_q=True), 1), (dict(d=257), 2), (dict(V=128, d=256), 2),
])
def test_suffix_attention_rejects_bad_arguments_on_the_host(bad, status):
    """Argument errors return before any device work (fake pointers are
    never dereferenced)."""
    from speculative_decoding_verification_filter_b200 import _binding as b
    lib = b.load_library()
    fake = ctypes.c_void_p(0x1000)
    a = dict(R=2, V=8, H=4, Hkv=2, d=16, dt=0, scale=0.25)
    a.update({k: v for k, v in bad.items() if k != "null_q"})
    q = None if bad.get("null_q") else fake
    st = lib.uno_tree_suffix_attention_merge(q, fake, fake, a["dt"], a["R"], a["V"], a["H"], a["Hkv"], a["d"],
                                             a["scale"], fake, fake, fake, fake, fake, fake, None, None)
    assert st == status


def test_misaligned_cycle_word_rejected_on_the_host():
    """A device cycle word must be 4-byte aligned; a misaligned address is an
    argument error returned before any device work."""
    from speculative_decoding_verification_filter_b200 import _binding as b
    lib = b.load_library()
    fake = ctypes.c_void_p(0x1000)
    rng = b._Rng(1, 0, 0, ctypes.c_void_p(0x1002))
    sp = b._Params(1.0, 5, 0.9)
    st = lib.uno_filter_softmax(fake, 0, 4, 10, 10, 1, sp, 8, fake, fake, fake, None, ctypes.byref(rng), fake, fake,
                                fake, 1 << 20, None)
    assert st == 1
    st = lib.uno_tree_verify(fake, 1, 1, 4, 8, 1000, b._Params(1.0, 50, 0.95), fake, fake, fake, rng, fake, fake,
                             fake, fake, fake, fake, 1 << 24, None)
    assert st == 1


@pytest.mark.parametrize("bad", ["null", "order", "kmax", "misaligned", "null_array"])
def test_request_params_rejected_on_the_host(bad):
    """The per-request entry points check the parameter struct on the host
    before any device work (the fake pointers are never dereferenced)."""
    from speculative_decoding_verification_filter_b200 import _binding as b
    lib = b.load_library()
    fake = ctypes.c_void_p(0x1000)
    a = dict(T=0x1000, k=0x2000, p=0x3000, kmax=5, order=0)
    if bad == "order":
        a["order"] = 7
    elif bad == "kmax":
        a["kmax"] = 0
    elif bad == "misaligned":
        a["k"] = 0x2002
    elif bad == "null_array":
        a["p"] = None
    rp = None if bad == "null" else ctypes.byref(
        b._ReqParams(ctypes.c_void_p(a["T"]), ctypes.c_void_p(a["k"]), ctypes.c_void_p(a["p"]) if a["p"] else None,
                     a["kmax"], a["order"]))
    st = lib.uno_filter_softmax_params(fake, 0, 4, 10, 10, 1, rp, 8, fake, fake, fake, None, None, None, fake, fake,
                                       1 << 20, None)
    assert st == 1
    st = lib.uno_linear_verify_params(fake, 1, 1, 4, 1000, rp, fake, fake, fake, fake, 8, b._Rng(1, 0), fake, fake,
                                      fake, fake, fake, 1 << 24, None)
    assert st == 1
