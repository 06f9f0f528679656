"""uno_linear_verify_noalloc, the entry point for callers that cannot give the
library device memory (a serving loop whose free memory all belongs to its
KV-cache pool, or a plugin host without an allocator), must return what
uno_linear_verify returns with a caller workspace, and what the oracle returns.

This file is collected last on purpose: it passes when run alone in a fresh
process and when run after every other test."""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import oracle
from _parity import Events, compare_requests, to_device
from speculative_decoding_verification_filter_b200 import (uno_filter_softmax, uno_linear_verify,
                                                          uno_linear_verify_noalloc)
from speculative_decoding_verification_filter_b200 import _binding as b
from speculative_decoding_verification_filter_b200.inputs import Workload, linear_draft, linear_target

KEYS = ("tokens", "accept_len", "num_tokens", "flags")
NOALLOC_SCRATCH_BYTES = 8 << 20  # UNO_NOALLOC_SCRATCH_BYTES


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Checked on the host before any device work.  The call runs in a child
    process that sees no GPU, so a regression that reached a launch would
    report a CUDA error there instead of starting kernels on the fake
    pointers."""
    lib = b.load_library()
    assert lib.uno_linear_verify_workspace_bytes(512, 16, 151936, 200) > NOALLOC_SCRATCH_BYTES
    child = textwrap.dedent("""
        import ctypes
        from speculative_decoding_verification_filter_b200 import _binding as b
        lib = b.load_library()
        fake = ctypes.c_void_p(0x1000)
        st = lib.uno_linear_verify_noalloc(fake, 1, 512, 16, 151936, b._Params(1.0, 200, 0.95), fake, fake, fake,
                                           fake, 200, b._Rng(1, 0, 0), fake, fake, fake, fake, None)
        print(st)
    """)
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-c", child], cwd=root, env=env, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr
    assert int(out.stdout.strip().splitlines()[-1]) == 2  # UNO_ERR_UNSUPPORTED


# (R, B, vocab, dtype, top_k): the batch shape of the linear 8/1/8 workload,
# an fp32 vocabulary with a ragged tail, a few rows (fewer rows than SMs: one
# CTA per row) and top_k above 64 (the general row kernel)
CASES = [
    (64, 8, 151936, "bf16", 50),
    (64, 8, 5003, "f32", 50),
    (2, 3, 151936, "bf16", 50),
    (3, 4, 40000, "f32", 100),
]


@pytest.mark.gpu
@pytest.mark.parametrize("R,B,vocab,dtype,top_k", CASES)
def test_noalloc_matches_the_workspace_entry_point_and_the_oracle(R, B, vocab, dtype, top_k):
    w = Workload("noalloc", "linear", R=R, B=B, vocab=vocab, dtype=dtype, sigma=1.0, noise=0.7, peak=8.0, seed=77,
                 top_k=top_k)
    sp = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)
    q_np, p_np = linear_draft(w), linear_target(w)
    q, p = to_device(q_np, w.dtype), to_device(p_np, w.dtype)
    ev = Events()
    for cycle in (0, 1):  # two calls in a row: the shared array keeps the last call's contents
        rng = (w.seed, cycle, 0)
        gq = uno_filter_softmax(q, rows_per_request=w.B, rng=rng, **sp)
        drafts = gq["sample"].reshape(w.R, w.B)
        ref = uno_linear_verify(p, drafts, gq["ids"], gq["probs"], gq["count"], R=w.R, B=w.B, rng=rng, **sp)
        got = uno_linear_verify_noalloc(p, drafts, gq["ids"], gq["probs"], gq["count"], R=w.R, B=w.B, rng=rng, **sp)
        torch.cuda.synchronize()
        for key in KEYS:  # integer results: the tests' tolerance is exact equality
            assert torch.equal(got[key], ref[key]), (cycle, key)
        acc = got["accept_len"].cpu().numpy()
        assert np.all((acc >= 0) & (acc <= w.B))
        # the oracle on the first and last requests, from its own filtered drafts
        for r in sorted({0, w.R - 1}):
            rq = oracle.filter_softmax(q_np[r * w.B:(r + 1) * w.B], w.dtype, w.temperature, w.top_k, w.top_p,
                                       rows_per_request=w.B, rng=(w.seed, cycle, r))
            ro = oracle.linear_verify(p_np[r * (w.B + 1):(r + 1) * (w.B + 1)], w.dtype, 1, w.B, w.temperature,
                                      w.top_k, w.top_p, rq["sample"].reshape(1, w.B), rq["ids"], rq["probs"],
                                      rq["count"], rng=(w.seed, cycle, r))
            compare_requests(got, ro, ev, KEYS, reqs=[r])
    ev.check()
