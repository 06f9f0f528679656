"""uno_linear_verify_noalloc, the entry point for callers that cannot give the
library device memory (a serving loop whose free memory all belongs to its
KV-cache pool, or a plugin host without an allocator), must return what
uno_linear_verify returns with a caller workspace.

This file is collected last on purpose: it passes when run alone in a fresh
process and when run after every other test."""
import ctypes

import numpy as np
import pytest
import torch

from _parity import to_device
from speculative_decoding_verification_filter_b200 import (uno_filter_softmax, uno_linear_verify,
                                                          uno_linear_verify_noalloc)
from speculative_decoding_verification_filter_b200 import _binding as b
from speculative_decoding_verification_filter_b200.inputs import Workload, linear_draft, linear_target

KEYS = ("tokens", "accept_len", "num_tokens", "flags")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Checked on the host before any device work, so no GPU is needed: 512
    requests with B = 16 at top_k 200 need more scratch than the fixed array
    holds."""
    lib = b.load_library()
    fake = ctypes.c_void_p(0x1000)
    st = lib.uno_linear_verify_noalloc(fake, 1, 512, 16, 151936, b._Params(1.0, 200, 0.95), fake, fake, fake, fake,
                                       200, b._Rng(1, 0, 0), fake, fake, fake, fake, None)
    assert st == 2  # UNO_ERR_UNSUPPORTED


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,vocab", [("bf16", 151936), ("f32", 5003)])
def test_noalloc_matches_the_workspace_entry_point_twice(dtype, vocab):
    w = Workload("noalloc", "linear", R=64, B=8, vocab=vocab, dtype=dtype, sigma=1.0, noise=0.7, peak=8.0, seed=77)
    sp = dict(temperature=w.temperature, top_k=w.top_k, top_p=w.top_p)
    q = to_device(linear_draft(w), w.dtype)
    p = to_device(linear_target(w), w.dtype)
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
