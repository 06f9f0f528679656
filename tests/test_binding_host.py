"""The Python binding checks array shapes on the host, before any device work.

The kernels index every array by the sizes passed with it, so a mis-shaped
array must be refused before a launch.  Each check below runs without a GPU:
the device step is replaced by a stub that raises, so a call that passes the
shape checks stops there, having touched no device.
"""
import pytest
import torch

from speculative_decoding_verification_filter_b200 import _binding as b


class _Reached(Exception):
    pass


@pytest.fixture(autouse=True)
def _no_device(monkeypatch):
    def stop(*_):
        raise _Reached()
    monkeypatch.setattr(b, "_device_of", stop)
    b.load_library()


def _i32(*shape):
    return torch.zeros(shape, dtype=torch.int32)


def _f32(*shape):
    return torch.zeros(shape, dtype=torch.float32)


SP = dict(temperature=1.0, top_k=4, top_p=0.9)


def _linear_args(R=3, B=2, vocab=16, cap=4):
    return dict(target_logits=_f32(R * (B + 1), vocab), draft_ids=_i32(R, B), q_ids=_i32(R * B, cap),
                q_probs=_f32(R * B, cap), q_count=_i32(R * B))


def test_filter_shapes():
    with pytest.raises(_Reached):
        b.uno_filter_softmax(_f32(4, 16), **SP)
    with pytest.raises(ValueError):
        b.uno_filter_softmax(_f32(16), **SP)
    with pytest.raises(ValueError):
        b.uno_filter_softmax(_f32(16, 4).t(), **SP)  # inner stride 4


@pytest.mark.parametrize("fn", [b.uno_linear_verify, b.uno_linear_verify_noalloc])
def test_linear_shapes(fn):
    R, B = 3, 2
    with pytest.raises(_Reached):
        fn(**_linear_args(), R=R, B=B, rng=(1, 0), **SP)
    with pytest.raises(_Reached):  # [R, B+1, vocab] logits are accepted too
        fn(**dict(_linear_args(), target_logits=_f32(R, B + 1, 16)), R=R, B=B, rng=(1, 0), **SP)
    bad = [
        dict(target_logits=_f32(R * B, 16)),   # B rows per request, not B+1
        dict(draft_ids=_i32(R, B - 1)),
        dict(q_ids=_i32(R * B - 1, 4), q_probs=_f32(R * B - 1, 4)),
        dict(q_probs=_f32(R * B, 3)),          # narrower than q_ids
        dict(q_ids=_i32(R * B * 4)),           # not [rows, cap]
        dict(q_count=_i32(R * B + 1)),
    ]
    for change in bad:
        with pytest.raises(ValueError):
            fn(**dict(_linear_args(), **change), R=R, B=B, rng=(1, 0), **SP)
    with pytest.raises(ValueError):
        fn(**_linear_args(), R=0, B=B, rng=(1, 0), **SP)


def test_tree_expand_shapes():
    R, B, cap = 2, 3, 5
    ok = dict(q_ids=_i32(R * B, cap), q_probs=_f32(R * B, cap), q_count=_i32(R * B))
    with pytest.raises(_Reached):
        b.uno_tree_topk_expand(**ok, R=R, B=B, K=2, V=4)
    for change in [dict(q_probs=_f32(R * B, cap - 1)), dict(q_count=_i32(R)),
                   dict(q_ids=_i32(R, cap), q_probs=_f32(R, cap))]:
        with pytest.raises(ValueError):
            b.uno_tree_topk_expand(**dict(ok, **change), R=R, B=B, K=2, V=4)


def test_tree_verify_shapes():
    R, B, V, vocab = 2, 2, 4, 16
    ok = dict(target_logits=_f32(R * V, vocab), node_token=_i32(R, V), node_parent=_i32(R, V),
              num_nodes=_i32(R))
    with pytest.raises(_Reached):
        b.uno_tree_verify(**ok, R=R, B=B, V=V, rng=(1, 0), **SP)
    for change in [dict(target_logits=_f32(R * V - 1, vocab)), dict(node_token=_i32(R, V - 1)),
                   dict(node_parent=_i32(R - 1, V)), dict(num_nodes=_i32(R + 1))]:
        with pytest.raises(ValueError):
            b.uno_tree_verify(**dict(ok, **change), R=R, B=B, V=V, rng=(1, 0), **SP)


def test_suffix_attention_shapes():
    R, V, H, Hkv, d = 2, 5, 4, 2, 8
    ok = dict(q=_f32(R, V, H, d), k=_f32(R, V, Hkv, d), v=_f32(R, V, Hkv, d), node_parent=_i32(R, V),
              num_nodes=_i32(R), o_prefix=_f32(R, V, H, d), lse_prefix=_f32(R, V, H))
    with pytest.raises(_Reached):
        b.uno_tree_suffix_attention_merge(**ok, scale=0.3)
    for change in [dict(q=_f32(R, V, H * d)), dict(k=_f32(R, V, Hkv, d + 1)), dict(v=_f32(R, V - 1, Hkv, d)),
                   dict(k=torch.zeros((R, V, Hkv, d), dtype=torch.bfloat16)), dict(node_parent=_i32(R, V + 1)),
                   dict(num_nodes=_i32(R + 1)), dict(o_prefix=_f32(R, V, H, d - 1)), dict(lse_prefix=_f32(R, V))]:
        with pytest.raises(ValueError):
            b.uno_tree_suffix_attention_merge(**dict(ok, **change), scale=0.3)
