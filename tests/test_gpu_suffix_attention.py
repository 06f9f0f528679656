"""GPU parity of uno_tree_suffix_attention_merge with the oracle (through the
C ABI).

Tolerance: the kernel accumulates d <= 128 products and the softmax sums in
binary32 and uses binary32 exp/log; on unit-normal data that moves outputs
and LSEs by a few 1e-6.  The bar, 5e-5 absolute on both, leaves a margin of
about ten.  Both sides read the same inputs: bf16 rows are decoded exactly,
and the prefix state is the binary32 array the kernel receives.
"""
import numpy as np
import pytest
import torch

import oracle.suffix_attention as SA
from _defs import bf16_to_f32
from _parity import np_of, to_device
from speculative_decoding_verification_filter_b200 import FLAG_BAD_TREE, uno_tree_suffix_attention_merge
from speculative_decoding_verification_filter_b200.inputs import to_bf16_bits

pytestmark = pytest.mark.gpu

TOL = 5e-5


def _tensor(x, dtype):
    """(device tensor, the float64 values the kernel sees)."""
    if dtype == "bf16":
        bits = to_bf16_bits(x.astype(np.float32))
        return to_device(bits, "bf16"), bf16_to_f32(bits).astype(np.float64)
    x32 = x.astype(np.float32)
    return to_device(x32, "f32"), x32.astype(np.float64)


def _case(R, V, H, Hkv, d, L, seed, dtype, num_nodes=None, chain=False, empty_prefix=()):
    rng = np.random.default_rng(seed)
    scale = 1.0 / np.sqrt(d)
    q_d, q = _tensor(rng.standard_normal((R, V, H, d)), dtype)
    k_d, k = _tensor(rng.standard_normal((R, V, Hkv, d)), dtype)
    v_d, v = _tensor(rng.standard_normal((R, V, Hkv, d)), dtype)
    if chain:
        parent = np.tile(np.arange(-1, V - 1), (R, 1))
    else:
        parent = np.array([[-1] + [int(rng.integers(0, j)) for j in range(1, V)] for _ in range(R)])
    n = np.full(R, V) if num_nodes is None else np.asarray(num_nodes)
    op = np.zeros((R, V, H, d), dtype=np.float32)
    lp = np.zeros((R, V, H), dtype=np.float32)
    for r in range(R):
        Lr = 0 if r in empty_prefix else L
        kp = rng.standard_normal((Lr, Hkv, d))
        vp = rng.standard_normal((Lr, Hkv, d))
        a, b = SA.prefix_attention(q[r], kp, vp, scale)
        op[r], lp[r] = a, b
    dev = dict(q=q_d, k=k_d, v=v_d, node_parent=torch.from_numpy(parent.astype(np.int32)).cuda(),
               num_nodes=torch.from_numpy(n.astype(np.int32)).cuda(), o_prefix=torch.from_numpy(op).cuda(),
               lse_prefix=torch.from_numpy(lp).cuda())
    host = dict(q=q, k=k, v=v, parent=parent, n=n, op=op.astype(np.float64), lp=lp.astype(np.float64))
    return dev, host, scale


def _check(dev, host, scale, skip=()):
    out = uno_tree_suffix_attention_merge(**dev, scale=scale)
    torch.cuda.synchronize()
    o, lse, flags = np_of(out["o"]), np_of(out["lse"]), np_of(out["flags"])
    R = o.shape[0]
    for r in range(R):
        if r in skip:
            continue
        n = int(host["n"][r])
        ro, rl = SA.suffix_attention_merge(host["q"][r, :n], host["k"][r, :n], host["v"][r, :n],
                                           host["parent"][r, :n], host["op"][r, :n], host["lp"][r, :n], scale)
        assert np.max(np.abs(o[r, :n] - ro)) < TOL, r
        assert np.max(np.abs(lse[r, :n] - rl)) < TOL, r
        assert np.all(o[r, n:] == 0) and np.all(np.isneginf(lse[r, n:]))  # nodes past num_nodes
        assert flags[r] == 0
    return o, lse, flags


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_small_trees_with_padding_and_an_empty_prefix(dtype):
    dev, host, scale = _case(3, 9, 4, 2, 16, 23, 1, dtype, num_nodes=[9, 6, 9], empty_prefix=(2,))
    _check(dev, host, scale)


def test_attention_shape_of_an_8b_model():
    # 32 query heads over 8 key/value heads, head dim 128, a 32-node tree
    dev, host, scale = _case(4, 32, 32, 8, 128, 64, 2, "bf16")
    _check(dev, host, scale)


def test_largest_tree_as_a_chain():
    dev, host, scale = _case(2, 128, 4, 4, 64, 17, 3, "f32", chain=True)
    _check(dev, host, scale)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])  # the CUDA-core and the tensor-core kernel
def test_bad_tree_is_flagged_and_confined_to_its_request(dtype):
    dev, host, scale = _case(3, 8, 4, 2, 32, 9, 4, dtype)
    parent = dev["node_parent"].clone()
    parent[1, 3] = 6  # a parent after its child
    dev["node_parent"] = parent
    _, _, flags = _check(dev, host, scale, skip=(1,))
    assert flags[1] == FLAG_BAD_TREE


# bf16 rows with d a multiple of 16 take the tensor-core kernel: stacked rows
# G * V spanning several 128-row tiles, V not a multiple of 16, head dims 32
# to 256, the largest tree, and padding past num_nodes
@pytest.mark.parametrize("R,V,H,Hkv,d,L,seed,kw", [
    (2, 40, 16, 2, 32, 12, 11, {}),
    (3, 20, 8, 1, 256, 30, 12, dict(num_nodes=[20, 7, 13])),
    (2, 128, 4, 4, 64, 5, 13, dict(chain=True)),
    (2, 128, 2, 1, 64, 9, 14, {}),
    (5, 3, 4, 4, 16, 0, 15, dict(empty_prefix=(0, 1, 2, 3, 4))),
])
def test_tensor_core_shapes(R, V, H, Hkv, d, L, seed, kw):
    dev, host, scale = _case(R, V, H, Hkv, d, L, seed, "bf16", **kw)
    _check(dev, host, scale)


def test_misaligned_arrays_take_the_cuda_core_kernel():
    """The 8B-model shape with q, k, v and o_prefix starting one element past
    a 16-byte boundary: the tensor-core kernel would move them 16 bytes at a
    time, so the call runs on the CUDA-core kernel and matches the oracle."""
    dev, host, scale = _case(2, 32, 32, 8, 128, 20, 5, "bf16")

    def shifted(t):
        flat = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
        view = flat[1:].view(t.shape)
        view.copy_(t)
        return view

    for key in ("q", "k", "v", "o_prefix"):
        dev[key] = shifted(dev[key])
        assert dev[key].data_ptr() % 16 != 0, key
    _check(dev, host, scale)
