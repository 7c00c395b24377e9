"""dsa_select_blocks_static: the selection with its scratch in the library's
static device array instead of a caller workspace.

The host tests check the size limit and the argument checks without a GPU.
The GPU tests compare the static-scratch call with dsa_select_blocks (the
workspace call) on two calls in a row, with different inputs and shapes, so
that a result left behind by the previous call would show. Both calls run the
same pooling and selection kernels, so the selections must match exactly.
This file is collected last so that it also runs after the other GPU tests.
"""
import pytest
import torch

from dynamic_block_sparse_02_b200 import WORKLOADS, Workload, binding as B
from dynamic_block_sparse_02_b200 import workloads as W
from dynamic_block_sparse_02_b200.attention import BlockSparseAttention

from parity import dev_bf16

FAKE = 0x10000  # an aligned non-null address; never dereferenced by the host tests
STATIC_SCRATCH_BYTES = 16 << 20


def pooled_bytes(Bn, Hq, Hkv, N, d, block):
    nb = N // block
    up = lambda x: (x + 255) // 256 * 256
    return up(Bn * Hq * nb * d * 4) + up(Bn * Hkv * nb * d * 4)


def call_static(p, q=FAKE, k=FAKE, idx=FAKE, cnt=FAKE):
    return B.raw("dsa_select_blocks_static")(p.ref, q, k, idx, cnt, None)


def test_static_select_rejects_problems_beyond_its_scratch():
    # 32 query + 8 KV heads at N=32768, block 64, d=128: 10 MiB, fits
    assert pooled_bytes(1, 32, 8, 32768, 128, 64) == 10 << 20
    # twice the batch: 20 MiB, rejected before any device call
    big = B.Params(B=2, Hq=32, Hkv=8, N=32768, d=128, block=64, k_free=8)
    assert call_static(big) == B.DSA_ERR_WORKSPACE
    # 24 + 8 heads of 1024 blocks x 128 floats fill the 16 MiB exactly; 27 + 9 do not fit
    assert pooled_bytes(1, 24, 8, 65536, 128, 64) == STATIC_SCRATCH_BYTES
    assert pooled_bytes(1, 27, 9, 65536, 128, 64) > STATIC_SCRATCH_BYTES
    assert call_static(B.Params(B=1, Hq=27, Hkv=9, N=65536, d=128, block=64, k_free=8)) \
        == B.DSA_ERR_WORKSPACE
    # argument errors come before the size check
    assert call_static(B.Params(B=1, Hq=27, Hkv=8, N=65536, d=128, block=64)) \
        == B.DSA_ERR_INVALID_ARG


def test_static_select_argument_checks():
    p = B.Params(B=1, Hq=4, Hkv=2, N=1024, d=128, block=64, k_free=2)
    assert call_static(p, q=None) == B.DSA_ERR_INVALID_ARG
    assert call_static(p, k=FAKE + 2) == B.DSA_ERR_INVALID_ARG
    assert call_static(p, cnt=None) == B.DSA_ERR_INVALID_ARG
    assert call_static(B.Params(B=1, Hq=4, Hkv=2, N=1000, d=128, block=64)) == B.DSA_ERR_UNSUPPORTED
    for change in (dict(B=0), dict(N=0)):
        e = B.Params(**(dict(B=1, Hq=4, Hkv=2, N=1024, d=128, block=64) | change))
        assert call_static(e, q=None, k=None, idx=None, cnt=None) == B.DSA_OK


CASES = [
    # (B, Hq, Hkv, N, d, block, k_free, local_window, n_sink, k_per_head)
    (2, 8, 2, 64 * 37, 128, 64, 5, 2, 1, None),
    (2, 4, 4, 32 * 45, 64, 32, 0, 1, 0, [1, 2, 4, 8]),
    (1, 4, 1, 128 * 21, 128, 128, 4, 1, 0, None),
]


def run_twice(w, kph, seeds):
    """The workspace call on each input, then the static call on each input,
    back to back on one stream; returns both selections per input."""
    att = BlockSparseAttention.from_workload(w, k_per_head=kph)
    inputs = []
    for seed in seeds:
        x = W.make_inputs(w, seed=seed)
        inputs.append((dev_bf16(x["q"]), dev_bf16(x["k"])))
    ref = [att.select_blocks(q, k) for q, k in inputs]
    got = []
    for q, k in inputs:
        idx, cnt = att.empty_selection()
        idx.fill_(-7)
        cnt.fill_(-7)
        B.dsa_select_blocks_static(att.params, q, k, idx, cnt)
        got.append((idx, cnt))
    torch.cuda.synchronize()
    assert att.check_status() == B.DSA_OK
    return ref, got


def assert_same(ref, got, tag):
    for n, ((i_ws, c_ws), (i_st, c_st)) in enumerate(zip(ref, got)):
        assert torch.equal(c_st, c_ws), (tag, n)
        assert torch.equal(i_st, i_ws), (tag, n)


@pytest.mark.gpu
def test_static_select_matches_workspace_call_twice_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    torch.cuda.set_device(0)
    for ci, (Bn, Hq, Hkv, N, d, bs, kf, lw, ns, kph) in enumerate(CASES):
        w = Workload(f"static-{ci}", Bn, Hq, Hkv, N, d, bs, k_free=kf, local_window=lw, n_sink=ns)
        ref, got = run_twice(w, kph, (11, 12))
        assert_same(ref, got, ci)


@pytest.mark.gpu
def test_static_select_full_size_32k():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    torch.cuda.set_device(0)
    w = WORKLOADS["32k-gqa"]
    assert pooled_bytes(w.B, w.Hq, w.Hkv, w.N, w.d, w.block) <= STATIC_SCRATCH_BYTES
    ref, got = run_twice(w, None, (0, 1))
    assert_same(ref, got, w.name)
