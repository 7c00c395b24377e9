"""The failure path of the pipelined kernels, made to happen on purpose.

Every wait inside the tcgen05 attention kernels, the tcgen05 backward and the
decode kernel is bounded. With the workspace's wait limit set to 1 ns the first
wait that does not succeed at once gives up: the kernel must report
DSA_ERR_DEVICE_TIMEOUT through dsa_check_status (and not fault or hang: it
drains its copies and tensor-core products with the default limit before it
frees its tensor memory). The flag clears once read, and the next call with the
default limit must be correct again (parity with the oracle), on the same
workspace and the same buffers.
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_02_b200 import Workload, binding as B
from dynamic_block_sparse_02_b200 import workloads as W
from dynamic_block_sparse_02_b200.attention import BlockSparseAttention

from parity import assert_attention_close, dev_bf16, dev_i32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    torch.cuda.set_device(0)


def oracle_lists(w, x):
    s = oracle.block_scores(oracle.pool_blocks(x["q"], w.block), oracle.pool_blocks(x["k"], w.block))
    return oracle.select_blocks(s, w.k_free, w.local_window, w.n_sink)


SHAPES = {
    # name: (B, Hq, Hkv, N, d, block, k_free, local_window, n_sink)
    "bs64-d128": (1, 8, 2, 64 * 40, 128, 64, 6, 2, 1),
    "bs128-d128": (1, 4, 1, 128 * 20, 128, 128, 4, 1, 0),
    "bs32-d64": (2, 4, 4, 32 * 50, 64, 32, 5, 1, 0),
}


@pytest.mark.parametrize("name", list(SHAPES))
def test_attention_wait_gives_up_then_recovers(name):
    Bn, Hq, Hkv, N, d, bs, k, lw, ns = SHAPES[name]
    w = Workload(name, Bn, Hq, Hkv, N, d, bs, k_free=k, local_window=lw, n_sink=ns)
    x = W.make_inputs(w, seed=81)
    idx, cnt = oracle_lists(w, x)
    o_ref, _ = oracle.sparse_attention(x["q"], x["k"], x["v"], idx, cnt, bs)
    att = BlockSparseAttention.from_workload(w, attn_kernel=B.DSA_ATTN_TCGEN05)
    q, kk, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    di, dc = dev_i32(idx), dev_i32(cnt)
    out = att.empty_out()
    att.set_wait_limit(1)
    att.sparse_attn(q, kk, v, di, dc, out)
    assert att.check_status() == B.DSA_ERR_DEVICE_TIMEOUT
    assert att.check_status() == B.DSA_OK  # read once, then cleared
    att.set_wait_limit(0)
    out.zero_()
    att.sparse_attn(q, kk, v, di, dc, out)
    assert att.check_status() == B.DSA_OK
    assert_attention_close(out.double().cpu().numpy(), o_ref, name + " after the timeout")


def test_backward_wait_gives_up_then_recovers():
    w = Workload("bwd", 1, 8, 2, 64 * 24, 128, 64, k_free=4, local_window=2, n_sink=1)
    x = W.make_inputs(w, seed=82)
    do_bits = W.f32_to_bf16_bits(np.random.default_rng(83).standard_normal(x["q"].shape).astype(np.float32))
    idx, cnt = oracle_lists(w, x)
    att = BlockSparseAttention.from_workload(w, attn_kernel=B.DSA_ATTN_TCGEN05)
    q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    di, dc = dev_i32(idx), dev_i32(cnt)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    att.sparse_attn(q, k, v, di, dc, out, lse)
    assert att.check_status() == B.DSA_OK
    dout = dev_bf16(do_bits)
    att.set_wait_limit(1)
    att.sparse_attn_backward(q, k, v, out, lse, dout, di, dc)
    assert att.check_status() == B.DSA_ERR_DEVICE_TIMEOUT
    att.set_wait_limit(0)
    dq, dk, dv = att.sparse_attn_backward(q, k, v, out, lse, dout, di, dc)
    assert att.check_status() == B.DSA_OK
    refs = oracle.sparse_attention_backward(x["q"], x["k"], x["v"], do_bits, idx, cnt, w.block)
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        gn = g.double().cpu().numpy()
        rel = np.linalg.norm(gn - r) / np.linalg.norm(r)
        assert rel <= 1e-2 and np.abs(gn - r).max() <= 2e-2 * np.abs(r).max(), (name, rel)


def test_decode_wait_gives_up_then_recovers():
    w = Workload("dec", 1, 8, 2, 64 * 40, 128, 64, k_free=6, local_window=1, n_sink=1)
    x = W.make_inputs(w, seed=84)
    L = w.N - 17
    att = BlockSparseAttention.from_workload(w)
    k, v = dev_bf16(x["k"]), dev_bf16(x["v"])
    kp = att.pooled_key_cache()
    att.pool_keys(k, kp, 0, (L - 1) // w.block)
    qtok = np.ascontiguousarray(x["q"][:, :, L - 1, :])
    q = dev_bf16(qtok)
    att.set_wait_limit(1)
    att.decode(q, k, v, kp, L)
    assert att.check_status() == B.DSA_ERR_DEVICE_TIMEOUT
    att.set_wait_limit(0)
    out = att.decode(q, k, v, kp, L)
    assert att.check_status() == B.DSA_OK
    _, _, o_ref, _ = oracle.decode(qtok, x["k"], x["v"], L, w.block, w.k_free, w.local_window, w.n_sink)
    rel = np.linalg.norm(out.double().cpu().numpy() - o_ref) / np.linalg.norm(o_ref)
    assert rel <= 5e-3, rel
