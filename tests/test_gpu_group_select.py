"""GPU parity of the group-shared selection rule (one kept list per KV head,
chosen from the sum of its query heads' block scores) against the fp64 oracle,
through the C ABI: the fused call, the split calls (bit for bit equal to the
fused one), and attention over the group lists.
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_02_b200 import WORKLOADS, Workload, binding as B
from dynamic_block_sparse_02_b200 import workloads as W
from dynamic_block_sparse_02_b200.attention import BlockSparseAttention

from parity import assert_attention_close, compare_selection, dev_bf16, dev_i32

pytestmark = pytest.mark.gpu

GROUP = B.DSA_SELECT_GROUP_TOPK


@pytest.fixture(scope="module", autouse=True)
def need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    torch.cuda.set_device(0)


# name: (B, Hq, Hkv, N, d, block, k_free, local_window, n_sink)
CASES = {
    "g4-d128-bs64-ragged": (2, 8, 2, 64 * 37, 128, 64, 5, 2, 1),
    "g8-d64-bs64": (1, 8, 1, 64 * 33, 64, 64, 3, 3, 0),
    "g1-d64-bs32": (2, 4, 4, 32 * 45, 64, 32, 4, 1, 0),
    "g2-d128-bs128": (1, 4, 2, 128 * 21, 128, 128, 4, 1, 1),
    "g4-nb-1024": (1, 4, 1, 32 * 1024, 64, 32, 7, 1, 1),
}


def group_reference(w, x):
    qp = oracle.pool_blocks(x["q"], w.block)
    kp = oracle.pool_blocks(x["k"], w.block)
    s = oracle.block_scores(qp, kp)
    idx, cnt = oracle.select_blocks_group(s, w.group, w.k_free, w.local_window, w.n_sink)
    gs = np.repeat(oracle.group_scores(s, w.group), w.group, axis=1)  # per head, for the tie rule
    return gs, idx, cnt


@pytest.mark.parametrize("name", list(CASES))
def test_group_selection_fused_split_and_attention(name):
    Bn, Hq, Hkv, N, d, bs, k, lw, ns = CASES[name]
    w = Workload(name, Bn, Hq, Hkv, N, d, bs, k_free=k, local_window=lw, n_sink=ns)
    x = W.make_inputs(w, seed=21)
    gs, idx_ref, cnt_ref = group_reference(w, x)
    q, kk, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    att = BlockSparseAttention.from_workload(w, select_mode=GROUP)
    idx, cnt = att.select_blocks(q, kk)
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    # every head of a group got the same list
    for u in range(Hkv):
        for h in range(u * w.group + 1, (u + 1) * w.group):
            np.testing.assert_array_equal(idx_h[:, h], idx_h[:, u * w.group])
            np.testing.assert_array_equal(cnt_h[:, h], cnt_h[:, u * w.group])
    n, ties, bad = compare_selection(idx_h, cnt_h, idx_ref, cnt_ref, gs, [k] * Hq, lw, ns)
    assert not bad, bad[:5]
    # split path: per-head scores, then the group selection from them
    sc = att.block_scores(q, kk)
    idx_s, cnt_s = att.topk_select(sc)
    np.testing.assert_array_equal(idx_s.cpu().numpy(), idx_h)
    np.testing.assert_array_equal(cnt_s.cpu().numpy(), cnt_h)
    # attention over the oracle's group lists, and the fused forward on rows that agree
    o_ref, _ = oracle.sparse_attention(x["q"], x["k"], x["v"], idx_ref, cnt_ref, w.block)
    out = att.sparse_attn(q, kk, v, dev_i32(idx_ref), dev_i32(cnt_ref))
    assert att.check_status() == B.DSA_OK
    assert_attention_close(out.double().cpu().numpy(), o_ref, name)
    idx_f, cnt_f = att.empty_selection()
    out_f = att.forward(q, kk, v, None, None, idx_f, cnt_f)
    np.testing.assert_array_equal(idx_f.cpu().numpy(), idx_h)
    same = (idx_h == idx_ref).all(axis=-1)
    rows = np.repeat(same, w.block, axis=-1)
    assert_attention_close(out_f.double().cpu().numpy()[rows], o_ref[rows], name + " fused")
    assert att.check_status() == B.DSA_OK


def test_group_selection_full_32k():
    w = WORKLOADS["32k-gqa"]
    x = W.make_inputs(w, seed=3)
    gs, idx_ref, cnt_ref = group_reference(w, x)
    att = BlockSparseAttention.from_workload(w, select_mode=GROUP)
    idx, cnt = att.select_blocks(dev_bf16(x["q"]), dev_bf16(x["k"]))
    n, ties, bad = compare_selection(idx.cpu().numpy(), cnt.cpu().numpy(), idx_ref, cnt_ref, gs,
                                     [w.k_free] * w.Hq, w.local_window, w.n_sink)
    assert not bad, bad[:5]
    assert att.check_status() == B.DSA_OK
