"""GPU parity: every step of the CUDA path against the fp64 oracle, through the C ABI.

Small cases span several tiles and ragged tails (nb not a multiple of the
32-lane selection warp, odd block counts, per-head budgets, empty rows). The
full-size workloads are checked in tests/test_gpu_fullsize.py.
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_02_b200 import WORKLOADS, Workload, binding as B
from dynamic_block_sparse_02_b200 import workloads as W
from dynamic_block_sparse_02_b200.attention import BlockSparseAttention

from parity import (assert_attention_close, assert_lse_close, compare_selection, dev_bf16,
                    dev_i32)

pytestmark = pytest.mark.gpu

KERNELS = [B.DSA_ATTN_AUTO, B.DSA_ATTN_MMA_SYNC]


@pytest.fixture(scope="module", autouse=True)
def need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    torch.cuda.set_device(0)


# name: (B, Hq, Hkv, N, d, block, k_free, local_window, n_sink, k_per_head)
SMALL = {
    "tiny-mha": (1, 2, 2, 512, 64, 64, 3, 1, 0, None),
    "gqa-d128-bs64-ragged": (2, 8, 2, 64 * 37, 128, 64, 5, 2, 1, None),
    "gqa-d128-bs128": (1, 4, 1, 128 * 21, 128, 128, 4, 1, 0, None),
    "mha-d64-bs32-perhead": (2, 4, 4, 32 * 45, 64, 32, 0, 1, 0, [1, 2, 4, 8]),
    "d64-bs128": (1, 2, 1, 128 * 9, 64, 128, 2, 1, 1, None),
    "d128-bs32": (1, 4, 2, 32 * 70, 128, 32, 6, 1, 2, None),
    "d64-bs64-g8": (1, 8, 1, 64 * 33, 64, 64, 3, 3, 0, None),
    "dense": (1, 2, 1, 64 * 12, 128, 64, 1000, 1, 0, None),
    "empty-rows": (1, 2, 2, 64 * 5, 64, 64, 0, 0, 0, None),
    "window-only": (1, 2, 1, 64 * 10, 128, 64, 0, 3, 0, None),
    "sinks-no-window": (1, 2, 2, 32 * 40, 64, 32, 3, 0, 4, None),
    "nb-1024": (1, 1, 1, 32 * 1024, 64, 32, 7, 1, 1, None),
}


def spec_workload(name):
    Bn, Hq, Hkv, N, d, bs, k, w, ns, kph = SMALL[name]
    return Workload(name, Bn, Hq, Hkv, N, d, bs, k_free=k, local_window=w, n_sink=ns), kph


def oracle_reference(w, x, kph):
    qp = oracle.pool_blocks(x["q"], w.block)
    kp = oracle.pool_blocks(x["k"], w.block)
    s = oracle.block_scores(qp, kp)
    k = kph if kph is not None else w.k_free
    idx, cnt = oracle.select_blocks(s, k, w.local_window, w.n_sink)
    return s, idx, cnt


def per_head(w, kph):
    return kph if kph is not None else [w.k_free] * w.Hq


@pytest.mark.parametrize("name", list(SMALL))
def test_small_case_all_steps(name):
    w, kph = spec_workload(name)
    x = W.make_inputs(w, seed=7)
    s64, idx_ref, cnt_ref = oracle_reference(w, x, kph)
    o_ref, lse_ref = oracle.sparse_attention(x["q"], x["k"], x["v"], idx_ref, cnt_ref, w.block)

    q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    att = BlockSparseAttention.from_workload(w, k_per_head=kph)
    # steps 1-2: block scores
    sc = att.block_scores(q, k)
    sc_h = sc.cpu().numpy().astype(np.float64)
    tri = np.tril(np.ones((w.nb, w.nb), dtype=bool))
    assert np.all(np.isneginf(sc_h[..., ~tri]))
    np.testing.assert_allclose(sc_h[..., tri], s64[..., tri], rtol=1e-5, atol=1e-6)
    # step 3 on the GPU's scores, against the oracle's selection
    idx_s, cnt_s = att.topk_select(sc)
    idx_s, cnt_s = idx_s.cpu().numpy(), cnt_s.cpu().numpy()
    n, ties, bad = compare_selection(idx_s, cnt_s, idx_ref, cnt_ref, s64, per_head(w, kph),
                                     w.local_window, w.n_sink)
    assert not bad, bad[:5]
    # fused path: identical selection to the split path, bit for bit
    idx_f, cnt_f = att.empty_selection()
    out_f, lse_f = att.empty_out(), att.empty_lse()
    att.forward(q, k, v, out_f, lse_f, idx_f, cnt_f)
    np.testing.assert_array_equal(idx_f.cpu().numpy(), idx_s)
    np.testing.assert_array_equal(cnt_f.cpu().numpy(), cnt_s)
    # step 4 on the oracle's selection, with each attention kernel
    for kern in KERNELS:
        a2 = BlockSparseAttention.from_workload(w, k_per_head=kph, attn_kernel=kern)
        out, lse = a2.empty_out(), a2.empty_lse()
        a2.sparse_attn(q, k, v, dev_i32(idx_ref), dev_i32(cnt_ref), out, lse)
        assert a2.check_status() == B.DSA_OK
        assert_attention_close(out.double().cpu().numpy(), o_ref, f"{name} kernel {kern}")
        assert_lse_close(lse.cpu().numpy().astype(np.float64), lse_ref, f"{name} kernel {kern}")
    # the fused path's output, on rows whose selection equals the oracle's
    same = (idx_s == idx_ref).all(axis=-1)
    rows = np.repeat(same, w.block, axis=-1)
    o_f = out_f.double().cpu().numpy()
    assert_attention_close(o_f[rows], o_ref[rows], f"{name} fused")
    assert att.check_status() == B.DSA_OK


def tc_supported(w):
    return w.block in (32, 64, 128) and w.d in (64, 128)


def test_auto_kernel_choice_on_the_gpu():
    # AUTO: the tcgen05 kernels for every block size
    for block, want in ((32, 1), (64, 1), (128, 1)):
        p = B.Params(1, 4, 2, block * 16, 128, block, k_free=2)
        assert B.dsa_attn_uses_tcgen05(p) == want, block
        assert B.dsa_attn_uses_tcgen05(B.Params(1, 4, 2, block * 16, 128, block, k_free=2,
                                                attn_kernel=B.DSA_ATTN_TCGEN05)) == 1


def test_explicit_tcgen05_kernel_or_unsupported():
    for name in SMALL:
        w, kph = spec_workload(name)
        x = W.make_inputs(w, seed=9)
        s64, idx_ref, cnt_ref = oracle_reference(w, x, kph)
        att = BlockSparseAttention.from_workload(w, k_per_head=kph, attn_kernel=B.DSA_ATTN_TCGEN05)
        q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
        if not tc_supported(w):
            with pytest.raises(B.DsaError) as e:
                att.sparse_attn(q, k, v, dev_i32(idx_ref), dev_i32(cnt_ref))
            assert e.value.status == B.DSA_ERR_UNSUPPORTED
            continue
        o_ref, lse_ref = oracle.sparse_attention(x["q"], x["k"], x["v"], idx_ref, cnt_ref, w.block)
        out, lse = att.empty_out(), att.empty_lse()
        att.sparse_attn(q, k, v, dev_i32(idx_ref), dev_i32(cnt_ref), out, lse)
        assert att.check_status() == B.DSA_OK
        assert_attention_close(out.double().cpu().numpy(), o_ref, name + " tcgen05")
        assert_lse_close(lse.cpu().numpy().astype(np.float64), lse_ref, name + " tcgen05")


def test_exact_score_ties_pick_lower_block_index():
    # Key blocks repeat one of three patterns, so many block scores tie exactly;
    # the selection must keep the lower block indices among equal scores.
    w = Workload("ties", 1, 4, 2, 64 * 70, 128, 64, k_free=9, local_window=1, n_sink=1)
    x = W.make_inputs(w, seed=13)
    kb = x["k"].reshape(w.B, w.Hkv, w.nb, w.block, w.d)
    pattern = np.arange(w.nb) % 3
    x["k"] = np.ascontiguousarray(kb[:, :, pattern]).reshape(w.B, w.Hkv, w.N, w.d)
    s64, idx_ref, cnt_ref = oracle_reference(w, x, None)
    att = BlockSparseAttention.from_workload(w)
    q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    idx, cnt = att.select_blocks(q, k)
    np.testing.assert_array_equal(cnt.cpu().numpy(), cnt_ref)
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref)
    sc = att.block_scores(q, k)
    idx2, cnt2 = att.topk_select(sc)
    np.testing.assert_array_equal(idx2.cpu().numpy(), idx_ref)


@pytest.mark.parametrize("kern", KERNELS)
def test_ones_value_gives_ones(kern):
    w = Workload("ones", 1, 4, 2, 64 * 20, 128, 64, k_free=3, local_window=2, n_sink=1)
    x = W.make_inputs(w, seed=3, tensors=("q", "k"))
    x["q"] = W.f32_to_bf16_bits(W.bf16_bits_to_f32(x["q"]) * 4)  # sharper softmax
    q, k = dev_bf16(x["q"]), dev_bf16(x["k"])
    v = torch.ones((w.B, w.Hkv, w.N, w.d), dtype=torch.bfloat16, device="cuda")
    att = BlockSparseAttention.from_workload(w, attn_kernel=kern)
    out = att.forward(q, k, v)
    assert torch.all(out == 1.0)
    assert att.check_status() == B.DSA_OK


@pytest.mark.parametrize("d", [64, 128])
def test_out_of_range_index_is_skipped_and_flagged(d):
    w = Workload("bad-idx", 1, 2, 2, 64 * 8, d, 64, k_free=2, local_window=1, n_sink=0)
    x = W.make_inputs(w, seed=5)
    s64, idx_ref, cnt_ref = oracle_reference(w, x, None)
    bad_idx = idx_ref.copy()
    bad_idx[0, 1, 5, 0] = 7   # a future block (j > i)
    bad_idx[0, 0, 3, 1] = -4  # negative
    q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    for kern in KERNELS:
        a2 = BlockSparseAttention.from_workload(w, attn_kernel=kern)
        out = a2.sparse_attn(q, k, v, dev_i32(bad_idx), dev_i32(cnt_ref))
        assert a2.check_status() == B.DSA_ERR_DEVICE_BOUNDS
        assert a2.check_status() == B.DSA_OK  # the flag clears once read
        # the row without the bad entry matches the oracle on the cleaned list
        clean = idx_ref.copy()
        o_ref, _ = oracle.sparse_attention(x["q"], x["k"], x["v"], clean, cnt_ref, w.block)
        o = out.double().cpu().numpy()
        assert_attention_close(o[0, 1, :5 * 64], o_ref[0, 1, :5 * 64], "untouched rows")


def cleaned_lists(idx, cnt, nb):
    """The lists the kernels use: entry t of row (b, h, i) is kept only if
    0 <= j <= i and j is greater than entry t - 1 of the row as given."""
    out = np.full_like(idx, -1)
    c = np.zeros_like(cnt)
    for (b, h, i), n in np.ndenumerate(cnt):
        row = idx[b, h, i, :n]
        keep = [int(j) for t, j in enumerate(row) if 0 <= j <= i and (t == 0 or j > row[t - 1])]
        out[b, h, i, :len(keep)] = keep
        c[b, h, i] = len(keep)
    return out, c


def disorder(idx_ref, cnt_ref):
    """A repeated entry in one row and a step down in another."""
    bad = idx_ref.copy()
    rows = [(b, h, i) for (b, h, i), n in np.ndenumerate(cnt_ref) if n >= 3]
    (b0, h0, i0), (b1, h1, i1) = rows[-1], rows[-2]
    bad[b0, h0, i0, 1] = bad[b0, h0, i0, 0]                                   # repeat
    bad[b1, h1, i1, 0], bad[b1, h1, i1, 1] = bad[b1, h1, i1, 1], bad[b1, h1, i1, 0]  # step down
    return bad


@pytest.mark.parametrize("d,block", [(128, 64), (64, 32), (128, 128)])
def test_repeated_or_descending_entries_are_skipped_and_flagged(d, block):
    w = Workload("bad-order", 1, 2, 2, block * 8, d, block, k_free=3, local_window=1, n_sink=0)
    x = W.make_inputs(w, seed=11)
    s64, idx_ref, cnt_ref = oracle_reference(w, x, None)
    bad = disorder(idx_ref, cnt_ref)
    clean, ccnt = cleaned_lists(bad, cnt_ref, w.nb)
    assert not np.array_equal(clean, idx_ref)
    o_ref, l_ref = oracle.sparse_attention(x["q"], x["k"], x["v"], clean, ccnt, w.block)
    q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    for kern in (B.DSA_ATTN_AUTO, B.DSA_ATTN_TCGEN05, B.DSA_ATTN_MMA_SYNC):
        a2 = BlockSparseAttention.from_workload(w, attn_kernel=kern)
        out, lse = a2.empty_out(), a2.empty_lse()
        a2.sparse_attn(q, k, v, dev_i32(bad), dev_i32(cnt_ref), out, lse)
        assert a2.check_status() == B.DSA_ERR_DEVICE_BOUNDS, kern
        assert a2.check_status() == B.DSA_OK
        assert_attention_close(out.double().cpu().numpy(), o_ref, f"kernel {kern}")
        assert_lse_close(lse.double().cpu().numpy(), l_ref, f"kernel {kern}")


@pytest.mark.parametrize("block,d,scale", [(64, 128, 0.5), (32, 64, 0.02), (128, 128, 0.4), (64, 64, 1.0)])
def test_custom_scale_every_kernel(block, d, scale):
    # a softmax scale other than 1/sqrt(d): sharp ones move the running maxima
    # by many powers of two from block to block (the rescale path), a small one
    # flattens the weights
    w = Workload("scale", 2, 4, 2, block * 10, d, block, k_free=3, local_window=1, n_sink=1, scale=scale)
    x = W.make_inputs(w, seed=21)
    s64, idx_ref, cnt_ref = oracle_reference(w, x, None)
    o_ref, l_ref = oracle.sparse_attention(x["q"], x["k"], x["v"], idx_ref, cnt_ref, w.block, scale=scale)
    q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    for kern in (B.DSA_ATTN_AUTO, B.DSA_ATTN_TCGEN05, B.DSA_ATTN_MMA_SYNC):
        a2 = BlockSparseAttention.from_workload(w, attn_kernel=kern)
        out, lse = a2.empty_out(), a2.empty_lse()
        a2.sparse_attn(q, k, v, dev_i32(idx_ref), dev_i32(cnt_ref), out, lse)
        assert a2.check_status() == B.DSA_OK
        assert_attention_close(out.double().cpu().numpy(), o_ref, f"kernel {kern} scale {scale}")
        assert_lse_close(lse.double().cpu().numpy(), l_ref, f"kernel {kern} scale {scale}")


@pytest.mark.parametrize("block,d", [(64, 128), (32, 64), (128, 128)])
def test_forward_is_deterministic(block, d):
    # persistent CTAs take work items from a global counter, so which CTA runs
    # which item changes from run to run; each item's sums run in a fixed
    # order, so two runs agree bit for bit
    w = Workload("det", 2, 8, 2, block * 48, d, block, k_free=9, local_window=2, n_sink=1)
    x = W.make_inputs(w, seed=31)
    q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    for kern in (B.DSA_ATTN_AUTO, B.DSA_ATTN_MMA_SYNC):
        att = BlockSparseAttention.from_workload(w, attn_kernel=kern)
        runs = []
        for _ in range(2):
            idx, cnt = att.empty_selection()
            out, lse = att.empty_out(), att.empty_lse()
            att.forward(q, k, v, out, lse, idx, cnt)
            torch.cuda.synchronize()
            runs.append((out, lse, idx, cnt))
        assert att.check_status() == B.DSA_OK
        for ta, tb in zip(*runs):
            assert torch.equal(ta, tb), kern


def test_cuda_graph_capture_replays_forward():
    w = WORKLOADS["tiny"]
    x = W.make_inputs(w)
    q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    att = BlockSparseAttention.from_workload(w)
    ref = att.forward(q, k, v).clone()
    out = att.empty_out()
    s = torch.cuda.Stream()
    att.stream = s
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        att.forward(q, k, v, out)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
