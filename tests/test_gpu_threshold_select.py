"""GPU parity of the threshold selection rule (forced blocks plus the blocks
whose share of the softmax over the row's block logits is >= tau, at most k)
against the fp64 oracle, through the C ABI.

A block may fall on the other side of tau on the GPU only when its oracle
probability p_j is within delta_j * tau of tau, delta_j being the bound on the
relative error of the GPU's fp32 probability (the same bound include/dsa.h
states for DSA_SELECT_THRESHOLD):
  eps_j   = (bs + d) * 2^-24 * sum_d mean|q_d| * mean|k_jd|   fp32 error of s(i, j)
            (block means of bs terms, then a d-term dot product; mean|.| over
            the block's rows)
  eta_j   = c2 * (eps_j + max eps) + 2^-23 * c2 * |s_j - max s|   exponent error
  delta_j = ln2 * (eta_j + max eta) + (i + 5) * 2^-24 + 2^-21
with c2 = scale * log2(e); the ln2 terms are the errors of 2^x from errors in x
(for the block and for the normaliser's largest term), (i + 5) 2^-24 the fp32
sum of i + 1 terms and the products, 2^-21 the exp2 approximation. The usual
near-tie rule applies at the k-th score.
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_02_b200 import WORKLOADS, Workload, binding as B
from dynamic_block_sparse_02_b200 import workloads as W
from dynamic_block_sparse_02_b200.attention import BlockSparseAttention

from parity import TIE_REL, assert_attention_close, dev_bf16, dev_i32

pytestmark = pytest.mark.gpu

THR = B.DSA_SELECT_THRESHOLD
U32 = 2.0 ** -24


def block_abs_means(bits, block):
    """mean over each block's rows of |x| (fp64) [B, H, nb, d]."""
    x = np.abs(W.bf16_bits_to_f32(bits).astype(np.float64))
    Bn, H, N, d = x.shape
    return x.reshape(Bn, H, N // block, block, d).mean(axis=3)


def prob_error_bound(aq, ak, s_row, i, block, d, c2):
    """delta_j of the module docstring for every causal block j of one row."""
    eps = (block + d) * U32 * (ak[:i + 1] @ aq)
    m = np.max(s_row[:i + 1])
    eta = c2 * (eps + eps.max()) + 2 * U32 * c2 * np.abs(s_row[:i + 1] - m)
    return np.log(2.0) * (eta + eta.max()) + (i + 5) * U32 + 2.0 ** -21


@pytest.fixture(scope="module", autouse=True)
def need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    torch.cuda.set_device(0)


def compare_threshold(idx_g, cnt_g, idx_r, cnt_r, s64, tau, k, w, ns, scale, aq, ak, block, d):
    """Unexcused row mismatches: every block in the symmetric difference must
    sit at the threshold (|p_j - tau| <= delta_j * tau) or tie with the k-th
    candidate's score (TIE_REL)."""
    B_, Hq, nb, _ = idx_r.shape
    g = Hq // ak.shape[1]
    c2 = scale * np.log2(np.e)
    bad = []
    for b in range(B_):
        for h in range(Hq):
            for i in range(nb):
                g = idx_g[b, h, i, :cnt_g[b, h, i]].tolist()
                r = idx_r[b, h, i, :cnt_r[b, h, i]].tolist()
                if not np.all(idx_g[b, h, i, cnt_g[b, h, i]:] == -1) or g != sorted(set(g)):
                    bad.append((b, h, i, "layout"))
                    continue
                if g == r:
                    continue
                p = oracle.block_probabilities(s64[b, h, i], i, scale)
                forced = oracle.forced_set(i, w, ns)
                cand = [j for j in range(i + 1) if j not in forced]
                srt = sorted(cand, key=lambda j: (-float(np.float32(s64[b, h, i, j])), j))
                kth = s64[b, h, i, srt[min(k, len(srt)) - 1]] if srt and k > 0 else None
                delta = prob_error_bound(aq[b, h, i], ak[b, h // g], s64[b, h, i], i, block, d, c2)
                for j in set(g) ^ set(r):
                    at_bar = abs(p[j] - tau) <= delta[j] * tau
                    at_cut = kth is not None and abs(s64[b, h, i, j] - kth) <= TIE_REL * max(
                        abs(s64[b, h, i, j]), abs(kth))
                    if j in forced or not (at_bar or at_cut):
                        bad.append((b, h, i, j, float(p[j])))
    return bad


CASES = {
    # name: (B, Hq, Hkv, N, d, block, k_free, local_window, n_sink, tau)
    "d128-bs64-tau0.02": (2, 8, 2, 64 * 37, 128, 64, 8, 2, 1, 0.02),
    "d64-bs32-tau0.005": (1, 4, 4, 32 * 90, 64, 32, 16, 1, 0, 0.005),
    "d128-bs128-tau0.05": (1, 4, 1, 128 * 21, 128, 128, 6, 1, 1, 0.05),
    "d64-bs64-tau-large": (1, 4, 2, 64 * 40, 64, 64, 30, 1, 1, 0.2),
}


@pytest.mark.parametrize("name", list(CASES))
def test_threshold_selection_parity(name):
    Bn, Hq, Hkv, N, d, bs, k, lw, ns, tau = CASES[name]
    w = Workload(name, Bn, Hq, Hkv, N, d, bs, k_free=k, local_window=lw, n_sink=ns)
    x = W.make_inputs(w, seed=31)
    # sharper block logits than N(0,1) inputs give, so the threshold bites
    x["q"] = W.f32_to_bf16_bits(W.bf16_bits_to_f32(x["q"]) * 64.0)
    scale = 1.0 / np.sqrt(d)
    s64 = oracle.block_scores(oracle.pool_blocks(x["q"], bs), oracle.pool_blocks(x["k"], bs))
    idx_r, cnt_r = oracle.select_blocks_threshold(s64, tau, k, lw, ns, scale)
    att = BlockSparseAttention.from_workload(w, select_mode=THR, select_tau=tau)
    q, kk, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    idx, cnt = att.select_blocks(q, kk)
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    aq, ak = block_abs_means(x["q"], bs), block_abs_means(x["k"], bs)
    bad = compare_threshold(idx_h, cnt_h, idx_r, cnt_r, s64, tau, k, lw, ns, scale, aq, ak, bs, d)
    assert not bad, bad[:5]
    # the rule is doing something: some rows keep fewer than k free blocks
    full = np.array([min(i + 1, k + len(oracle.forced_set(i, lw, ns))) for i in range(w.nb)])
    assert np.any(cnt_r < full[None, None, :])
    # split path equals the fused one bit for bit
    idx_s, cnt_s = att.topk_select(att.block_scores(q, kk))
    np.testing.assert_array_equal(idx_s.cpu().numpy(), idx_h)
    np.testing.assert_array_equal(cnt_s.cpu().numpy(), cnt_h)
    # attention over the variable-length lists
    o_ref, _ = oracle.sparse_attention(x["q"], x["k"], x["v"], idx_r, cnt_r, bs)
    out = att.sparse_attn(q, kk, v, dev_i32(idx_r), dev_i32(cnt_r))
    assert att.check_status() == B.DSA_OK
    assert_attention_close(out.double().cpu().numpy(), o_ref, name)
