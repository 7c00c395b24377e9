"""Pins for the fp64 oracle against facts independent of it.

Each test checks the oracle against something other than itself: closed forms
built by hand, brute-force enumeration, the counts the pages print, or a
textbook routine (PyTorch's scaled_dot_product_attention in fp64 on the CPU).
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from dynamic_block_sparse_02_b200 import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore")


def bits(x):
    """Exact bf16 bit patterns of values that bf16 represents exactly."""
    x32 = np.asarray(x, dtype=np.float32)
    u = x32.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "test value not exactly representable in bf16"
    return (u >> 16).astype(np.uint16)


def rand_bits(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return W.f32_to_bf16_bits((g.standard_normal(shape) * scale).astype(np.float32))


def f64(b):
    return torch.from_numpy(oracle.bf16_to_f64(b))


# ---------------------------------------------------------------------------
# Pooling
# ---------------------------------------------------------------------------

def test_pool_arithmetic_progression_closed_form():
    # x[r, c] = +r for even c, -r for odd c; the mean of rows i*bs .. i*bs+bs-1
    # is i*bs + (bs-1)/2 (with the sign of the column).
    N, d, bs = 256, 4, 32
    r = np.arange(N, dtype=np.float32)[:, None]
    sign = np.where(np.arange(d) % 2 == 0, 1.0, -1.0).astype(np.float32)[None, :]
    x = bits((r * sign)[None, None])
    p = oracle.pool_blocks(x, bs)
    expect = (np.arange(N // bs) * bs + (bs - 1) / 2.0)[:, None] * sign
    assert p.shape == (1, 1, N // bs, d)
    np.testing.assert_array_equal(p[0, 0], expect)


def test_pool_column_sums_and_within_block_permutation():
    x = rand_bits((2, 3, 256, 16), seed=1)
    p = oracle.pool_blocks(x, 64)
    col = oracle.bf16_to_f64(x).sum(axis=2)
    np.testing.assert_allclose(p.sum(axis=2) * 64, col, rtol=0, atol=1e-10)
    perm = np.concatenate([np.random.default_rng(2).permutation(64) + 64 * i for i in range(4)])
    np.testing.assert_allclose(oracle.pool_blocks(x[:, :, perm], 64), p, rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------
# Scores
# ---------------------------------------------------------------------------

def test_scores_closed_form_and_causal_mask():
    # Q block i rows = (i+1) e0, K block j rows = (j+2) e0 + e1 (e1 has no Q
    # partner): s(i, j) = (i+1)(j+2) for j <= i, -inf above. A transposed
    # operand would give (j+1)(i+2).
    nb, bs, d = 5, 4, 3
    q = np.zeros((1, 1, nb * bs, d), np.float32)
    k = np.zeros((1, 1, nb * bs, d), np.float32)
    for i in range(nb):
        q[0, 0, i * bs:(i + 1) * bs, 0] = i + 1
        k[0, 0, i * bs:(i + 1) * bs, 0] = i + 2
        k[0, 0, i * bs:(i + 1) * bs, 1] = 1
    s = oracle.block_scores(oracle.pool_blocks(bits(q), bs), oracle.pool_blocks(bits(k), bs))
    for i in range(nb):
        for j in range(nb):
            if j <= i:
                assert s[0, 0, i, j] == (i + 1) * (j + 2)
            else:
                assert s[0, 0, i, j] == -np.inf


def test_scores_gqa_head_mapping():
    # 6 query heads over 2 KV heads: query head h reads KV head h // 3.
    Hq, Hkv, nb, bs, d = 6, 2, 3, 2, 2
    q = np.zeros((1, Hq, nb * bs, d), np.float32)
    q[..., 0] = 1
    k = np.zeros((1, Hkv, nb * bs, d), np.float32)
    for g in range(Hkv):
        k[0, g, :, 0] = 10 * (g + 1)
    s = oracle.block_scores(oracle.pool_blocks(bits(q), bs), oracle.pool_blocks(bits(k), bs))
    for h in range(Hq):
        assert s[0, h, 2, 0] == 10 * (h // 3 + 1)


# ---------------------------------------------------------------------------
# Selection
# ---------------------------------------------------------------------------

def brute_force_select(s32_row, i, k, w, ns):
    """Best set by enumeration: the forced set plus the size-min(k,|C|) subset
    of the free blocks with the largest exact score sum, ties to the
    lexicographically smallest sorted index tuple."""
    forced = set(range(max(0, i - w + 1), i + 1)) if w > 0 else set()
    forced |= set(range(min(ns, i + 1)))
    free = [j for j in range(i + 1) if j not in forced]
    take = min(k, len(free))
    best = None
    for combo in itertools.combinations(free, take):
        total = sum((Fraction(float(s32_row[j])) for j in combo), Fraction(0))
        key = (-total, combo)
        if best is None or key < best[0]:
            best = (key, combo)
    return sorted(forced | set(best[1]))


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("k,w,ns", [(0, 1, 0), (1, 1, 0), (2, 1, 1), (3, 2, 1), (4, 0, 0),
                                    (3, 0, 2), (8, 1, 0)])
def test_select_matches_brute_force(seed, k, w, ns):
    nb = 8
    g = np.random.default_rng(seed)
    if seed % 2:
        scores = g.integers(-2, 3, size=(1, 2, nb, nb)).astype(np.float64)  # many exact ties
    else:
        scores = g.standard_normal((1, 2, nb, nb))
    scores[..., np.triu_indices(nb, 1)[0], np.triu_indices(nb, 1)[1]] = -np.inf
    idx, cnt = oracle.select_blocks(scores, k, w, ns)
    s32 = scores.astype(np.float32)
    for h in range(2):
        for i in range(nb):
            expect = brute_force_select(s32[0, h, i], i, k, w, ns)
            got = list(idx[0, h, i, :cnt[0, h, i]])
            assert got == expect, (h, i, got, expect)
            assert np.all(idx[0, h, i, cnt[0, h, i]:] == -1)


def test_select_ties_go_to_lower_index():
    nb = 6
    scores = np.zeros((1, 1, nb, nb))
    scores[..., np.triu_indices(nb, 1)[0], np.triu_indices(nb, 1)[1]] = -np.inf
    idx, cnt = oracle.select_blocks(scores, 2, 1, 0)
    assert list(idx[0, 0, 5, :cnt[0, 0, 5]]) == [0, 1, 5]
    # scores equal only after fp32 rounding still tie
    scores[0, 0, 5, :5] = [1.0, 1.0 + 1e-12, 1.0, 0.5, 1.0 + 2e-12]
    idx, cnt = oracle.select_blocks(scores, 2, 1, 0)
    assert list(idx[0, 0, 5, :cnt[0, 0, 5]]) == [0, 1, 5]


def forced_count(i, w, ns):
    """|F(i)| in closed form: the window's size plus the sinks left of it."""
    return min(w, i + 1) + min(ns, max(0, i - w + 1))


def kept_total(nb, k, w, ns):
    return sum(min(i + 1, forced_count(i, w, ns) + k) for i in range(nb))


def test_kept_block_totals_closed_form():
    # Kept-block totals per head, from the selection rule and each workload's
    # settings: C1 26, C2 2151, C3 32093, C4 64480, C5 4572/8568/16368/31200.
    wl = W.WORKLOADS
    assert kept_total(8, 3, 1, 0) == 26
    assert kept_total(wl["8k-gqa"].nb, 16, 1, 1) == 2151
    assert kept_total(wl["32k-gqa"].nb, 64, 2, 1) == 32093
    assert kept_total(wl["128k-structured"].nb, 64, 1, 0) == 64480
    assert [kept_total(512, k, 1, 0) for k in (8, 16, 32, 64)] == [4572, 8568, 16368, 31200]


@pytest.mark.parametrize("nb,k,w,ns", [(8, 3, 1, 0), (128, 16, 1, 1), (512, 64, 2, 1),
                                       (37, 5, 3, 2), (20, 0, 0, 3)])
def test_oracle_counts_match_closed_form(nb, k, w, ns):
    g = np.random.default_rng(nb)
    scores = g.standard_normal((1, 1, nb, nb))
    scores[..., np.triu_indices(nb, 1)[0], np.triu_indices(nb, 1)[1]] = -np.inf
    idx, cnt = oracle.select_blocks(scores, k, w, ns)
    for i in range(nb):
        assert cnt[0, 0, i] == min(i + 1, forced_count(i, w, ns) + k)
    assert int(cnt.sum()) == kept_total(nb, k, w, ns)


def test_select_invariant_under_positive_scaling_of_q():
    q = rand_bits((1, 2, 1024, 32), 5)
    k = rand_bits((1, 2, 1024, 32), 6)
    s = oracle.block_scores(oracle.pool_blocks(q, 32), oracle.pool_blocks(k, 32))
    idx, cnt = oracle.select_blocks(s, 4, 1, 1)
    q2 = W.f32_to_bf16_bits(W.bf16_bits_to_f32(q) * np.float32(4.0))  # exact x4
    s2 = oracle.block_scores(oracle.pool_blocks(q2, 32), oracle.pool_blocks(k, 32))
    idx2, cnt2 = oracle.select_blocks(s2, 4, 1, 1)
    np.testing.assert_array_equal(idx, idx2)
    np.testing.assert_array_equal(cnt, cnt2)


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def sdpa(q_bits, k_bits, v_bits, mask=None, causal=False, scale=None):
    q, k, v = f64(q_bits), f64(k_bits), f64(v_bits)
    g = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(g, dim=1)
    v = v.repeat_interleave(g, dim=1)
    return F.scaled_dot_product_attention(q, k, v, attn_mask=mask, is_causal=causal,
                                          scale=scale).numpy()


def mask_from_selection(idx, cnt, N, bs):
    """Boolean [B,H,N,N] mask: key t visible to row r iff block(t) is kept for block(r) and t <= r."""
    B, H, nb, _ = idx.shape
    m = np.zeros((B, H, N, N), dtype=bool)
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                for j in idx[b, h, i, :cnt[b, h, i]]:
                    m[b, h, i * bs:(i + 1) * bs, j * bs:(j + 1) * bs] = True
    m &= np.tril(np.ones((N, N), dtype=bool))[None, None]
    return torch.from_numpy(m)


def test_dense_case_equals_causal_sdpa():
    B, Hq, Hkv, N, d, bs = 2, 4, 2, 256, 32, 32
    q, k, v = rand_bits((B, Hq, N, d), 10), rand_bits((B, Hkv, N, d), 11), rand_bits((B, Hkv, N, d), 12)
    idx, cnt, (o, lse) = oracle.forward(q, k, v, bs, k_free=N // bs, local_window=1, n_sink=0)
    assert np.all(cnt[..., -1] == N // bs)
    ref = sdpa(q, k, v, causal=True)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    # log-sum-exp against torch.logsumexp of the causally masked logits
    kk = f64(k).repeat_interleave(Hq // Hkv, dim=1)
    logits = (f64(q) @ kk.transpose(-1, -2)) / math.sqrt(d)
    logits = logits.masked_fill(~torch.tril(torch.ones(N, N, dtype=torch.bool)), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(logits, dim=-1).numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("bs,k,w,ns,g", [(16, 2, 1, 0, 1), (32, 3, 2, 1, 2), (16, 1, 0, 1, 4),
                                         (64, 1, 1, 0, 1)])
def test_sparse_equals_sdpa_with_block_mask(bs, k, w, ns, g):
    B, Hkv, N, d = 1, 2, 256, 16
    Hq = Hkv * g
    q, kk, v = rand_bits((B, Hq, N, d), 20 + bs), rand_bits((B, Hkv, N, d), 21), rand_bits((B, Hkv, N, d), 22)
    idx, cnt, (o, lse) = oracle.forward(q, kk, v, bs, k, w, ns)
    mask = mask_from_selection(idx, cnt, N, bs)
    ref = sdpa(q, kk, v, mask=mask)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_block_diagonal_local_attention():
    # window 1, no sinks, k = 0: each 32-token block attends causally to itself only.
    B, H, N, d, bs = 1, 2, 128, 8, 32
    q, k, v = rand_bits((B, H, N, d), 30), rand_bits((B, H, N, d), 31), rand_bits((B, H, N, d), 32)
    _, cnt, (o, _) = oracle.forward(q, k, v, bs, 0, 1, 0)
    assert np.all(cnt == 1)
    nb = N // bs
    r = lambda x: x.reshape(B, H * nb, bs, d)
    ref = sdpa(r(q), r(k), r(v), causal=True).reshape(B, H, N, d)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_weights_sum_to_one_and_ones_value_gives_ones():
    B, H, N, d, bs = 1, 2, 256, 16, 32
    q, k = rand_bits((B, H, N, d), 40, 3.0), rand_bits((B, H, N, d), 41, 3.0)
    v1 = bits(np.ones((B, H, N, d), np.float32))
    idx, cnt, (o, _) = oracle.forward(q, k, v1, bs, 2, 1, 1)
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-13)
    qf, kf = oracle.bf16_to_f64(q[0, 1]), oracle.bf16_to_f64(k[0, 1])
    for i in range(N // bs):
        keys = oracle.kept_keys(idx[0, 1, i], cnt[0, 1, i], bs)
        wts, _ = oracle.block_weights(qf[i * bs:(i + 1) * bs], kf, keys, i, bs, 0.25)
        np.testing.assert_allclose(wts.sum(axis=1), 1.0, rtol=0, atol=1e-13)
        assert np.all(wts >= 0)


def test_gqa_equals_mha_with_repeated_kv():
    B, Hq, Hkv, N, d, bs = 1, 8, 2, 256, 16, 32
    q, k, v = rand_bits((B, Hq, N, d), 50), rand_bits((B, Hkv, N, d), 51), rand_bits((B, Hkv, N, d), 52)
    idx, cnt, (o, lse) = oracle.forward(q, k, v, bs, 2, 1, 1)
    rep = lambda x: np.repeat(x, Hq // Hkv, axis=1)
    idx2, cnt2, (o2, lse2) = oracle.forward(q, rep(k), rep(v), bs, 2, 1, 1)
    np.testing.assert_array_equal(idx, idx2)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)


def test_empty_selection_gives_zero_output():
    q, k, v = rand_bits((1, 1, 128, 8), 60), rand_bits((1, 1, 128, 8), 61), rand_bits((1, 1, 128, 8), 62)
    idx, cnt, (o, lse) = oracle.forward(q, k, v, 32, 0, 0, 0)
    assert np.all(cnt == 0) and np.all(idx == -1)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_items_subset_matches_full_result():
    q, k, v = rand_bits((2, 4, 256, 16), 70), rand_bits((2, 2, 256, 16), 71), rand_bits((2, 2, 256, 16), 72)
    idx, cnt, (o, lse) = oracle.forward(q, k, v, 32, 2, 1, 1)
    items = [(1, 3, 7), (0, 0, 0), (1, 2, 4)]
    res = oracle.sparse_attention(q, k, v, idx, cnt, 32, items=items)
    for (b, h, i), (ob, lb) in res.items():
        np.testing.assert_array_equal(ob, o[b, h, i * 32:(i + 1) * 32])
        np.testing.assert_array_equal(lb, lse[b, h, i * 32:(i + 1) * 32])


def test_hand_worked_example():
    # One head, d=2, 2-token blocks, 3 blocks; window 1, no sink, one free pick.
    Q = np.array([[1, 0], [1, 0], [0, 1], [0, 1], [1, 1], [1, -1]], np.float32)
    K = np.array([[2, 0], [0, 0], [0, 2], [0, 2], [1, 1], [-1, 1]], np.float32)
    V = np.array([[1, 0], [0, 1], [5, 5], [7, 7], [1, 1], [2, -2]], np.float32)
    q, k, v = (bits(x[None, None]) for x in (Q, K, V))
    V = V.astype(np.float64)
    # pooled q: [1,0], [0,1], [1,0]; pooled k: [1,0], [0,2], [0,1]
    # scores: row0 [1]; row1 [0, 2]; row2 [1, 0, 1]
    idx, cnt, (o, lse) = oracle.forward(q, k, v, 2, 1, 1, 0)
    assert [list(idx[0, 0, i, :cnt[0, 0, i]]) for i in range(3)] == [[0], [0, 1], [0, 2]]
    c = 1 / math.sqrt(2)
    # row 5 (q=[1,-1]) sees t=0,1,4,5 with logits 2c, 0, 0, -2c
    e = [math.exp(2 * c), 1.0, 1.0, math.exp(-2 * c)]
    z = sum(e)
    vr = [V[0], V[1], V[4], V[5]]
    expect5 = sum(ei * vi for ei, vi in zip(e, vr)) / z
    np.testing.assert_allclose(o[0, 0, 5], expect5, rtol=0, atol=1e-15)
    assert abs(lse[0, 0, 5] - math.log(z)) < 1e-15
    # row 4 (q=[1,1]) sees t=0,1,4 (t=5 is in the future) with logits 2c, 0, 2c
    e4 = [math.exp(2 * c), 1.0, math.exp(2 * c)]
    expect4 = (e4[0] * V[0] + e4[1] * V[1] + e4[2] * V[4]) / sum(e4)
    np.testing.assert_allclose(o[0, 0, 4], expect4, rtol=0, atol=1e-15)
    # row 2 (q=[0,1], block 1 keeps {0,1}) sees t=0,1,2 with logits 0, 0, 2c
    e2 = [1.0, 1.0, math.exp(2 * c)]
    expect2 = (e2[0] * V[0] + e2[1] * V[1] + e2[2] * V[2]) / sum(e2)
    np.testing.assert_allclose(o[0, 0, 2], expect2, rtol=0, atol=1e-15)


# ---------------------------------------------------------------------------
# The pages' printed pair counts
# ---------------------------------------------------------------------------

def load_golden_counts():
    path = os.path.join(os.path.dirname(__file__), "golden", "pages_pair_counts.txt")
    rows = []
    for line in open(path, encoding="utf-8"):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append(line.split(None, 5))
    return rows


def test_pair_counts_printed_on_pages():
    rows = load_golden_counts()
    assert len(rows) == 3
    for r in rows:
        if r[0] == "pairs":
            n, printed, tol = int(r[1]), int(r[2]), float(r[3])
            got = oracle.dense_pairs(n)
            assert abs(got - printed) <= tol * printed, (n, got, printed)
        else:
            n, m, ratio, tol = int(r[1]), int(r[2]), int(r[3]), float(r[4])
            assert oracle.dense_pairs(m) / oracle.dense_pairs(n) == ratio


def test_attended_pairs_dense_causal():
    N, bs = 256, 32
    nb = N // bs
    idx = np.tile(np.arange(nb, dtype=np.int32), (1, 1, nb, 1))
    cnt = (np.arange(nb, dtype=np.int32) + 1)[None, None]
    for i in range(nb):
        idx[0, 0, i, i + 1:] = -1
    assert oracle.attended_pairs(idx, cnt, bs) == oracle.dense_pairs(N, causal=True)


# ---------------------------------------------------------------------------
# Group-shared selection (one list per KV head from the summed head scores)
# ---------------------------------------------------------------------------

def _causal(scores):
    nb = scores.shape[-1]
    scores[..., np.triu_indices(nb, 1)[0], np.triu_indices(nb, 1)[1]] = -np.inf
    return scores


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("group,k,w,ns", [(2, 2, 1, 0), (3, 3, 2, 1), (4, 1, 1, 1), (2, 0, 1, 0)])
def test_group_select_matches_brute_force(seed, group, k, w, ns):
    """Brute force on the exact (Fraction) sum of the heads' fp32-representable
    scores; with integer scores the sum is exact in every precision."""
    nb, kvh = 7, 2
    g = np.random.default_rng(100 + seed)
    if seed % 2:
        scores = g.integers(-2, 3, size=(1, kvh * group, nb, nb)).astype(np.float64)
    else:
        scores = np.round(g.standard_normal((1, kvh * group, nb, nb)) * 64) / 64  # exact in fp32
    _causal(scores)
    idx, cnt = oracle.select_blocks_group(scores, group, k, w, ns)
    for u in range(kvh):
        for i in range(nb):
            heads = range(u * group, (u + 1) * group)
            summed = [float(sum(Fraction(float(scores[0, h, i, j])) for h in heads)) if j <= i else -np.inf
                      for j in range(nb)]
            expect = brute_force_select(np.array(summed), i, k, w, ns)
            for h in heads:
                got = list(idx[0, h, i, :cnt[0, h, i]])
                assert got == expect, (u, h, i, got, expect)


def test_group_of_one_is_the_per_head_rule():
    g = np.random.default_rng(7)
    scores = _causal(g.standard_normal((2, 3, 9, 9)))
    a = oracle.select_blocks(scores, 3, 2, 1)
    b = oracle.select_blocks_group(scores, 1, 3, 2, 1)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_group_of_identical_heads_keeps_each_heads_own_list():
    g = np.random.default_rng(8)
    one = _causal(g.standard_normal((1, 1, 10, 10)))
    scores = np.repeat(one, 4, axis=1)  # four identical query heads sharing a KV head
    own = oracle.select_blocks(one, 4, 1, 1)
    grp = oracle.select_blocks_group(scores, 4, 4, 1, 1)
    for h in range(4):
        assert np.array_equal(grp[0][0, h], own[0][0, 0])
        assert np.array_equal(grp[1][0, h], own[1][0, 0])


def test_group_select_counts_follow_the_closed_form():
    nb, group, k, w, ns = 16, 4, 5, 2, 1
    g = np.random.default_rng(9)
    scores = _causal(g.standard_normal((1, 8, nb, nb)))
    idx, cnt = oracle.select_blocks_group(scores, group, k, w, ns)
    for i in range(nb):
        forced = set(range(max(0, i - w + 1), i + 1)) | set(range(min(ns, i + 1)))
        assert np.all(cnt[0, :, i] == min(i + 1, k + len(forced)))
    assert int(cnt.sum()) == 8 * sum(min(i + 1, k + w + ns) for i in range(nb))


# ---------------------------------------------------------------------------
# Threshold selection (block probability >= tau, at most k)
# ---------------------------------------------------------------------------

def test_threshold_worked_example():
    """Row 3 with logits ln 1, ln 2, ln 3, ln 4: block probabilities 0.1, 0.2,
    0.3, 0.4; block 3 is the forced diagonal."""
    nb = 4
    scores = _causal(np.zeros((1, 1, nb, nb)))
    scores[0, 0, 3, :4] = np.log([1.0, 2.0, 3.0, 4.0])
    p = oracle.block_probabilities(scores[0, 0, 3], 3, 1.0)
    np.testing.assert_allclose(p, [0.1, 0.2, 0.3, 0.4], rtol=1e-14)
    row = lambda tau, k: list(oracle.select_blocks_threshold(scores, tau, k, 1, 0, 1.0)[0][0, 0, 3])
    assert row(0.15, 5)[:3] == [1, 2, 3]      # 0.2 and 0.3 pass
    assert row(0.15, 1)[:2] == [2, 3]         # cap at k: the better of the two
    assert row(0.25, 5)[:2] == [2, 3]         # only 0.3 passes
    assert row(0.35, 5)[:1] == [3]            # none pass: the forced block alone
    assert row(0.05, 5)[:4] == [0, 1, 2, 3]   # all pass


def test_threshold_limits_reduce_to_top_k():
    g = np.random.default_rng(11)
    scores = _causal(g.standard_normal((1, 2, 12, 12)))
    for k in (0, 2, 5):
        lo = oracle.select_blocks_threshold(scores, 1e-300, k, 2, 1, 0.5)
        ref = oracle.select_blocks(scores, k, 2, 1)
        assert np.array_equal(lo[0], ref[0]) and np.array_equal(lo[1], ref[1])
        hi = oracle.select_blocks_threshold(scores, 1.5, k, 2, 1, 0.5)
        none = oracle.select_blocks(scores, 0, 2, 1, width=ref[0].shape[-1])
        assert np.array_equal(hi[0], none[0]) and np.array_equal(hi[1], none[1])


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("tau,k,w,ns,scale", [(0.1, 3, 1, 0, 1.0), (0.05, 2, 2, 1, 0.7),
                                              (0.2, 8, 1, 1, 2.0), (0.01, 1, 0, 2, 1.3)])
def test_threshold_matches_brute_force(seed, tau, k, w, ns, scale):
    nb = 8
    g = np.random.default_rng(200 + seed)
    scores = _causal(g.standard_normal((1, 1, nb, nb)) * 1.5)
    idx, cnt = oracle.select_blocks_threshold(scores, tau, k, w, ns, scale)
    s32 = scores.astype(np.float32)
    for i in range(nb):
        logits = [scale * float(scores[0, 0, i, j]) for j in range(i + 1)]
        mx = max(logits)
        e = [math.exp(v - mx) for v in logits]
        z = math.fsum(e)
        forced = set(range(max(0, i - w + 1), i + 1)) if w > 0 else set()
        forced |= set(range(min(ns, i + 1)))
        passing = [j for j in range(i + 1) if j not in forced and e[j] / z >= tau]
        expect = brute_force_select(s32[0, 0, i], i, min(k, len(passing)), w, ns)
        assert list(idx[0, 0, i, :cnt[0, 0, i]]) == expect, (i, passing)


# ---------------------------------------------------------------------------
# Decode (one query token against a KV cache)
# ---------------------------------------------------------------------------

def _bf16(x):
    return W.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def test_decode_dense_is_textbook_attention_of_the_last_token():
    g = np.random.default_rng(41)
    Bn, Hq, Hkv, N, d, bs, L = 2, 4, 2, 256, 16, 32, 201
    q = _bf16(g.standard_normal((Bn, Hq, d)))
    k = _bf16(g.standard_normal((Bn, Hkv, N, d)))
    v = _bf16(g.standard_normal((Bn, Hkv, N, d)))
    idx, cnt, out, lse = oracle.decode(q, k, v, L, bs, 1000, 1, 0)
    qf, kf, vf = (W.bf16_bits_to_f32(a).astype(np.float64) for a in (q, k, v))
    for b in range(Bn):
        for h in range(Hq):
            assert cnt[b, h] == (L - 1) // bs + 1
            x = kf[b, h // 2, :L] @ qf[b, h] / math.sqrt(d)
            p = np.exp(x - x.max())
            np.testing.assert_allclose(out[b, h], (p / p.sum()) @ vf[b, h // 2, :L], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(lse[b, h], x.max() + math.log(p.sum()), rtol=1e-13)


def test_decode_matches_the_prefill_row_of_a_constant_query_block():
    """When every row of the last query block equals q and the block is
    complete, the block mean is q: decode keeps the prefill's row and its
    output is the prefill output of the block's last token."""
    g = np.random.default_rng(42)
    Bn, Hq, Hkv, N, d, bs = 1, 4, 2, 12 * 32, 16, 32
    k_free, w, ns = 3, 1, 1
    L = N
    qtok = g.standard_normal((Bn, Hq, d)).astype(np.float32)
    Q = g.standard_normal((Bn, Hq, N, d)).astype(np.float32)
    Q[:, :, N - bs:] = qtok[:, :, None, :]
    K = g.standard_normal((Bn, Hkv, N, d)).astype(np.float32)
    V = g.standard_normal((Bn, Hkv, N, d)).astype(np.float32)
    idx_p, cnt_p, (o_p, lse_p) = oracle.forward(_bf16(Q), _bf16(K), _bf16(V), bs, k_free, w, ns)
    idx, cnt, out, lse = oracle.decode(_bf16(qtok), _bf16(K), _bf16(V), L, bs, k_free, w, ns)
    i = N // bs - 1
    np.testing.assert_array_equal(idx, idx_p[:, :, i, :idx.shape[-1]])
    np.testing.assert_array_equal(cnt, cnt_p[:, :, i])
    np.testing.assert_allclose(out, o_p[:, :, N - 1], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, lse_p[:, :, N - 1], rtol=1e-13)


def test_decode_partial_block_uses_present_keys_only():
    g = np.random.default_rng(43)
    Bn, Hq, Hkv, N, d, bs, L = 1, 2, 1, 128, 8, 32, 70   # block 2 holds keys 64..69
    q = _bf16(g.standard_normal((Bn, Hq, d)))
    k = _bf16(g.standard_normal((Bn, Hkv, N, d)) * 3)
    v = _bf16(g.standard_normal((Bn, Hkv, N, d)))
    idx, cnt, out, lse = oracle.decode(q, k, v, L, bs, 0, 1, 0)   # the diagonal block only
    assert list(idx[0, 0, :cnt[0, 0]]) == [2]
    qf, kf, vf = (W.bf16_bits_to_f32(a).astype(np.float64) for a in (q, k, v))
    for h in range(Hq):
        x = kf[0, 0, 64:70] @ qf[0, h] / math.sqrt(d)
        p = np.exp(x - x.max())
        np.testing.assert_allclose(out[0, h], (p / p.sum()) @ vf[0, 0, 64:70], rtol=1e-12, atol=1e-14)


def test_decode_group_of_identical_heads_equals_per_head():
    g = np.random.default_rng(44)
    d, bs, N, L = 16, 32, 20 * 32, 20 * 32 - 5
    one = g.standard_normal((1, 1, d))
    q = _bf16(np.repeat(one, 4, axis=1))
    k = _bf16(g.standard_normal((1, 1, N, d)))
    v = _bf16(g.standard_normal((1, 1, N, d)))
    a = oracle.decode(q, k, v, L, bs, 4, 2, 1)
    b = oracle.decode(q, k, v, L, bs, 4, 2, 1, mode="group")
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


# ---------------------------------------------------------------------------
# Backward (gradients of the sparse attention)
# ---------------------------------------------------------------------------

def _mixed_lists(B, Hq, nb, seed, keep_prob=0.6):
    """Random kept lists: the diagonal always, other causal blocks at random."""
    g = np.random.default_rng(seed)
    idx = np.full((B, Hq, nb, nb), -1, dtype=np.int32)
    cnt = np.zeros((B, Hq, nb), dtype=np.int32)
    for b in range(B):
        for h in range(Hq):
            for i in range(nb):
                lst = [j for j in range(i) if g.random() < keep_prob] + [i]
                idx[b, h, i, :len(lst)] = lst
                cnt[b, h, i] = len(lst)
    return idx, cnt


def _loss(q, k, v, gout, idx, cnt, bs):
    o, _ = oracle.sparse_attention(q, k, v, idx, cnt, bs)
    return float((o * gout).sum())


@pytest.mark.parametrize("seed", [0, 1])
def test_backward_matches_central_differences(seed):
    # L = sum(O * G) has dL/dO = G, so the gradients must equal the central
    # differences of the oracle's own forward along random directions
    B, Hq, Hkv, N, d, bs = 1, 4, 2, 12, 4, 3
    g = np.random.default_rng(100 + seed)
    q = g.standard_normal((B, Hq, N, d))
    k = g.standard_normal((B, Hkv, N, d))
    v = g.standard_normal((B, Hkv, N, d))
    gout = g.standard_normal((B, Hq, N, d))
    idx, cnt = _mixed_lists(B, Hq, N // bs, seed)
    dq, dk, dv = oracle.sparse_attention_backward(q, k, v, gout, idx, cnt, bs)
    eps = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for t in range(3):
            u = g.standard_normal(x.shape)
            args = {"q": q, "k": k, "v": v}
            args[name] = x + eps * u
            lp = _loss(args["q"], args["k"], args["v"], gout, idx, cnt, bs)
            args[name] = x - eps * u
            lm = _loss(args["q"], args["k"], args["v"], gout, idx, cnt, bs)
            fd = (lp - lm) / (2 * eps)
            an = float((grad * u).sum())
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_backward_dense_lists_match_autograd_of_causal_attention():
    # every causal block kept: the gradients are those of dense causal
    # attention, here through PyTorch's autograd on the textbook routine
    B, Hq, Hkv, N, d, bs = 1, 4, 2, 16, 8, 4
    q = rand_bits((B, Hq, N, d), 11)
    k = rand_bits((B, Hkv, N, d), 12)
    v = rand_bits((B, Hkv, N, d), 13)
    do = rand_bits((B, Hq, N, d), 14)
    nb = N // bs
    idx = np.full((B, Hq, nb, nb), -1, dtype=np.int32)
    cnt = np.zeros((B, Hq, nb), dtype=np.int32)
    for i in range(nb):
        idx[:, :, i, :i + 1] = np.arange(i + 1)
        cnt[:, :, i] = i + 1
    dq, dk, dv = oracle.sparse_attention_backward(q, k, v, do, idx, cnt, bs)
    qt, kt, vt = (f64(x).requires_grad_(True) for x in (q, k, v))
    o = F.scaled_dot_product_attention(qt, kt.repeat_interleave(Hq // Hkv, 1),
                                       vt.repeat_interleave(Hq // Hkv, 1), is_causal=True)
    o.backward(f64(do))
    np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, kt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, vt.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_invariants():
    B, Hq, Hkv, N, d, bs = 2, 4, 2, 24, 8, 4
    q = rand_bits((B, Hq, N, d), 21)
    k = rand_bits((B, Hkv, N, d), 22)
    v = rand_bits((B, Hkv, N, d), 23)
    do = rand_bits((B, Hq, N, d), 24)
    idx, cnt = _mixed_lists(B, Hq, N // bs, 25, keep_prob=0.4)
    dq, dk, dv = oracle.sparse_attention_backward(q, k, v, do, idx, cnt, bs)
    g = Hq // Hkv
    # softmax weights sum to one: sum over keys of dV is the sum of dO over the
    # group's query rows (every row sees at least its own key)
    dof = oracle.bf16_to_f64(do)
    for b in range(B):
        for kvh in range(Hkv):
            np.testing.assert_allclose(dv[b, kvh].sum(axis=0), dof[b, kvh * g:(kvh + 1) * g].sum(axis=(0, 1)),
                                       rtol=1e-10, atol=1e-10)
            # shifting every key by one vector shifts each row's logits by a
            # constant: the softmax, hence the loss, does not move
            np.testing.assert_allclose(dk[b, kvh].sum(axis=0), 0.0, atol=1e-10)
    # query row 0 sees only key 0: its softmax is constant, its gradient 0
    np.testing.assert_allclose(dq[:, :, 0], 0.0, atol=1e-14)
    # a key block that no list keeps receives no gradient
    kept = np.zeros((B, Hkv, N // bs), dtype=bool)
    for b in range(B):
        for h in range(Hq):
            for i in range(N // bs):
                kept[b, h // g, idx[b, h, i, :cnt[b, h, i]]] = True
    for b, kvh, j in zip(*np.nonzero(~kept)):
        assert np.all(dk[b, kvh, j * bs:(j + 1) * bs] == 0) and np.all(dv[b, kvh, j * bs:(j + 1) * bs] == 0)


def test_backward_items_equal_the_full_result():
    B, Hq, Hkv, N, d, bs = 1, 4, 1, 16, 8, 4
    q = rand_bits((B, Hq, N, d), 31)
    k = rand_bits((B, Hkv, N, d), 32)
    v = rand_bits((B, Hkv, N, d), 33)
    do = rand_bits((B, Hq, N, d), 34)
    idx, cnt = _mixed_lists(B, Hq, N // bs, 35)
    dq, dk, dv = oracle.sparse_attention_backward(q, k, v, do, idx, cnt, bs)
    # dK/dV of key block 1: the query blocks whose lists keep it
    items = [(0, h, i) for h in range(Hq) for i in range(N // bs) if 1 in idx[0, h, i, :cnt[0, h, i]]]
    items = sorted(set(items) | {(0, 2, 3)})
    dqb, dkb, dvb = oracle.sparse_attention_backward(q, k, v, do, idx, cnt, bs, items=items)
    np.testing.assert_allclose(dqb[(0, 2, 3)], dq[0, 2, 12:16], rtol=0, atol=1e-13)
    np.testing.assert_allclose(dkb[(0, 0, 1)], dk[0, 0, 4:8], rtol=0, atol=1e-13)
    np.testing.assert_allclose(dvb[(0, 0, 1)], dv[0, 0, 4:8], rtol=0, atol=1e-13)
