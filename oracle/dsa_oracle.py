"""fp64 CPU oracle for dynamic top-k block-sparse causal attention (prefill).

TEST INFRASTRUCTURE. Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import or call this module. It shares no
code with the CUDA path: it never imports the ``dynamic_block_sparse_02_b200``
package, and that package never imports it.

What is computed, and where the pages say so:

* Block pooling and block scores. Each bs x bs tile of the attention matrix is
  decided as a unit (zblog.xzdbk.com/559 "dynamic sparse attention" post,
  section 硬件友好的稀疏计算实现: 64x64 blocks decided per block; "DeepSeek NSA"
  article, section 2.1: 32x32 blocks whose activation a light per-block
  predictor estimates). The pages never define the block estimate; the plain
  reading used here is score(i, j) = mean(Q block i) . mean(K block j).
* Selection. Each (query head, query block) keeps forced blocks (a local
  window ending at the diagonal, plus global sink blocks) and the top-k of the
  remaining causal key blocks (zblog post, section 基于Top-k选择的局部-全局混合:
  top-k with a local window plus global tokens; "稀疏注意力 vs Flash Attention
  v2", section 1: content-aware top-k and hybrid local+global modes). The
  ranking is taken on fp32 scores, because the "DeepSeek NSA" article, section
  2.2, keeps the routing decision in FP32; the oracle rounds its fp64 score to
  fp32 once and ranks on that, ties going to the lower block index.
* Group-shared selection (an alternative rule): one list per KV head, chosen
  by the same rule from the sum of its query heads' block scores and used by
  all of them (see group_scores).
* Threshold selection (an alternative rule): forced blocks plus the blocks
  whose share of the softmax over the row's block logits reaches tau, at most
  k of them (see select_blocks_threshold).
* Attention. softmax(Q K^T * scale) V over the kept key blocks only, with the
  causal mask inside the diagonal block ("稀疏注意力 vs Flash Attention v2",
  section 1 pseudocode: scores, then the sparsity pattern, then softmax with
  1/sqrt(d_k), then the product with V). Query head h reads KV head
  h // (Hq/Hkv) (GQA sharing; zblog post, section on speculative decoding,
  GQA/MQA remark).
* Decode (see decode): one query token against a KV cache, its own block
  scored by the mean of its present keys, the prefill rules on that row.
* Backward (see sparse_attention_backward): the exact gradients of the
  attention over the kept blocks with the lists held fixed.

Every function here is pinned by tests/test_oracle_pins.py against facts
independent of it (hand-built closed forms, brute force, PyTorch's textbook
attention and its autograd, central differences, invariants).

Everything is fp64 except the single fp32 rounding of the scores used for
ranking. The softmax is the exact two-pass form (row max, then the sum of
exponentials, then the weights), not an online one.

Readings of points the pages leave open (each repeated in the design notes):
a row whose kept set is empty has output 0 and log-sum-exp -inf; the pooled
diagonal block is the plain mean of all its rows (the causal mask inside it
does not enter the pooling); scores are unscaled (a positive scale cannot change
the ranking).
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np


# ---------------------------------------------------------------------------
# Input widening
# ---------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float64 exactly."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# Step 1: block pooling
# ---------------------------------------------------------------------------

def pool_blocks(x_bits: np.ndarray, block: int) -> np.ndarray:
    """Block means of a bf16 tensor [B,H,N,d] -> fp64 [B,H,N/block,d].

    pooled[b,h,i,:] = (1/block) * sum over rows r of block i of x[b,h,r,:].
    The per-block activation estimate of the "DeepSeek NSA" article, section
    2.1, read as a plain mean over the block's rows.
    """
    B, H, N, d = x_bits.shape
    if N % block:
        raise ValueError("N must be a multiple of the block size")
    nb = N // block
    out = np.empty((B, H, nb, d), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            x = bf16_to_f64(x_bits[b, h])
            out[b, h] = x.reshape(nb, block, d).mean(axis=1)
    return out


# ---------------------------------------------------------------------------
# Step 2: block scores
# ---------------------------------------------------------------------------

def block_scores(qp: np.ndarray, kp: np.ndarray) -> np.ndarray:
    """Causal block scores s[b,h,i,j] = qp[b,h,i] . kp[b, h // g, j] for j <= i.

    Entries above the diagonal (j > i) are -inf. No 1/sqrt(d) factor: a
    positive scale does not change the ranking ("DeepSeek NSA" section 2.2
    computes the routing scores at full precision before block sparsifying).
    """
    B, Hq, nb, d = qp.shape
    Hkv = kp.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    g = Hq // Hkv
    s = np.empty((B, Hq, nb, nb), dtype=np.float64)
    upper = np.triu(np.ones((nb, nb), dtype=bool), k=1)
    for b in range(B):
        for h in range(Hq):
            s[b, h] = qp[b, h] @ kp[b, h // g].T
            s[b, h][upper] = -np.inf
    return s


# ---------------------------------------------------------------------------
# Step 3: selection
# ---------------------------------------------------------------------------

def forced_set(i: int, local_window: int, n_sink: int) -> set:
    """Forced key blocks of query block i: the local window {i-w+1 .. i} and sinks {0 .. n_sink-1}.

    zblog post, section 基于Top-k选择的局部-全局混合 (local window plus global
    tokens); only causal blocks (j <= i) are ever forced.
    """
    win = set(range(max(0, i - local_window + 1), i + 1)) if local_window > 0 else set()
    sink = set(range(0, min(n_sink, i + 1)))
    return win | sink


def row_width(nb: int, k_max: int, local_window: int, n_sink: int) -> int:
    """Width of one row of the index output: min(nb, k + window + sinks)."""
    return min(nb, k_max + local_window + n_sink)


def select_blocks(scores: np.ndarray, k_free, local_window: int, n_sink: int,
                  width: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Kept key blocks per (b, query head, query block).

    S(i) = F(i) united with the min(k, |C(i)|) best blocks of
    C(i) = {0..i} minus F(i), where "best" orders by fp32 score descending, then
    block index ascending. ``k_free`` is an int, or one int per query head.
    Returns idx int32 [B,Hq,nb,width] (ascending, padded with -1) and cnt int32
    [B,Hq,nb].
    """
    B, Hq, nb, _ = scores.shape
    ks = np.full(Hq, int(k_free), dtype=np.int64) if np.isscalar(k_free) else \
        np.asarray(k_free, dtype=np.int64)
    if width is None:
        width = row_width(nb, int(ks.max()) if Hq else 0, local_window, n_sink)
    idx = np.full((B, Hq, nb, width), -1, dtype=np.int32)
    cnt = np.zeros((B, Hq, nb), dtype=np.int32)
    s32 = scores.astype(np.float32)  # the ranking precision (fp32 routing)
    for b in range(B):
        for h in range(Hq):
            for i in range(nb):
                forced = forced_set(i, local_window, n_sink)
                free = np.ones(i + 1, dtype=bool)
                free[sorted(forced)] = False
                cand = np.nonzero(free)[0].astype(np.int64)
                take = min(int(ks[h]), cand.size)
                if take > 0:
                    # lexsort: last key is primary -> score descending, index ascending
                    order = np.lexsort((cand, -s32[b, h, i, cand].astype(np.float64)))
                    picks = cand[order[:take]]
                else:
                    picks = np.empty(0, dtype=np.int64)
                kept = sorted(forced | set(int(j) for j in picks))
                if len(kept) > width:
                    raise ValueError("row width too small for the kept set")
                idx[b, h, i, :len(kept)] = kept
                cnt[b, h, i] = len(kept)
    return idx, cnt


def group_scores(scores: np.ndarray, group: int) -> np.ndarray:
    """Scores of the group-shared rule: for KV head g, the sum over its query
    heads h = g*group .. g*group+group-1 of their block scores (fp64, -inf
    above the diagonal). Returns [B, Hq/group, nb, nb].

    Follows the zblog.xzdbk.com/559 post (section on speculative decoding:
    with MQA/GQA the shared KV cache lowers the cost of keeping the sparse
    index) and the DSA post, section 2.1 (the indexer merges the lists of its
    index heads). The pages give no rule for combining the heads; the plain
    reading used here is the sum of the heads' block scores.
    """
    B, Hq, nb, _ = scores.shape
    if Hq % group:
        raise ValueError("Hq must be a multiple of the group size")
    s = scores.reshape(B, Hq // group, group, nb, nb)
    out = np.zeros((B, Hq // group, nb, nb), dtype=np.float64)
    for u in range(group):
        out += s[:, :, u]
    return out


def select_blocks_group(scores: np.ndarray, group: int, k_free: int, local_window: int,
                        n_sink: int, width: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Group-shared selection: one kept list per (b, KV head, query block),
    chosen by the same rule as select_blocks from the group's summed scores,
    and given to every query head of the group.

    Returns idx int32 [B,Hq,nb,width] and cnt int32 [B,Hq,nb] like
    select_blocks, with identical rows for the heads of a group.
    """
    B, Hq, nb, _ = scores.shape
    gs = group_scores(scores, group)
    idx_g, cnt_g = select_blocks(gs, int(k_free), local_window, n_sink, width)
    idx = np.repeat(idx_g, group, axis=1)
    cnt = np.repeat(cnt_g, group, axis=1)
    return idx, cnt


def block_probabilities(scores_row: np.ndarray, i: int, scale: float) -> np.ndarray:
    """Softmax over the causal key blocks 0..i of one query block's logits
    scale * s(i, j), in fp64 (the block-level attention distribution that the
    threshold rule compares with tau)."""
    z = scale * np.asarray(scores_row[:i + 1], dtype=np.float64)
    e = np.exp(z - z.max())
    return e / e.sum()


def select_blocks_threshold(scores: np.ndarray, tau: float, k_free, local_window: int,
                            n_sink: int, scale: float,
                            width: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Threshold selection: the forced set plus every remaining causal block
    whose block probability (block_probabilities) is >= tau, at most k_free of
    them (the best by the top-k order when more pass).

    Follows the DeepSeek NSA article, section 2.2 (block_sparsify with a
    threshold on the fp32 scores, 0.1 there) and section 4.2 (start the
    threshold at 0.05), and the zblog post's adaptive k-or-threshold advice
    (section 模型精度与稀疏度的动态平衡). The pages do not say what the
    threshold is compared with; the plain reading used here is each block's
    share of the softmax over the row's causal block logits.
    """
    B, Hq, nb, _ = scores.shape
    ks = np.full(Hq, int(k_free), dtype=np.int64) if np.isscalar(k_free) else \
        np.asarray(k_free, dtype=np.int64)
    if width is None:
        width = row_width(nb, int(ks.max()) if Hq else 0, local_window, n_sink)
    keff = np.zeros((B, Hq, nb), dtype=np.int64)
    for b in range(B):
        for h in range(Hq):
            for i in range(nb):
                forced = forced_set(i, local_window, n_sink)
                p = block_probabilities(scores[b, h, i], i, scale)
                passing = sum(1 for j in range(i + 1) if j not in forced and p[j] >= tau)
                keff[b, h, i] = min(int(ks[h]), passing)
    idx = np.full((B, Hq, nb, width), -1, dtype=np.int32)
    cnt = np.zeros((B, Hq, nb), dtype=np.int32)
    for b in range(B):
        for h in range(Hq):
            for i in range(nb):
                # the ranking of select_blocks on this row, with the row's own budget
                idx[b, h, i], cnt[b, h, i] = _select_row(scores[b, h, i], i, int(keff[b, h, i]),
                                                         local_window, n_sink, width)
    return idx, cnt


def _select_row(scores_row: np.ndarray, i: int, k: int, local_window: int, n_sink: int,
                width: int) -> Tuple[np.ndarray, int]:
    """select_blocks for one row with budget k: forced set plus the k best
    candidates by fp32 score, ties to the lower index; ascending, -1 padded."""
    forced = forced_set(i, local_window, n_sink)
    cand = np.array([j for j in range(i + 1) if j not in forced], dtype=np.int64)
    take = min(k, cand.size)
    s32 = np.asarray(scores_row, dtype=np.float64).astype(np.float32)
    if take > 0:
        order = np.lexsort((cand, -s32[cand].astype(np.float64)))
        picks = cand[order[:take]]
    else:
        picks = np.empty(0, dtype=np.int64)
    kept = sorted(forced | set(int(j) for j in picks))
    if len(kept) > width:
        raise ValueError("row width too small for the kept set")
    out = np.full(width, -1, dtype=np.int32)
    out[:len(kept)] = kept
    return out, len(kept)


# ---------------------------------------------------------------------------
# Step 4: attention over the kept blocks
# ---------------------------------------------------------------------------

def kept_keys(idx_row: np.ndarray, n: int, block: int) -> np.ndarray:
    """Token indices of the kept key blocks, ascending."""
    blocks = np.asarray(idx_row[:n], dtype=np.int64)
    if blocks.size == 0:
        return np.empty(0, dtype=np.int64)
    return (blocks[:, None] * block + np.arange(block)[None, :]).reshape(-1)


def block_weights(qblk: np.ndarray, kfull: np.ndarray, keys: np.ndarray, i: int, block: int,
                  scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Exact softmax weights of one query block over the given keys.

    qblk: fp64 [block, d] (rows i*block .. i*block+block-1); kfull: fp64 [N, d].
    Returns W [block, len(keys)] with zeros at causally masked positions, and
    lse [block] (natural log; -inf for a row with no visible key).
    Two passes: row max of the visible logits, then the sum of exponentials.
    """
    rows = i * block + np.arange(block)
    if keys.size == 0:
        return np.zeros((block, 0)), np.full(block, -np.inf)
    logits = (qblk @ kfull[keys].T) * scale
    visible = keys[None, :] <= rows[:, None]
    logits = np.where(visible, logits, -np.inf)
    m = logits.max(axis=1)
    has = np.isfinite(m)
    m_safe = np.where(has, m, 0.0)
    e = np.where(visible, np.exp(logits - m_safe[:, None]), 0.0)
    l = e.sum(axis=1)
    w = np.where(has[:, None], e / np.where(has, l, 1.0)[:, None], 0.0)
    lse = np.where(has, m_safe + np.log(np.where(has, l, 1.0)), -np.inf)
    return w, lse


def sparse_attention(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray,
                     idx: np.ndarray, cnt: np.ndarray, block: int, scale: float = 0.0,
                     items: Optional[Iterable[Tuple[int, int, int]]] = None):
    """Block-sparse causal attention over the kept blocks, in fp64.

    O[b,h,r] = sum over visible kept keys t of softmax_t(q_r . k_t * scale) v_t,
    with K/V of KV head h // (Hq/Hkv). ``scale`` 0 means 1/sqrt(d). Inputs are
    bf16 bit patterns (uint16), widened exactly, or fp64 arrays.

    With ``items`` None, returns (O fp64 [B,Hq,N,d], lse fp64 [B,Hq,N]).
    Otherwise ``items`` lists (b, h, i) query blocks and the result is a dict
    mapping each item to (O [block,d], lse [block]).
    """
    B, Hq, N, d = q_bits.shape
    Hkv = k_bits.shape[1]
    g = Hq // Hkv
    if scale == 0.0:
        scale = 1.0 / math.sqrt(d)
    nb = N // block
    full = items is None
    if full:
        items = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(nb)]
        out = np.zeros((B, Hq, N, d))
        lse = np.full((B, Hq, N), -np.inf)
    else:
        res = {}
    items = sorted(items)
    cache_kv = {}
    cache_q = {}
    for (b, h, i) in items:
        kvh = h // g
        if (b, kvh) not in cache_kv:
            cache_kv.clear()
            cache_kv[(b, kvh)] = (_f64(k_bits[b, kvh]), _f64(v_bits[b, kvh]))
        kf, vf = cache_kv[(b, kvh)]
        if (b, h) not in cache_q:
            cache_q.clear()
            cache_q[(b, h)] = _f64(q_bits[b, h])
        qf = cache_q[(b, h)]
        keys = kept_keys(idx[b, h, i], int(cnt[b, h, i]), block)
        w, l = block_weights(qf[i * block:(i + 1) * block], kf, keys, i, block, scale)
        o = w @ vf[keys] if keys.size else np.zeros((block, d))
        if full:
            out[b, h, i * block:(i + 1) * block] = o
            lse[b, h, i * block:(i + 1) * block] = l
        else:
            res[(b, h, i)] = (o, l)
    return (out, lse) if full else res


# ---------------------------------------------------------------------------
# The whole path
# ---------------------------------------------------------------------------

def forward(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray, block: int, k_free,
            local_window: int, n_sink: int, scale: float = 0.0,
            items: Optional[Sequence[Tuple[int, int, int]]] = None):
    """Pool, score, select, attend. Returns (idx, cnt, attention result).

    The attention result is as for ``sparse_attention`` (full arrays, or a dict
    over ``items``).
    """
    qp = pool_blocks(q_bits, block)
    kp = pool_blocks(k_bits, block)
    s = block_scores(qp, kp)
    idx, cnt = select_blocks(s, k_free, local_window, n_sink)
    att = sparse_attention(q_bits, k_bits, v_bits, idx, cnt, block, scale, items)
    return idx, cnt, att


# ---------------------------------------------------------------------------
# Backward: gradients of the sparse attention with respect to Q, K and V
# ---------------------------------------------------------------------------

def _f64(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) widened exactly; any other array taken as fp64."""
    return bf16_to_f64(x) if x.dtype == np.uint16 else np.asarray(x, dtype=np.float64)


def sparse_attention_backward(q, k, v, dout, idx: np.ndarray, cnt: np.ndarray, block: int,
                              scale: float = 0.0,
                              items: Optional[Iterable[Tuple[int, int, int]]] = None):
    """Gradients of the block-sparse causal attention, in fp64.

    The pages mention training with the sparse pattern (DeepSeek NSA article,
    section 2.2) but give no backward rule; the plain reading is the exact
    gradient of O = softmax(Q K^T * scale) V over the kept, causally visible
    keys, with the kept lists held fixed (selection is a discrete choice and
    passes no gradient). Per query block (b, h, i) with kept keys T:
      P = the softmax weights (block_weights), dP = dO V_T^T,
      D_r = sum_t P[r, t] dP[r, t]  (equal to dO_r . O_r),
      dS = P * (dP - D),
      dQ_i = scale * dS K_T,  dK_T += scale * dS^T Q_i,  dV_T += P^T dO_i,
    where dK, dV of KV head g sum over its query heads (GQA sharing).

    q, dout: [B, Hq, N, d]; k, v: [B, Hkv, N, d]; bf16 bit patterns (uint16)
    or fp64. With ``items`` None, returns (dq [B,Hq,N,d], dk [B,Hkv,N,d],
    dv [B,Hkv,N,d]). Otherwise ``items`` lists (b, h, i) query blocks and the
    result is (dq_blocks, dk_blocks, dv_blocks): dq_blocks[(b, h, i)] is
    [block, d]; dk_blocks[(b, g, j)] and dv_blocks[(b, g, j)] are [block, d],
    the contributions of the listed query blocks to key block j.
    """
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    if scale == 0.0:
        scale = 1.0 / math.sqrt(d)
    nb = N // block
    full = items is None
    if full:
        items = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(nb)]
        dq = np.zeros((B, Hq, N, d))
        dk = np.zeros((B, Hkv, N, d))
        dv = np.zeros((B, Hkv, N, d))
    else:
        dq_b, dk_b, dv_b = {}, {}, {}
    items = sorted(items)
    cache_kv, cache_q = {}, {}
    for (b, h, i) in items:
        kvh = h // g
        if (b, kvh) not in cache_kv:
            cache_kv.clear()
            cache_kv[(b, kvh)] = (_f64(k[b, kvh]), _f64(v[b, kvh]))
        kf, vf = cache_kv[(b, kvh)]
        if (b, h) not in cache_q:
            cache_q.clear()
            cache_q[(b, h)] = (_f64(q[b, h]), _f64(dout[b, h]))
        qf, dof = cache_q[(b, h)]
        rows = slice(i * block, (i + 1) * block)
        keys = kept_keys(idx[b, h, i], int(cnt[b, h, i]), block)
        if keys.size == 0:
            if not full:
                dq_b[(b, h, i)] = np.zeros((block, d))
            continue
        qb, dob = qf[rows], dof[rows]
        w, _ = block_weights(qb, kf, keys, i, block, scale)
        kt, vt = kf[keys], vf[keys]
        dp = dob @ vt.T
        drow = (w * dp).sum(axis=1)
        ds = w * (dp - drow[:, None])
        dq_i = scale * (ds @ kt)
        dk_t = scale * (ds.T @ qb)
        dv_t = w.T @ dob
        if full:
            dq[b, h, rows] = dq_i
            np.add.at(dk[b, kvh], keys, dk_t)
            np.add.at(dv[b, kvh], keys, dv_t)
        else:
            dq_b[(b, h, i)] = dq_i
            for c, j in enumerate(np.asarray(idx[b, h, i][:int(cnt[b, h, i])], dtype=np.int64)):
                sl = slice(c * block, (c + 1) * block)
                key = (b, kvh, int(j))
                if key not in dk_b:
                    dk_b[key] = np.zeros((block, d))
                    dv_b[key] = np.zeros((block, d))
                dk_b[key] += dk_t[sl]
                dv_b[key] += dv_t[sl]
    return (dq, dk, dv) if full else (dq_b, dk_b, dv_b)


# ---------------------------------------------------------------------------
# Decode: one new query token against a KV cache
# ---------------------------------------------------------------------------

def decode(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray, length: int, block: int,
           k_free, local_window: int, n_sink: int, scale: float = 0.0, mode: str = "topk",
           tau: float = 0.0, return_scores: bool = False):
    """One decode step: query token q [B, Hq, d] at position length-1, keys and
    values [B, Hkv, >= length, d] (only the first ``length`` are read).

    The token's query block is i = (length-1) // block. Block scores are
    q . mean(K block j) for j <= i, the mean taken over the block's present
    keys (all of them for j < i, the first length - i*block for j = i).
    Selection follows the prefill rules on that single row ("topk", "group":
    the group's query heads' scores summed, "threshold": block probability >=
    tau, at most k); attention is softmax(q K^T * scale) V over the present keys
    of the kept blocks (the pages: store the sparse index with the KV cache and
    reuse it at inference, zblog.xzdbk.com/559 post, section 动态开销与计算收益的
    权衡, point 2).

    Returns idx int32 [B,Hq,W], cnt int32 [B,Hq], out fp64 [B,Hq,d], lse fp64 [B,Hq]
    (and, with return_scores, the row's block scores [B,Hq,i+1] in fp64).
    """
    q = bf16_to_f64(q_bits)
    k = bf16_to_f64(k_bits)
    v = bf16_to_f64(v_bits)
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    i = (length - 1) // block
    nb_row = i + 1
    if scale == 0.0:
        scale = 1.0 / math.sqrt(d)
    ks = np.full(Hq, int(k_free), dtype=np.int64) if np.isscalar(k_free) else \
        np.asarray(k_free, dtype=np.int64)
    width = row_width(k.shape[2] // block, int(ks.max()) if Hq else 0, local_window, n_sink)
    kmeans = np.zeros((B, Hkv, nb_row, d))
    for j in range(nb_row):
        hi = min((j + 1) * block, length)
        kmeans[:, :, j] = k[:, :, j * block:hi].mean(axis=2)
    scores = np.einsum("bhd,bhjd->bhj", q, np.repeat(kmeans, g, axis=1))  # [B, Hq, i+1]
    if mode == "group":
        summed = scores.reshape(B, Hkv, g, nb_row).sum(axis=2)
        scores = np.repeat(summed, g, axis=1)
    idx = np.full((B, Hq, width), -1, dtype=np.int32)
    cnt = np.zeros((B, Hq), dtype=np.int32)
    out = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            row = scores[b, h]
            kk = int(ks[h])
            if mode == "threshold":
                forced = forced_set(i, local_window, n_sink)
                p = block_probabilities(row, i, scale)
                kk = min(kk, sum(1 for j in range(i + 1) if j not in forced and p[j] >= tau))
            idx[b, h], cnt[b, h] = _select_row(row, i, kk, local_window, n_sink, width)
            keys = np.concatenate([np.arange(j * block, min((j + 1) * block, length))
                                   for j in idx[b, h, :cnt[b, h]]]) if cnt[b, h] else np.empty(0, int)
            if keys.size == 0:
                continue
            kv = h // g
            logits = scale * (k[b, kv, keys] @ q[b, h])
            mx = logits.max()
            e = np.exp(logits - mx)
            z = e.sum()
            out[b, h] = (e / z) @ v[b, kv, keys]
            lse[b, h] = mx + math.log(z)
    if return_scores:
        return idx, cnt, out, lse, scores
    return idx, cnt, out, lse


def attended_pairs(idx: np.ndarray, cnt: np.ndarray, block: int) -> int:
    """Number of (query, key) score pairs that the kept blocks make visible (causal)."""
    total = 0
    for i_flat in np.ndindex(cnt.shape):
        i = i_flat[-1]
        for j in idx[i_flat][:cnt[i_flat]]:
            total += block * (block + 1) // 2 if j == i else block * block
    return total


def dense_pairs(n: int, causal: bool = False) -> int:
    """Score pairs of dense attention over n tokens: n^2, or n(n+1)/2 with the causal mask."""
    return n * (n + 1) // 2 if causal else n * n
