"""Helpers shared by the GPU parity tests: device upload and the comparison rules.

Selection rule: kept-block sets must equal the oracle's, except that a block
may differ when its fp64 oracle score lies within 1e-5 (relative) of the
row's cut-off score (the oracle's k-th best free score), the near-tie case in
which fp32 rounding may legitimately reorder blocks.
Attention rule (over the oracle's own selection): max |O_gpu - O_ref| <= 2e-2
and ||O_gpu - O_ref||_2 / ||O_ref||_2 <= 5e-3.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TIE_REL = 1e-5
ATOL_MAX = 2e-2
REL_RMS = 5e-3
# Log-sum-exp of a row, natural log: the row sum adds the bf16-rounded P (each
# within 2^-8 of its fp32 value, the bf16 unit roundoff), so ln(row sum) is
# within -ln(1 - 2^-8) = 3.92e-3; the fp32 sums add at most n * 2^-24 relative
# (2.6e-4 at the 4,288 keys of a 32K row) and the fp32 logits and ex2.approx
# about 1e-5. A sharp softmax, where one P carries the sum, reaches the first
# term; many comparable terms average it out.
LSE_ATOL = 4.5e-3


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def dev_i32(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).cuda()


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def forced(i, w, ns):
    return oracle.forced_set(i, w, ns)


def compare_selection(idx_gpu, cnt_gpu, idx_ref, cnt_ref, scores64, k_per_head, w, ns,
                      rows=None):
    """Returns (n_rows_checked, n_tie_rows, list of unexcused mismatches).

    scores64: oracle fp64 scores [B,Hq,nb,nb]. k_per_head: ints per head.
    rows: optional iterable of (b, h, i) to check (default all).
    """
    B, Hq, nb, _ = idx_ref.shape
    if rows is None:
        rows = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(nb)]
    bad, ties, n = [], 0, 0
    for (b, h, i) in rows:
        n += 1
        g = set(idx_gpu[b, h, i, :cnt_gpu[b, h, i]].tolist())
        r = set(idx_ref[b, h, i, :cnt_ref[b, h, i]].tolist())
        pad_ok = np.all(idx_gpu[b, h, i, cnt_gpu[b, h, i]:] == -1)
        asc = list(idx_gpu[b, h, i, :cnt_gpu[b, h, i]])
        if not pad_ok or asc != sorted(asc) or len(set(asc)) != len(asc):
            bad.append((b, h, i, "layout"))
            continue
        if g == r:
            continue
        if len(g) != len(r):
            bad.append((b, h, i, "count", len(g), len(r)))
            continue
        f = forced(i, w, ns)
        if not f <= g:
            bad.append((b, h, i, "forced"))
            continue
        free = np.array([j for j in range(i + 1) if j not in f])
        s = scores64[b, h, i]
        order = free[np.lexsort((free, -s[free].astype(np.float32).astype(np.float64)))]
        k = min(int(k_per_head[h]), free.size)
        cut = s[order[k - 1]]
        ok = True
        for j in g ^ r:
            if abs(s[j] - cut) > TIE_REL * max(abs(s[j]), abs(cut)):
                ok = False
        if ok:
            ties += 1
        else:
            bad.append((b, h, i, "order", sorted(g - r), sorted(r - g)))
    return n, ties, bad


def attention_errors(o_gpu: np.ndarray, o_ref: np.ndarray):
    diff = o_gpu - o_ref
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    den = float(np.linalg.norm(o_ref))
    rel = float(np.linalg.norm(diff)) / den if den > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_attention_close(o_gpu, o_ref, what=""):
    max_abs, rel = attention_errors(o_gpu, o_ref)
    assert max_abs <= ATOL_MAX and rel <= REL_RMS, f"{what}: max_abs={max_abs:.3e} rel_rms={rel:.3e}"
    return max_abs, rel


def assert_lse_close(l_gpu, l_ref, what=""):
    fin = np.isfinite(l_ref)
    assert np.array_equal(fin, np.isfinite(l_gpu)), f"{what}: -inf pattern differs"
    if fin.any():
        err = float(np.max(np.abs(l_gpu[fin] - l_ref[fin])))
        assert err <= LSE_ATOL, f"{what}: lse max err {err:.3e}"
