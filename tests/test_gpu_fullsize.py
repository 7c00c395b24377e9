"""GPU parity at the full workload sizes, in the benchmark's launch configuration.

For each of the five workloads:
  - selection: every row of dsa_forward's kept lists against the oracle's
    (set comparison with the near-tie rule of tests/parity.py);
  - attention: dsa_sparse_attn_fwd on the oracle's own lists, element by
    element, on EVERY query block of tiny, 8k-gqa, 32k-gqa and batched-32,
    and on a seeded 1/16 of the (head, query block) pairs of 128k-structured
    plus the last query block of every head; max |O - O_ref| <= 2e-2 and
    ||O - O_ref|| / ||O_ref|| <= 5e-3 over everything checked, and the
    log-sum-exp within 2e-3;
  - dsa_forward's own output on every checked block whose selection equals
    the oracle's.
The backward at 32K runs the oracle's backward over every query block (every
dK and dV block is compared) and compares dQ on a seeded 1/16 of the query
blocks. The oracle runs on every host core (oracle.parallel: spawn-started
worker processes, one BLAS thread each).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.parallel import OraclePool
from dynamic_block_sparse_02_b200 import WORKLOADS, WORKLOAD_ORDER, binding as B
from dynamic_block_sparse_02_b200 import workloads as W
from dynamic_block_sparse_02_b200.attention import BlockSparseAttention

from parity import ATOL_MAX, LSE_ATOL, REL_RMS, compare_selection, dev_bf16, dev_i32

pytestmark = pytest.mark.gpu

REL_RMS_BWD = 1e-2   # the backward tolerance of tests/test_gpu_backward.py
MAX_REL_BWD = 2e-2


@pytest.fixture(scope="module", autouse=True)
def need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    torch.cuda.set_device(0)


class RowScores:
    """Oracle block scores computed row by row on demand (fp64, -inf above
    the diagonal), indexable like the [B, Hq, nb, nb] array."""

    def __init__(self, x, block, group):
        self.qp = oracle.pool_blocks(x["q"], block)
        self.kp = oracle.pool_blocks(x["k"], block)
        self.g = group

    def __getitem__(self, key):
        b, h, i = key
        nb = self.qp.shape[2]
        row = np.full(nb, -np.inf)
        row[:i + 1] = self.kp[b, h // self.g, :i + 1] @ self.qp[b, h, i]
        return row


def width_of(w, kph):
    return oracle.row_width(w.nb, max(kph) if kph is not None else w.k_free, w.local_window, w.n_sink)


class Accum:
    """Running max-abs and sums of squares over everything checked."""

    def __init__(self):
        self.max_abs = 0.0
        self.d2 = 0.0
        self.r2 = 0.0
        self.lse_err = 0.0
        self.blocks = 0

    def add(self, o_g, o_r, l_g=None, l_r=None, what=""):
        diff = o_g - o_r
        self.max_abs = max(self.max_abs, float(np.abs(diff).max()) if diff.size else 0.0)
        self.d2 += float(np.sum(diff * diff))
        self.r2 += float(np.sum(o_r * o_r))
        self.blocks += 1
        if l_r is not None:
            fin = np.isfinite(l_r)
            assert np.array_equal(fin, np.isfinite(l_g)), f"{what}: -inf pattern of lse differs"
            if fin.any():
                self.lse_err = max(self.lse_err, float(np.abs(l_g[fin] - l_r[fin]).max()))

    def check(self, what):
        rel = (self.d2 ** 0.5) / max(self.r2 ** 0.5, 1e-30)
        print(f"{what}: {self.blocks} blocks, max_abs={self.max_abs:.3e} rel_rms={rel:.3e} "
              f"lse_err={self.lse_err:.3e}")
        assert self.max_abs <= ATOL_MAX and rel <= REL_RMS, (what, self.max_abs, rel)
        assert self.lse_err <= LSE_ATOL, (what, self.lse_err)


def checked_items(w):
    """Every query block, except for the 128K workload: a seeded 1/16 of its
    (head, query block) pairs plus the last query block of every head."""
    every = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(w.nb)]
    if w.name != "128k-structured":
        return every
    g = np.random.default_rng(2024)
    pick = g.choice(len(every), size=len(every) // 16, replace=False)
    items = {every[t] for t in pick}
    items.update((b, h, w.nb - 1) for b in range(w.B) for h in range(w.Hq))
    return sorted(items)


@pytest.mark.parametrize("name", list(WORKLOAD_ORDER))
def test_full_workload(name):
    w = WORKLOADS[name]
    kph = W.per_head_k(w)
    kph = None if kph is None else [int(t) for t in kph]
    k_sel = kph if kph is not None else w.k_free
    x = W.make_inputs(w)
    width = width_of(w, kph)
    bs = w.block
    with OraclePool(dict(q=x["q"], k=x["k"], v=x["v"])) as pool:
        idx_ref, cnt_ref = pool.select(w.B, w.Hkv, w.group, bs, k_sel, w.local_window, w.n_sink, width)
        pool.put("idx", idx_ref)
        pool.put("cnt", cnt_ref)

        q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
        att = BlockSparseAttention.from_workload(w, k_per_head=kph)
        assert att.width == width
        # the whole path, as the benchmark runs it
        idx_g, cnt_g = att.empty_selection()
        out_f, lse_f = att.empty_out(), att.empty_lse()
        att.forward(q, k, v, out_f, lse_f, idx_g, cnt_g)
        assert att.check_status() == B.DSA_OK
        idx_h, cnt_h = idx_g.cpu().numpy(), cnt_g.cpu().numpy()
        n, ties, bad = compare_selection(idx_h, cnt_h, idx_ref, cnt_ref, RowScores(x, bs, w.group),
                                         kph if kph is not None else [w.k_free] * w.Hq,
                                         w.local_window, w.n_sink)
        print(f"{name}: {n} rows, {ties} near-tie rows, {len(bad)} mismatches")
        assert not bad, bad[:5]
        # the attention kernel on the oracle's lists
        out, lse = att.empty_out(), att.empty_lse()
        att.sparse_attn(q, k, v, dev_i32(idx_ref), dev_i32(cnt_ref), out, lse)
        assert att.check_status() == B.DSA_OK
        o_h = out.float().cpu().numpy()
        l_h = lse.cpu().numpy()
        o_fh = out_f.float().cpu().numpy()
        # where AUTO runs the warp-MMA kernel, the tcgen05 kernel is checked too
        o_th = l_th = None
        if B.dsa_attn_uses_tcgen05(att.params) == 0:
            att_t = BlockSparseAttention.from_workload(w, k_per_head=kph, attn_kernel=B.DSA_ATTN_TCGEN05)
            att_t.sparse_attn(q, k, v, dev_i32(idx_ref), dev_i32(cnt_ref), out, lse)
            assert att_t.check_status() == B.DSA_OK
            o_th, l_th = out.float().cpu().numpy(), lse.cpu().numpy()
        del q, k, v, out, lse, out_f, lse_f
        items = checked_items(w)
        acc, acc_f, acc_t = Accum(), Accum(), Accum()
        step = 2048
        for s0 in range(0, len(items), step):
            batch = items[s0:s0 + step]
            ref = pool.attention(batch, bs)
            for (b, h, i) in batch:
                rows = slice(i * bs, (i + 1) * bs)
                o_r, l_r = ref[(b, h, i)]
                acc.add(o_h[b, h, rows].astype(np.float64), o_r, l_h[b, h, rows].astype(np.float64), l_r,
                        f"{name} {(b, h, i)}")
                if np.array_equal(idx_h[b, h, i], idx_ref[b, h, i]):
                    acc_f.add(o_fh[b, h, rows].astype(np.float64), o_r)
                if o_th is not None:
                    acc_t.add(o_th[b, h, rows].astype(np.float64), o_r, l_th[b, h, rows].astype(np.float64),
                              l_r, f"{name} tcgen05 {(b, h, i)}")
    acc.check(f"{name} attention on the oracle's lists")
    if o_th is not None:
        acc_t.check(f"{name} tcgen05 kernel on the oracle's lists")
    acc_f.check(f"{name} dsa_forward on rows selected as the oracle")
    assert acc_f.blocks >= 0.99 * acc.blocks


def check_grad(name, g, r):
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    assert np.all(np.isfinite(g)), name
    scale = max(np.abs(r).max(), 1e-30)
    rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    mx = np.abs(g - r).max() / scale
    print(f"{name}: rel_rms={rel:.3e} max_rel={mx:.3e}")
    assert rel <= REL_RMS_BWD and mx <= MAX_REL_BWD, (name, rel, mx)


def test_backward_full_size_32k():
    w = WORKLOADS["32k-gqa"]
    x = W.make_inputs(w, seed=68)
    do_bits = W.f32_to_bf16_bits(np.random.default_rng(69).standard_normal(x["q"].shape).astype(np.float32))
    bs, g = w.block, w.group
    width = width_of(w, None)
    every = [(0, h, i) for h in range(w.Hq) for i in range(w.nb)]
    pick = np.random.default_rng(70).choice(len(every), size=len(every) // 16, replace=False)
    q_items = sorted(every[t] for t in pick)
    with OraclePool(dict(q=x["q"], k=x["k"], v=x["v"], dout=do_bits)) as pool:
        idx, cnt = pool.select(w.B, w.Hkv, g, bs, w.k_free, w.local_window, w.n_sink, width)
        pool.put("idx", idx)
        pool.put("cnt", cnt)
        att = BlockSparseAttention.from_workload(w)
        q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
        di, dc = dev_i32(idx), dev_i32(cnt)
        out = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
        att.sparse_attn(q, k, v, di, dc, out, lse)
        dq, dk, dv = att.sparse_attn_backward(q, k, v, out, lse, dev_bf16(do_bits), di, dc)
        torch.cuda.synchronize()
        assert att.check_status() == B.DSA_OK
        dq_h, dk_h, dv_h = (t.float().cpu().numpy().astype(np.float64) for t in (dq, dk, dv))
        del q, k, v, out, lse, dq, dk, dv
        rq, rk, rv = pool.backward(every, bs, keep_dq=q_items, per_worker=1)
    gq = np.concatenate([dq_h[b, h, i * bs:(i + 1) * bs] for (b, h, i) in q_items])
    check_grad("dq (1/16 of the query blocks)", gq, np.concatenate([rq[it] for it in q_items]))
    rk_full = np.zeros_like(dk_h)
    rv_full = np.zeros_like(dv_h)
    for (b, kvh, j), val in rk.items():
        rk_full[b, kvh, j * bs:(j + 1) * bs] = val
    for (b, kvh, j), val in rv.items():
        rv_full[b, kvh, j * bs:(j + 1) * bs] = val
    check_grad("dk (every key block)", dk_h, rk_full)
    check_grad("dv (every key block)", dv_h, rv_full)
    # key blocks no list keeps get exactly zero
    kept = np.zeros((w.Hkv, w.nb), dtype=bool)
    for h in range(w.Hq):
        for i in range(w.nb):
            kept[h // g, idx[0, h, i, :cnt[0, h, i]]] = True
    for kvh, j in np.argwhere(~kept):
        assert not np.any(dk_h[0, kvh, j * bs:(j + 1) * bs]) and not np.any(dv_h[0, kvh, j * bs:(j + 1) * bs])
