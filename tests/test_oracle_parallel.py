"""The oracle's process-pool runner returns the oracle's own per-item results."""
import numpy as np

import oracle
from oracle.parallel import OraclePool, host_cores
from dynamic_block_sparse_02_b200 import Workload
from dynamic_block_sparse_02_b200 import workloads as W


def test_pool_matches_serial_oracle():
    w = Workload("pool", 2, 4, 2, 64 * 9, 64, 64, k_free=3, local_window=1, n_sink=1)
    x = W.make_inputs(w, seed=4)
    s = oracle.block_scores(oracle.pool_blocks(x["q"], w.block), oracle.pool_blocks(x["k"], w.block))
    idx, cnt = oracle.select_blocks(s, w.k_free, w.local_window, w.n_sink)
    do = W.f32_to_bf16_bits(np.random.default_rng(0).standard_normal(x["q"].shape).astype(np.float32))
    items = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(w.nb)][::3]
    with OraclePool(dict(q=x["q"], k=x["k"], v=x["v"], idx=idx, cnt=cnt, dout=do), workers=3) as pool:
        got = pool.attention(items, w.block)
        gq, gk, gv = pool.backward(items, w.block)
    ref = oracle.sparse_attention(x["q"], x["k"], x["v"], idx, cnt, w.block, items=items)
    assert sorted(got) == sorted(ref)
    for it in items:
        np.testing.assert_array_equal(got[it][0], ref[it][0])
        np.testing.assert_array_equal(got[it][1], ref[it][1])
    rq, rk, rv = oracle.sparse_attention_backward(x["q"], x["k"], x["v"], do, idx, cnt, w.block, items=items)
    assert sorted(gq) == sorted(rq) and sorted(gk) == sorted(rk) and sorted(gv) == sorted(rv)
    for it in rq:
        np.testing.assert_array_equal(gq[it], rq[it])
    for key in rk:  # key-block sums may add the chunks in another order
        np.testing.assert_allclose(gk[key], rk[key], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(gv[key], rv[key], rtol=1e-12, atol=1e-12)
    assert host_cores() >= 1


def test_pool_selection_matches_serial_oracle():
    w = Workload("poolsel", 2, 6, 2, 32 * 23, 64, 32, k_free=4, local_window=2, n_sink=1)
    x = W.make_inputs(w, seed=5)
    kph = [1, 2, 3, 4, 5, 6]
    s = oracle.block_scores(oracle.pool_blocks(x["q"], w.block), oracle.pool_blocks(x["k"], w.block))
    width = oracle.row_width(w.nb, max(kph), w.local_window, w.n_sink)
    ref = oracle.select_blocks(s, kph, w.local_window, w.n_sink, width)
    with OraclePool(dict(q=x["q"], k=x["k"]), workers=2) as pool:
        got = pool.select(w.B, w.Hkv, w.group, w.block, kph, w.local_window, w.n_sink, width)
    np.testing.assert_array_equal(got[0], ref[0])
    np.testing.assert_array_equal(got[1], ref[1])
