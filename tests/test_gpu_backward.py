"""GPU parity of the backward pass (dsa_sparse_attn_bwd) against the fp64
oracle, through the C ABI.

The kept lists come from the oracle's selection and feed both sides; the GPU
forward (dsa_sparse_attn_fwd on those lists) supplies the out and lse that the
GPU backward takes. Tolerance (derived from the arithmetic): the GPU rounds P
and dS to bf16 before the products with dO, K and Q (relative error 2^-9 each)
and rounds dQ, dK, dV to bf16 (2^-9), and takes D = dO . O from the bf16
forward output; the sums are fp32. Each gradient tensor must meet
||g - r||_2 / ||r||_2 <= 1e-2 and max |g - r| <= 2e-2 * max |r|.
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_02_b200 import WORKLOADS, Workload, binding as B
from dynamic_block_sparse_02_b200 import workloads as W
from dynamic_block_sparse_02_b200.attention import BlockSparseAttention

from parity import bf16_to_f64, dev_bf16, dev_i32

pytestmark = pytest.mark.gpu
REL_RMS_BWD = 1e-2
MAX_REL_BWD = 2e-2


@pytest.fixture(scope="module", autouse=True)
def need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    torch.cuda.set_device(0)


def oracle_lists(w, x):
    qp = oracle.pool_blocks(x["q"], w.block)
    kp = oracle.pool_blocks(x["k"], w.block)
    s = oracle.block_scores(qp, kp)
    return oracle.select_blocks(s, w.k_free, w.local_window, w.n_sink)


KERNELS = [B.DSA_ATTN_AUTO, B.DSA_ATTN_MMA_SYNC]


def gpu_backward(w, x, do_bits, idx, cnt, kernel=B.DSA_ATTN_AUTO):
    att = BlockSparseAttention.from_workload(w, attn_kernel=kernel)
    q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    di, dc = dev_i32(idx), dev_i32(cnt)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    att.sparse_attn(q, k, v, di, dc, out, lse)
    dq, dk, dv = att.sparse_attn_backward(q, k, v, out, lse, dev_bf16(do_bits), di, dc)
    torch.cuda.synchronize()
    assert att.check_status() == B.DSA_OK
    return dq, dk, dv


@pytest.mark.parametrize("scale", [0.4, 0.03])
def test_backward_custom_scale(scale):
    w = Workload("scale-bwd", 1, 4, 2, 64 * 10, 128, 64, k_free=3, local_window=1, n_sink=1, scale=scale)
    x = W.make_inputs(w, seed=14)
    idx, cnt = oracle_lists(w, x)
    do_bits = W.f32_to_bf16_bits(np.random.default_rng(15).standard_normal(x["q"].shape).astype(np.float32))
    rq, rk, rv = oracle.sparse_attention_backward(x["q"], x["k"], x["v"], do_bits, idx, cnt, w.block,
                                                  scale=scale)
    for kern in KERNELS:
        dq, dk, dv = gpu_backward(w, x, do_bits, idx, cnt, kern)
        for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            check_grad(f"{name} kernel {kern} scale {scale}", g.float().cpu().numpy(), r)


def test_backward_skips_repeated_and_descending_entries():
    # the rule of the forward: an entry not greater than the one before it is
    # skipped and flagged; the gradients are those of the remaining lists
    from test_gpu_parity import cleaned_lists, disorder
    w = Workload("bad-order-bwd", 1, 4, 2, 64 * 8, 128, 64, k_free=3, local_window=1, n_sink=0)
    x = W.make_inputs(w, seed=12)
    idx, cnt = oracle_lists(w, x)
    bad = disorder(idx, cnt)
    clean, ccnt = cleaned_lists(bad, cnt, w.nb)
    do_bits = W.f32_to_bf16_bits(np.random.default_rng(13).standard_normal(x["q"].shape).astype(np.float32))
    rq, rk, rv = oracle.sparse_attention_backward(x["q"], x["k"], x["v"], do_bits, clean, ccnt, w.block)
    q, k, v = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    for kern in KERNELS:
        att = BlockSparseAttention.from_workload(w, attn_kernel=kern)
        out = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
        att.sparse_attn(q, k, v, dev_i32(bad), dev_i32(cnt), out, lse)
        assert att.check_status() == B.DSA_ERR_DEVICE_BOUNDS
        dq, dk, dv = att.sparse_attn_backward(q, k, v, out, lse, dev_bf16(do_bits), dev_i32(bad), dev_i32(cnt))
        torch.cuda.synchronize()
        assert att.check_status() == B.DSA_ERR_DEVICE_BOUNDS
        assert att.check_status() == B.DSA_OK
        for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            check_grad(f"{name} kernel {kern}", g.float().cpu().numpy(), r)


def check_grad(name, g, r):
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    assert np.all(np.isfinite(g)), name
    scale = max(np.abs(r).max(), 1e-30)
    rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    mx = np.abs(g - r).max() / scale
    assert rel <= REL_RMS_BWD and mx <= MAX_REL_BWD, (name, rel, mx)


CASES = {
    # name: (B, Hq, Hkv, N, d, block, k_free, local_window, n_sink)
    "gqa-d128-bs64": (2, 8, 2, 64 * 12, 128, 64, 3, 2, 1),
    "mha-d64-bs32": (1, 4, 4, 32 * 20, 64, 32, 4, 1, 1),
    "g4-d128-bs128": (1, 4, 1, 128 * 7, 128, 128, 2, 1, 1),
    "g2-d64-bs128": (1, 4, 2, 128 * 6, 64, 128, 2, 1, 0),
    "g8-d64-bs64": (1, 8, 1, 64 * 10, 64, 64, 3, 1, 1),
    "g2-d128-bs32": (1, 4, 2, 32 * 18, 128, 32, 5, 2, 2),
}


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("name", list(CASES))
def test_backward_parity(name, kernel):
    Bn, Hq, Hkv, N, d, bs, k, lw, ns = CASES[name]
    w = Workload(name, Bn, Hq, Hkv, N, d, bs, k_free=k, local_window=lw, n_sink=ns)
    x = W.make_inputs(w, seed=61)
    do_bits = W.f32_to_bf16_bits(np.random.default_rng(62).standard_normal(x["q"].shape).astype(np.float32))
    idx, cnt = oracle_lists(w, x)
    dq, dk, dv = gpu_backward(w, x, do_bits, idx, cnt, kernel)
    rq, rk, rv = oracle.sparse_attention_backward(x["q"], x["k"], x["v"], do_bits, idx, cnt, bs)
    check_grad("dq", bf16_to_f64(dq), rq)
    check_grad("dk", bf16_to_f64(dk), rk)
    check_grad("dv", bf16_to_f64(dv), rv)


@pytest.mark.parametrize("kernel", KERNELS)
def test_backward_caller_lists_with_empty_rows_and_no_diagonal(kernel):
    # rows with no kept block (lse = -inf: no gradient) and rows whose list
    # skips the diagonal block
    w = Workload("custom", 1, 4, 2, 64 * 8, 128, 64, k_free=3, local_window=1, n_sink=0)
    x = W.make_inputs(w, seed=63)
    do_bits = W.f32_to_bf16_bits(np.random.default_rng(64).standard_normal(x["q"].shape).astype(np.float32))
    nb, width = w.nb, 4
    rng = np.random.default_rng(65)
    idx = np.full((1, 4, nb, width), -1, dtype=np.int32)
    cnt = np.zeros((1, 4, nb), dtype=np.int32)
    for h in range(4):
        for i in range(nb):
            if (h + i) % 5 == 0:
                continue  # empty row
            pool = list(range(i)) if (h + i) % 3 == 0 and i > 0 else list(range(i + 1))
            lst = sorted(rng.choice(pool, size=min(width, len(pool)), replace=False).tolist())
            idx[0, h, i, :len(lst)] = lst
            cnt[0, h, i] = len(lst)
    dq, dk, dv = gpu_backward(w, x, do_bits, idx, cnt, kernel)
    rq, rk, rv = oracle.sparse_attention_backward(x["q"], x["k"], x["v"], do_bits, idx, cnt, w.block)
    check_grad("dq", bf16_to_f64(dq), rq)
    check_grad("dk", bf16_to_f64(dk), rk)
    check_grad("dv", bf16_to_f64(dv), rv)
    gq = bf16_to_f64(dq)
    for h in range(4):
        for i in range(nb):
            if cnt[0, h, i] == 0:
                assert np.all(gq[0, h, i * 64:(i + 1) * 64] == 0)


@pytest.mark.parametrize("kernel", KERNELS)
def test_backward_is_deterministic(kernel):
    Bn, Hq, Hkv, N, d, bs, k, lw, ns = CASES["gqa-d128-bs64"]
    w = Workload("det", Bn, Hq, Hkv, N, d, bs, k_free=k, local_window=lw, n_sink=ns)
    x = W.make_inputs(w, seed=66)
    do_bits = W.f32_to_bf16_bits(np.random.default_rng(67).standard_normal(x["q"].shape).astype(np.float32))
    idx, cnt = oracle_lists(w, x)
    a = gpu_backward(w, x, do_bits, idx, cnt, kernel)
    b = gpu_backward(w, x, do_bits, idx, cnt, kernel)
    for ta, tb in zip(a, b):
        assert torch.equal(ta, tb)
