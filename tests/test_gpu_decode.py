"""GPU parity of the decode step (one query token per head against a KV
cache, with the pooled key cache) against the fp64 oracle, through the C ABI:
the pooled cache, the kept blocks (near-tie rule at the k-th score, threshold
boundary for the threshold rule) and the output and log-sum-exp.
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_02_b200 import WORKLOADS, Workload, binding as B
from dynamic_block_sparse_02_b200 import workloads as W
from dynamic_block_sparse_02_b200.attention import BlockSparseAttention

from parity import TIE_REL, attention_errors, dev_bf16

pytestmark = pytest.mark.gpu
MODES = {"topk": B.DSA_SELECT_TOPK, "group": B.DSA_SELECT_GROUP_TOPK, "threshold": B.DSA_SELECT_THRESHOLD}


@pytest.fixture(scope="module", autouse=True)
def need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    torch.cuda.set_device(0)


def row_ok(g, r, s, i, k, w, ns, tau=None, scale=None):
    """A GPU row that differs from the oracle's is accepted when every block in
    the difference ties with the k-th candidate's score or sits at the threshold."""
    if g == r:
        return True
    forced = oracle.forced_set(i, w, ns)
    cand = sorted((j for j in range(i + 1) if j not in forced),
                  key=lambda j: (-float(np.float32(s[j])), j))
    kth = s[cand[min(k, len(cand)) - 1]] if cand and k > 0 else None
    p = oracle.block_probabilities(s, i, scale) if tau else None
    for j in set(g) ^ set(r):
        if j in forced:
            return False
        at_cut = kth is not None and abs(s[j] - kth) <= TIE_REL * max(abs(s[j]), abs(kth))
        at_bar = tau is not None and abs(p[j] - tau) <= 1e-4 * tau
        if not (at_cut or at_bar):
            return False
    return True


def run_decode(w, x, L, mode, tau=0.0, qscale=1.0):
    bs, d = w.block, w.d
    qtok = x["q"][:, :, L - 1, :].copy()
    if qscale != 1.0:
        qtok = W.f32_to_bf16_bits(W.bf16_bits_to_f32(qtok) * qscale)
    att = BlockSparseAttention.from_workload(w, select_mode=MODES[mode], select_tau=tau)
    kc, vc = dev_bf16(x["k"]), dev_bf16(x["v"])
    kp = att.pooled_key_cache()
    att.pool_keys(kc, kp, 0, (L - 1) // bs)
    idx = torch.empty((w.B, w.Hq, att.width), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.B, w.Hq), dtype=torch.int32, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    out = att.decode(dev_bf16(qtok), kc, vc, kp, L, None, lse, idx, cnt)
    torch.cuda.synchronize()
    assert att.check_status() == B.DSA_OK
    ref = oracle.decode(qtok, x["k"], x["v"], L, bs, w.k_free, w.local_window, w.n_sink,
                        scale=w.scale, mode=mode, tau=tau, return_scores=True)
    return att, kp, (idx.cpu().numpy(), cnt.cpu().numpy(), out.double().cpu().numpy(),
                     lse.cpu().numpy().astype(np.float64)), ref


def check(w, L, got, ref, tau=None):
    idx_g, cnt_g, out_g, lse_g = got
    idx_r, cnt_r, out_r, lse_r, s64 = ref
    i = (L - 1) // w.block
    scale = w.scale if w.scale else 1.0 / np.sqrt(w.d)
    same = np.zeros((w.B, w.Hq), dtype=bool)
    for b in range(w.B):
        for h in range(w.Hq):
            g = idx_g[b, h, :cnt_g[b, h]].tolist()
            r = idx_r[b, h, :cnt_r[b, h]].tolist()
            assert g == sorted(set(g)) and np.all(idx_g[b, h, cnt_g[b, h]:] == -1)
            assert row_ok(g, r, s64[b, h], i, w.k_free, w.local_window, w.n_sink, tau, scale), (b, h, g, r)
            same[b, h] = g == r
    max_abs, rel = attention_errors(out_g[same], out_r[same])
    assert max_abs <= 2e-2 and rel <= 5e-3, (max_abs, rel)
    fin = np.isfinite(lse_r) & same
    assert np.all(np.abs(lse_g[fin] - lse_r[fin]) <= 2e-3 * np.maximum(1.0, np.abs(lse_r[fin])))
    assert np.all(np.isneginf(lse_g[~np.isfinite(lse_r) & same]))


CASES = {
    # name: (B, Hq, Hkv, N, d, block, k_free, local_window, n_sink)
    "gqa-d128-bs64": (2, 8, 2, 64 * 20, 128, 64, 4, 2, 1),
    "mha-d64-bs32": (1, 4, 4, 32 * 45, 64, 32, 3, 1, 0),
    "gqa-d128-bs128": (1, 4, 1, 128 * 12, 128, 128, 3, 1, 1),
    "g8-d64-bs64-window-only": (1, 8, 1, 64 * 16, 64, 64, 0, 3, 0),
}
LENGTHS = [1, 31, 64, 65, 700]


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("mode", ["topk", "group"])
def test_decode_parity(name, mode):
    Bn, Hq, Hkv, N, d, bs, k, lw, ns = CASES[name]
    w = Workload(name, Bn, Hq, Hkv, N, d, bs, k_free=k, local_window=lw, n_sink=ns)
    x = W.make_inputs(w, seed=51)
    for L in LENGTHS + [N - 5, N]:
        if L > N:
            continue
        att, kp, got, ref = run_decode(w, x, L, mode)
        check(w, L, got, ref)
    # the pooled cache holds the block means
    nfull = (N - 1) // bs
    kp_ref = oracle.pool_blocks(x["k"][:, :, :nfull * bs], bs)
    np.testing.assert_allclose(kp.cpu().numpy()[:, :, :nfull].astype(np.float64), kp_ref, rtol=1e-5,
                               atol=1e-6)


@pytest.mark.parametrize("mode", ["topk", "group"])
def test_decode_custom_scale(mode):
    # a softmax scale other than 1/sqrt(d), large enough that the running
    # maxima move by many powers of two between blocks
    w = Workload("scale", 1, 8, 2, 64 * 24, 128, 64, k_free=5, local_window=2, n_sink=1, scale=0.45)
    x = W.make_inputs(w, seed=53)
    for L in (1, 64, 65, 777, 64 * 24):
        att, kp, got, ref = run_decode(w, x, L, mode)
        check(w, L, got, ref)


def test_decode_threshold():
    w = Workload("thr", 2, 8, 2, 64 * 30, 128, 64, k_free=10, local_window=1, n_sink=1)
    x = W.make_inputs(w, seed=52)
    for L in (65, 999, 64 * 30):
        att, kp, got, ref = run_decode(w, x, L, "threshold", tau=0.03, qscale=64.0)
        check(w, L, got, ref, tau=0.03)


@pytest.mark.parametrize("L", [32768, 20001])
def test_decode_full_size_32k(L):
    w = WORKLOADS["32k-gqa"]
    x = W.make_inputs(w, seed=53)
    att, kp, got, ref = run_decode(w, x, L, "topk")
    check(w, L, got, ref)
