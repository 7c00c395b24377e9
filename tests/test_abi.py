"""The C-ABI boundary on the host: the library loads, exports every declared
symbol, sizes its outputs and workspace, and rejects bad arguments with the
documented status before touching the device. No test here launches a kernel.
"""
import ctypes
import os
import re
import subprocess

import pytest

from dynamic_block_sparse_02_b200 import WORKLOADS, binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")

FAKE = 0x10000  # an aligned non-null address; never dereferenced by these tests


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for n in ("dsa_block_scores", "dsa_topk_select", "dsa_sparse_attn_fwd", "dsa_forward",
              "dsa_sparse_attn_bwd", "dsa_decode_fwd", "dsa_pool_keys",
              "dsa_workspace_size", "dsa_kmax", "dsa_check_status", "dsa_status_string",
              "dsa_attn_uses_tcgen05"):
        assert n in names


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(dsa_\w+)", out))
    assert set(names) <= exported, set(names) - exported
    for n in names:
        assert hasattr(B.raw(n), "__call__")
    assert set(names) == set(B.SIGNATURES)


def test_status_strings():
    for s in range(7):
        assert B.status_string(s) and B.status_string(s) != "unknown status"
    assert B.status_string(99) == "unknown status"


def kept_width(w, kmax_head):
    return min(w.nb, kmax_head + w.local_window + w.n_sink)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_kmax_and_workspace_size(name):
    w = WORKLOADS[name]
    kph = [8, 16, 32, 64] * (w.Hq // 4) if w.k_choices else None
    p = B.Params.from_workload(w, k_per_head=kph)
    width = B.dsa_kmax(p)
    assert width == kept_width(w, 64 if kph else w.k_free)
    expect = {"tiny": 4, "8k-gqa": 18, "32k-gqa": 67, "128k-structured": 65, "batched-32": 65}[name]
    assert width == expect
    ws = B.dsa_workspace_size(p)
    rnd = lambda x: (x + 255) // 256 * 256
    prefill = 256 + rnd(w.B * w.Hq * w.nb * w.d * 4) + rnd(w.B * w.Hkv * w.nb * w.d * 4) \
        + rnd(w.B * w.Hq * w.nb * width * 4) + rnd(w.B * w.Hq * w.nb * 4)
    # decode: scores [B, Hq, nb], partial states [B, Hq, min(64, nb), d + 4], counters
    decode = 256 + rnd(w.B * w.Hq * w.nb * 4) + rnd(w.B * w.Hq * min(64, w.nb) * (w.d + 4) * 4) \
        + rnd(w.B * w.Hkv * -(-(w.Hq // w.Hkv) // 8) * 4)
    # backward: D and base-2 lse per query row, one bitmap of ceil(G * nb / 32) words per key block,
    # the pair lists (G (nb - j) int32 slots for key block j) and their lengths
    G = w.Hq // w.Hkv
    backward = 256 + 2 * rnd(w.B * w.Hq * w.N * 4) + rnd(w.B * w.Hkv * w.nb * -(-(G * w.nb) // 32) * 4) \
        + rnd(w.B * w.Hkv * G * (w.nb * (w.nb + 1) // 2) * 4) + rnd(w.B * w.Hkv * w.nb * 4)
    assert ws == max(prefill, decode, backward)


def status_of_forward(p, q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=None, idx=None, cnt=None, ws=FAKE,
                      ws_bytes=1 << 40):
    return B.raw("dsa_forward")(p.ref, q, k, v, out, lse, idx, cnt, ws, ws_bytes, None)


BASE = dict(B=1, Hq=4, Hkv=2, N=1024, d=64, block=64, k_free=4, local_window=1, n_sink=1)


@pytest.mark.parametrize("change,status", [
    (dict(Hq=3), B.DSA_ERR_INVALID_ARG),          # Hq % Hkv != 0
    (dict(Hkv=0), B.DSA_ERR_INVALID_ARG),
    (dict(B=-1), B.DSA_ERR_INVALID_ARG),
    (dict(k_free=-1), B.DSA_ERR_INVALID_ARG),
    (dict(local_window=-1), B.DSA_ERR_INVALID_ARG),
    (dict(n_sink=-2), B.DSA_ERR_INVALID_ARG),
    (dict(scale=-1.0), B.DSA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), B.DSA_ERR_INVALID_ARG),
    (dict(attn_kernel=7), B.DSA_ERR_INVALID_ARG),
    (dict(d=96), B.DSA_ERR_UNSUPPORTED),
    (dict(block=48), B.DSA_ERR_UNSUPPORTED),
    (dict(N=1000), B.DSA_ERR_UNSUPPORTED),         # N % block != 0
    (dict(N=32 * 1025, block=32), B.DSA_ERR_UNSUPPORTED),  # nb > 1024
])
def test_invalid_params_rejected_before_any_launch(change, status):
    p = B.Params(**(BASE | change))
    assert status_of_forward(p) == status
    n = ctypes.c_size_t(0)
    assert B.raw("dsa_workspace_size")(p.ref, ctypes.byref(n)) == status
    assert B.dsa_kmax(p) == 0


def test_attention_kernel_choice_query():
    # answers that do not depend on the driver: the warp-MMA kernel when asked
    # for, -1 for an invalid problem
    assert B.dsa_attn_uses_tcgen05(B.Params(**(BASE | dict(attn_kernel=B.DSA_ATTN_MMA_SYNC)))) == 0
    assert B.dsa_attn_uses_tcgen05(B.Params(**(BASE | dict(d=96)))) == -1
    assert B.dsa_attn_uses_tcgen05(B.Params(**(BASE | dict(attn_kernel=7)))) == -1
    assert B.raw("dsa_attn_uses_tcgen05")(None) == -1


def test_negative_per_head_budget_rejected():
    p = B.Params(**BASE, k_per_head=[1, 2, -1, 3])
    assert status_of_forward(p) == B.DSA_ERR_INVALID_ARG
    p = B.Params(**(BASE | dict(Hq=512, Hkv=2)), k_per_head=[1] * 512)
    assert status_of_forward(p) == B.DSA_ERR_UNSUPPORTED


def test_null_and_misaligned_pointers_rejected():
    p = B.Params(**BASE)
    assert status_of_forward(p, q=None) == B.DSA_ERR_INVALID_ARG
    assert status_of_forward(p, v=FAKE + 2) == B.DSA_ERR_INVALID_ARG
    assert status_of_forward(p, out=None) == B.DSA_ERR_INVALID_ARG
    assert status_of_forward(p, idx=FAKE, cnt=None) == B.DSA_ERR_INVALID_ARG
    f = B.raw("dsa_sparse_attn_fwd")
    assert f(p.ref, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, FAKE, 1 << 40, None) == B.DSA_ERR_INVALID_ARG
    f = B.raw("dsa_block_scores")
    assert f(p.ref, FAKE, FAKE, None, FAKE, 1 << 40, None) == B.DSA_ERR_INVALID_ARG
    f = B.raw("dsa_topk_select")
    assert f(p.ref, FAKE, None, FAKE, None) == B.DSA_ERR_INVALID_ARG
    assert B.raw("dsa_kmax")(None) == 0
    assert B.raw("dsa_forward")(None, FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, 1, None) \
        == B.DSA_ERR_INVALID_ARG


def test_workspace_checks():
    p = B.Params(**BASE)
    # the forward's own part: header, pooled Q and K, idx and cnt rows
    b, hq, hkv, n, d, bs = (BASE[x] for x in ("B", "Hq", "Hkv", "N", "d", "block"))
    nb, width = n // bs, B.dsa_kmax(p)
    rnd = lambda x: (x + 255) // 256 * 256
    need = 256 + rnd(b * hq * nb * d * 4) + rnd(b * hkv * nb * d * 4) + rnd(b * hq * nb * width * 4) \
        + rnd(b * hq * nb * 4)
    assert need <= B.dsa_workspace_size(p)
    assert status_of_forward(p, ws=None) == B.DSA_ERR_WORKSPACE
    assert status_of_forward(p, ws_bytes=need - 1) == B.DSA_ERR_WORKSPACE
    assert status_of_forward(p, ws=FAKE + 8) == B.DSA_ERR_WORKSPACE
    assert B.raw("dsa_workspace_init")(None, 256, None) == B.DSA_ERR_WORKSPACE
    assert B.raw("dsa_workspace_init")(FAKE, 100, None) == B.DSA_ERR_WORKSPACE
    assert B.raw("dsa_check_status")(None, None) == B.DSA_ERR_WORKSPACE


def test_empty_problems_return_ok_without_touching_pointers():
    for change in (dict(B=0), dict(N=0)):
        p = B.Params(**(BASE | change))
        assert status_of_forward(p, q=None, k=None, v=None, out=None, ws=None) == B.DSA_OK
        assert B.dsa_workspace_size(p) == 256
        assert B.dsa_kmax(p) == 0


def test_select_mode_checks():
    base = dict(B=1, Hq=8, Hkv=2, N=1024, d=64, block=64, k_free=4, local_window=1, n_sink=1)
    assert status_of_forward(B.Params(**base, select_mode=7)) == B.DSA_ERR_INVALID_ARG
    assert status_of_forward(B.Params(**base, select_mode=-1)) == B.DSA_ERR_INVALID_ARG
    assert status_of_forward(B.Params(**base, select_tau=0.5)) == B.DSA_ERR_INVALID_ARG
    # the group rule shares one budget per KV head
    assert status_of_forward(B.Params(**base, k_per_head=[1] * 8, select_mode=B.DSA_SELECT_GROUP_TOPK)) \
        == B.DSA_ERR_INVALID_ARG
    big = dict(base, Hq=66, Hkv=1)
    assert status_of_forward(B.Params(**big, select_mode=B.DSA_SELECT_GROUP_TOPK)) == B.DSA_ERR_UNSUPPORTED
    # the threshold rule needs 0 < tau <= 1
    for tau in (0.0, -0.1, 1.5, float("nan")):
        assert status_of_forward(B.Params(**base, select_mode=B.DSA_SELECT_THRESHOLD, select_tau=tau)) \
            == B.DSA_ERR_INVALID_ARG
    thr = B.Params(**base, select_mode=B.DSA_SELECT_THRESHOLD, select_tau=0.05)
    assert B.dsa_kmax(thr) == B.dsa_kmax(B.Params(**base))
    ok = B.Params(**base, select_mode=B.DSA_SELECT_GROUP_TOPK)
    assert B.dsa_kmax(ok) == B.dsa_kmax(B.Params(**base))
    assert B.dsa_workspace_size(ok) == B.dsa_workspace_size(B.Params(**base))


def test_decode_argument_checks():
    p = B.Params(B=1, Hq=4, Hkv=2, N=1024, d=64, block=64, k_free=4, local_window=1, n_sink=1)
    dec = B.raw("dsa_decode_fwd")
    call = lambda length, q=FAKE, kp=FAKE, out=FAKE, idx=None, cnt=None, ws=FAKE, ws_bytes=256: \
        dec(p.ref, q, FAKE, FAKE, kp, length, out, None, idx, cnt, ws, ws_bytes, None)
    assert call(0) == B.DSA_ERR_INVALID_ARG
    assert call(1025) == B.DSA_ERR_INVALID_ARG
    assert call(10, q=None) == B.DSA_ERR_INVALID_ARG
    assert call(10, kp=FAKE + 4) == B.DSA_ERR_INVALID_ARG
    assert call(10, out=None) == B.DSA_ERR_INVALID_ARG
    assert call(10, idx=FAKE) == B.DSA_ERR_INVALID_ARG  # idx without cnt
    assert call(10, ws=None) == B.DSA_ERR_WORKSPACE
    assert call(10, ws_bytes=255) == B.DSA_ERR_WORKSPACE
    # the decode's own workspace: header, scores [1, 4, 16], partial states [1, 4, 16, 68], counters
    need = 256 + 256 + 4 * 16 * 68 * 4 + 256
    assert need <= B.dsa_workspace_size(p)
    assert call(10, ws_bytes=need - 1) == B.DSA_ERR_WORKSPACE
    pool = B.raw("dsa_pool_keys")
    assert pool(p.ref, FAKE, FAKE, -1, 3, None) == B.DSA_ERR_INVALID_ARG
    assert pool(p.ref, FAKE, FAKE, 4, 3, None) == B.DSA_ERR_INVALID_ARG
    assert pool(p.ref, FAKE, FAKE, 0, 17, None) == B.DSA_ERR_INVALID_ARG
    assert pool(p.ref, FAKE, FAKE, 3, 3, None) == B.DSA_OK  # empty range: nothing to do
    assert pool(p.ref, None, FAKE, 0, 2, None) == B.DSA_ERR_INVALID_ARG


def test_backward_argument_checks():
    p = B.Params(B=1, Hq=4, Hkv=2, N=1024, d=64, block=64, k_free=4, local_window=1, n_sink=1)
    bwd = B.raw("dsa_sparse_attn_bwd")

    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, dout=FAKE, idx=FAKE, cnt=FAKE, dq=FAKE,
                 dk=FAKE, dv=FAKE, ws=FAKE, ws_bytes=1 << 40)
        a.update(kw)
        return bwd(p.ref, a["q"], a["k"], a["v"], a["out"], a["lse"], a["dout"], a["idx"], a["cnt"],
                   a["dq"], a["dk"], a["dv"], a["ws"], a["ws_bytes"], None)

    for name in ("q", "k", "v", "out", "lse", "dout", "idx", "cnt", "dq", "dk", "dv"):
        assert call(**{name: None}) == B.DSA_ERR_INVALID_ARG, name
    assert call(dq=FAKE + 8) == B.DSA_ERR_INVALID_ARG  # misaligned
    assert call(ws=None) == B.DSA_ERR_WORKSPACE
    # D and lse2 [1, 4, 1024] fp32, then 2 x 16 bitmaps of ceil(2 * 16 / 32) = 1 word
    need = 256 + 2 * 16384 + 256
    assert need <= B.dsa_workspace_size(p)
    assert call(ws_bytes=need - 1) == B.DSA_ERR_WORKSPACE
