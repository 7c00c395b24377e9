"""Host-side accounting of bench.py, checked against counts written out by
hand: the algorithmic bytes of the decode step and of the selection, and the
algorithmic FLOPs of the backward."""
import numpy as np

import bench
from dynamic_block_sparse_02_b200 import Workload


def test_decode_bytes_counts_the_union_of_kept_blocks_per_kv_head():
    # B=1, 4 query heads over 2 KV heads, block 4, d 8, 5 blocks, length 18:
    # the token's block i = 17 // 4 = 4 holds 2 present keys (16, 17)
    w = Workload("t", 1, 4, 2, 20, 8, 4, k_free=1, local_window=1, n_sink=0)
    idx = np.full((1, 4, 3), -1, dtype=np.int32)
    cnt = np.zeros((1, 4), dtype=np.int32)
    idx[0, 0, :2], cnt[0, 0] = [1, 4], 2      # KV head 0: heads 0 and 1
    idx[0, 1, :2], cnt[0, 1] = [2, 4], 2
    idx[0, 2, :2], cnt[0, 2] = [0, 4], 2      # KV head 1: heads 2 and 3
    idx[0, 3, :2], cnt[0, 3] = [0, 4], 2
    got = bench.decode_bytes(w, idx, cnt, 18)
    # KV head 0 keys: blocks {1, 2} full (8 keys) + block 4 partial (2) = 10;
    # KV head 1: block 0 (4) + block 4 (2) = 6; K and V, bf16
    kv = (10 + 6) * 8 * 2 * 2
    pooled = 2 * 4 * 8 * 4       # complete blocks j < 4, fp32, once per KV head
    qo = 2 * 4 * 8 * 2           # query in, output out, bf16
    assert got == kv + pooled + qo


def test_backward_flops_are_five_products_per_kept_block():
    assert bench.backward_flops(3, 64, 128) == 3 * 5 * 2 * 64 * 64 * 128


def test_select_bytes_reads_q_and_k_once_and_writes_the_lists():
    w = Workload("t", 2, 4, 2, 256, 64, 32, k_free=3, local_window=1, n_sink=1)
    width = min(8, 3 + 1 + 1)
    expect = 2 * 4 * 256 * 64 * 2 + 2 * 2 * 256 * 64 * 2 + 2 * 4 * 8 * (width + 1) * 4
    assert bench.select_bytes(w) == expect


def test_single_gpu_modes_leave_other_ranks_idle(monkeypatch, capsys):
    # under torchrun the decode and backward measurements run on rank 0 alone
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--decode", "--steps", "1", "--warmup", "3"]) == 0
    assert bench.main(["--backward", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out == ""
