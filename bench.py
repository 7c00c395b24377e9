#!/usr/bin/env python
"""Benchmark of the block-sparse attention prefill path on B200.

One step = one pass of the whole path over the 32K workload (B=1, 32 query /
8 KV heads, d=128, 32768 tokens, 64x64 blocks, 64 free picks + 2-block
window + 1 sink): pool and score the blocks, select them, attend over the
kept blocks. The step calls dsa_select_blocks then dsa_sparse_attn_fwd, which
issue the same three kernels as dsa_forward, so that the attention kernel's
own duration can be read with CUDA events inside the timed region.

Prints ONE JSON line (rank 0). ``--impl reference`` times the fp64 CPU oracle
instead, on bounded samples of the same workload.

Multi-GPU (torchrun): every rank runs its own independent problem of the same
shape (weak scaling, no data-path collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from dynamic_block_sparse_02_b200 import WORKLOADS  # noqa: E402
from dynamic_block_sparse_02_b200 import workloads as W  # noqa: E402

METRIC = "sparse-attn prefill tokens/s at 32K; effective TFLOP/s vs bf16 tensor peak"
DEFAULT_WORKLOAD = "32k-gqa"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ATTN_SOURCES = ("attn_tc.cu",)  # the kernel whose DRAM traffic profiles/attn_traffic.json records
SELECT_MODES = {"topk": 0, "group": 1, "threshold": 2}


# ---------------------------------------------------------------------------
# host-side helpers (also used by the multi-process CPU tests)
# ---------------------------------------------------------------------------

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_seed(rank: int) -> int:
    """Each rank draws its own independent problem."""
    return 1000 + rank


def reduce_max(x: float, device=None) -> float:
    """Max of a scalar over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(tokens_per_rank_step: int, world: int, steps: int, max_ms: float) -> float:
    return tokens_per_rank_step * world * steps / (max_ms / 1e3)


# 148 SMs x 128 fp32 lanes x 2 FLOP per FMA x 1965 MHz (the part's maximum SM clock)
FP32_FMA_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def kept_flops(cnt_sum: int, block: int, d: int) -> float:
    """Algorithmic FLOPs of the attention step: 4 * bs^2 * d per kept block
    (Q K^T and P V, full tiles, diagonal tile counted in full)."""
    return 4.0 * block * block * d * cnt_sum


def select_bytes(w) -> float:
    """Algorithmic HBM bytes of steps 1-3: Q and K read once, index rows and
    counts written. Intermediates (pooled blocks, scores) are not counted."""
    q = w.B * w.Hq * w.N * w.d * 2
    k = w.B * w.Hkv * w.N * w.d * 2
    width = min(w.nb, w.k_free + w.local_window + w.n_sink)
    sel = w.B * w.Hq * w.nb * (width + 1) * 4
    return q + k + sel


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def attn_source_sha() -> str:
    h = hashlib.sha256()
    for name in ATTN_SOURCES:
        p = os.path.join(ROOT, "dynamic_block_sparse_02_b200", "csrc", name)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def recorded_decode_traffic(workload: str, select_mode: str):
    """DRAM bytes of one decode step (both kernels) from the committed ncu
    summary, or None when csrc/decode.cu has changed since it was captured."""
    try:
        with open(os.path.join(ROOT, "profiles", "decode_traffic.json")) as f:
            rec = json.load(f)
        src = os.path.join(ROOT, "dynamic_block_sparse_02_b200", "csrc", "decode.cu")
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except Exception:
        return None
    if rec.get("source_sha") != sha or rec.get("workload") != workload or rec.get("select_mode") != select_mode:
        return None
    return rec.get("dram_bytes_per_step")


def recorded_traffic(workload: str):
    """DRAM bytes per attention launch from the committed ncu summary, or None
    when the attention kernel's source has changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "attn_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("source_sha") != attn_source_sha() or rec.get("workload") != workload:
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self._t is not None:
            self._t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# CPU baseline: the oracle on a bounded sample of the workload
# ---------------------------------------------------------------------------

def oracle_sample(w, x, kph, budget_s: float, seed: int = 0, workers=None):
    """Time the oracle on a bounded sample on the host cores.

    Returns (estimated seconds per full step, description, wall seconds spent,
    cores used). All host cores run oracle workers (one BLAS thread each):
    pooling, scores and selection of every (batch, KV head) group are timed in
    full, one group per task; then attention runs over rounds of seeded random
    query blocks until ``budget_s`` seconds have passed, and its time is
    scaled by (kept blocks of the workload) / (kept blocks processed).
    """
    from oracle.parallel import OraclePool
    width = min(w.nb, (max(kph) if kph is not None else w.k_free) + w.local_window + w.n_sink)
    k = kph if kph is not None else w.k_free
    with OraclePool(dict(q=x["q"], k=x["k"], v=x["v"]), workers=workers) as pool:
        t0 = time.perf_counter()
        idx, cnt = pool.select(w.B, w.Hkv, w.group, w.block, k, w.local_window, w.n_sink, width)
        t_sel = time.perf_counter() - t0
        pool.put("idx", idx)
        pool.put("cnt", cnt)
        rng = np.random.default_rng(seed)
        order = [(b, h, i) for b in range(w.B) for h in range(w.Hq) for i in range(w.nb)]
        rng.shuffle(order)
        per_round = 2 * pool.workers
        done, blocks, t_att = 0, 0, 0.0
        while done < len(order) and t_att < budget_s:
            chunk = order[done:done + per_round]
            t_att += pool.timed_attention(chunk, w.block)
            blocks += int(sum(cnt[it] for it in chunk))
            done += len(chunk)
        cores = pool.workers
    total_blocks = float(cnt.sum())
    est = t_sel + t_att * total_blocks / max(blocks, 1)
    desc = (f"{w.name}: pooling/scores/selection of all {w.B * w.Hkv} (batch, KV head) groups timed "
            f"in full ({t_sel:.1f} s); attention on {done} seeded random query blocks ({blocks} kept "
            f"key blocks, {t_att:.1f} s) scaled to all {int(total_blocks)} kept blocks; "
            f"{cores} worker processes, one BLAS thread each")
    return est, desc, t_sel + t_att, cores


def run_reference(args, w):
    """The --impl reference arm: the oracle as it stands, on host cores.

    Each step is a bounded sample of the workload (see oracle_sample);
    ms_per_step is that sample's measured wall time, and value is the
    workload's tokens divided by the full step time extrapolated from it.
    """
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    kph = W.per_head_k(w)
    kph = None if kph is None else [int(t) for t in kph]
    x = W.make_inputs(w, seed=rank_seed(0))
    for _ in range(args.warmup):
        oracle_sample(w, x, kph, budget_s=min(1.0, args.ref_budget))
    ests, walls, desc, cores = [], [], "", 1
    for s in range(args.steps):
        est, desc, wall, cores = oracle_sample(w, x, kph, budget_s=args.ref_budget, seed=s)
        ests.append(est)
        walls.append(wall)
    est = statistics.median(ests)
    tokens = w.B * w.N
    value = tokens / est
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(walls) * 1e3,
        "ms_per_full_step_extrapolated": est * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(w),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


L2_BYTES = 126 << 20          # B200 L2
FLUSH_BYTES = 256 << 20       # written between timed steps when the inputs fit in L2


def input_bytes(w) -> int:
    return w.B * (w.Hq + 2 * w.Hkv) * w.N * w.d * 2


def needs_flush(w) -> bool:
    """Inputs below twice the L2 size would partly stay in L2 from one step to the next."""
    return input_bytes(w) < 2 * L2_BYTES


def config_dict(w):
    mb = input_bytes(w) / 1e6
    l2 = ("L2 flushed before every timed step (%d MB written; Q+K+V = %.1f MB); "
          "ms_per_step sums the steps' own event times" % (FLUSH_BYTES >> 20, mb)
          if needs_flush(w) else "inputs larger than L2: Q+K+V = %.0f MB per step > 126 MB" % mb)
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
            "block": w.block, "k_free": w.k_free, "local_window": w.local_window,
            "n_sink": w.n_sink, "l2": l2}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_ours(args, w):
    import torch
    import torch.distributed as dist
    from dynamic_block_sparse_02_b200 import binding as B
    from dynamic_block_sparse_02_b200.attention import BlockSparseAttention

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    kph = W.per_head_k(w)
    kph = None if kph is None else [int(t) for t in kph]
    x = W.make_inputs(w, seed=rank_seed(rank))
    to_t = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    q_h, k_h, v_h = (to_t(x[n]).pin_memory() for n in ("q", "k", "v"))
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    stream = torch.cuda.Stream(device=dev)
    att = BlockSparseAttention.from_workload(w, k_per_head=kph, device=dev, stream=stream,
                                             attn_kernel=args.attn_kernel,
                                             select_mode=SELECT_MODES[args.select_mode],
                                             select_tau=args.tau if args.select_mode == "threshold" else 0.0)
    idx, cnt = att.empty_selection()
    out = att.empty_out()

    def select():
        B.dsa_select_blocks(att.params, q, k, idx, cnt, att.ws, att.ws_bytes, stream)

    def attend():
        B.dsa_sparse_attn_fwd(att.params, q, k, v, idx, cnt, out, None, att.ws, att.ws_bytes, stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            select()
            attend()
    torch.cuda.synchronize(dev)
    status = B.dsa_check_status(att.ws, stream)
    if status != B.DSA_OK:
        raise RuntimeError("device error during warm-up: " + B.status_string(status))
    kept = int(cnt.sum().item())
    # rows whose kept list holds their own (diagonal) block
    diag = int((idx == torch.arange(w.nb, device=dev, dtype=idx.dtype).view(1, 1, -1, 1)).any(-1).sum().item())

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    sampler = ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else 0)
    if rank == 0 and not args.no_clocks:
        sampler.start()
    if world > 1:
        dist.barrier()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if needs_flush(w) else None
    torch.cuda.synchronize(dev)
    torch.cuda.nvtx.range_push("timed steps")
    with torch.cuda.stream(stream):
        for s in range(K):
            if flush is not None:
                flush.fill_(s & 0xff)
            ev[s][0].record(stream)
            select()
            ev[s][1].record(stream)
            attend()
            ev[s][2].record(stream)
    torch.cuda.synchronize(dev)
    torch.cuda.nvtx.range_pop()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if rank == 0 else None
    status = B.dsa_check_status(att.ws, stream)
    if status != B.DSA_OK:
        raise RuntimeError("device error during timing: " + B.status_string(status))

    if flush is None:
        total_ms = ev[0][0].elapsed_time(ev[-1][2])
    else:  # the flushes between steps are not part of the steps
        total_ms = sum(e[0].elapsed_time(e[2]) for e in ev)
    sel_ms = [e[0].elapsed_time(e[1]) for e in ev]
    att_ms = [e[1].elapsed_time(e[2]) for e in ev]
    max_total = reduce_max(total_ms, dev)
    tokens = w.B * w.N
    value = whole_job_tokens_per_s(tokens, world, K, max_total)

    # End to end through the public call, with host buffers: every step copies
    # its Q, K, V from pinned host memory and its output back, inside the timed
    # region. The copies run on their own streams (one per direction) into
    # double-buffered device tensors, so step s's input copy overlaps step
    # s-1's computation and its output copy overlaps step s+1's.
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    Ke = max(3, min(K, args.e2e_steps))
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    qb, kb, vb = [q, torch.empty_like(q)], [k, torch.empty_like(k)], [v, torch.empty_like(v)]
    ob = [out, torch.empty_like(out)]

    def e2e_run(nsteps, e_start=None, e_end=None):
        computed, out_done = [None, None], [None, None]
        if e_start is not None:
            e_start.record(s_in)
            stream.wait_event(e_start)
            s_out.wait_event(e_start)
        for st in range(nsteps):
            x2 = st % 2
            with torch.cuda.stream(s_in):
                if computed[x2] is not None:
                    s_in.wait_event(computed[x2])  # step st-2 has read buffer x2
                qb[x2].copy_(q_h, non_blocking=True)
                kb[x2].copy_(k_h, non_blocking=True)
                vb[x2].copy_(v_h, non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(s_in)
            stream.wait_event(ready)
            if out_done[x2] is not None:
                stream.wait_event(out_done[x2])  # step st-2's output has left ob[x2]
            att.forward(qb[x2], kb[x2], vb[x2], ob[x2])  # on the attention's own stream
            done = torch.cuda.Event()
            done.record(stream)
            computed[x2] = done
            with torch.cuda.stream(s_out):
                s_out.wait_event(done)
                out_h.copy_(ob[x2], non_blocking=True)
                moved = torch.cuda.Event()
                moved.record(s_out)
                out_done[x2] = moved
        if e_end is not None:
            s_out.wait_event(computed[(nsteps - 1) % 2])
            e_end.record(s_out)

    e2e_run(2)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(Ke, e0, e1)
    torch.cuda.synchronize(dev)
    e2e_ms = reduce_max(e0.elapsed_time(e1), dev)
    e2e_value = whole_job_tokens_per_s(tokens, world, Ke, e2e_ms)
    status = B.dsa_check_status(att.ws, stream)
    if status != B.DSA_OK:
        raise RuntimeError("device error in the end-to-end loop: " + B.status_string(status))

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_kind = load_peaks()
    uses_tc = B.dsa_attn_uses_tcgen05(att.params)  # the kernel step 4 ran
    att_avg = statistics.mean(att_ms)
    sel_avg = statistics.mean(sel_ms)
    flops = kept_flops(kept, w.block, w.d)
    achieved = flops / (att_avg / 1e3) / 1e12
    # the attention kernel runs as millisecond launches: the burst peak applies
    peak = float(peaks["bf16_tflops"])
    sel_gbs = select_bytes(w) / (sel_avg / 1e3) / 1e9
    score_flop = 2.0 * w.d * w.B * w.Hq * w.nb * (w.nb + 1) / 2
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        est, desc, spent, cores = oracle_sample(w, x, kph, budget_s=args.cpu_budget)
        cpu = {"value": tokens / est, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": desc + f" ({spent:.1f} s wall)"}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": max_total / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_dict(w),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "traffic": recorded_traffic(w.name) if uses_tc == 1 else None,
                     "kernel": "sparse attention (dsa_sparse_attn_fwd)",
                     "peak_kind": f"{peak_kind} bf16 dense, burst",
                     "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained",
                                                                     peaks["bf16_tflops"]))},
        "select": {"ms": sel_avg, "algorithmic_bytes": select_bytes(w), "GBps": sel_gbs,
                   "frac_hbm": sel_gbs / float(peaks["hbm_gbs"]), "bound": "hbm",
                   "frac_spec_8tbs": sel_gbs / 8000.0,
                   # the fp32 block-score products (j <= i) against the nominal fp32 FMA rate
                   "score_gflop": score_flop / 1e9,
                   "score_tflops_at_select_time": score_flop / (sel_avg / 1e3) / 1e12,
                   "fp32_fma_peak_tflops_nominal": FP32_FMA_PEAK_TFLOPS},
        "attention_ms": att_avg,
        "attention_tokens_per_s": tokens * world / (att_avg / 1e3),
        "effective_tflops_diag_half": kept_flops(1, w.block, w.d) * (kept - 0.5 * diag) / (att_avg / 1e3) / 1e12,
        "kept_blocks_per_step": kept,
        "effective_tflops": achieved,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": int(q_h.numel() + k_h.numel() + v_h.numel()) * 2,
                "d2h_bytes_per_step": int(out_h.numel()) * 2,
                "overlap": "copies on one stream per direction, double-buffered, overlapping "
                           "the neighbouring steps' computation"},
        "gpu_launches": 3 * K,
        "clocks": clocks,
        "attn_kernel": {0: "auto", 1: "tcgen05", 2: "mma.sync"}[args.attn_kernel]
                       + {1: " (tcgen05)", 0: " (mma.sync)"}.get(uses_tc, "") * (args.attn_kernel == 0),
    }
    if args.select_mode != "topk":
        line["config"]["select_mode"] = args.select_mode
        if args.select_mode == "threshold":
            line["config"]["tau"] = args.tau
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# Decode step (one query token per sequence against a full KV cache)
# ---------------------------------------------------------------------------

DECODE_METRIC = "sparse-attn decode tokens/s at 32K context (one token per sequence per step)"


def decode_bytes(w, idx, cnt, length) -> float:
    """Algorithmic HBM bytes of one decode step: the present keys and values of
    the union of kept blocks of each KV head's query heads, the pooled key rows
    of the complete blocks (once per KV head), the query and the output."""
    total = 0
    i = (length - 1) // w.block
    for b in range(w.B):
        for g in range(w.Hkv):
            blocks = set()
            for h in range(g * w.group, (g + 1) * w.group):
                blocks.update(int(j) for j in idx[b, h, :cnt[b, h]])
            keys = sum(min((j + 1) * w.block, length) - j * w.block for j in blocks)
            total += keys * w.d * 2 * 2 + i * w.d * 4
    total += 2 * w.B * w.Hq * w.d * 2
    return float(total)


def run_decode(args, w):
    import torch
    from dynamic_block_sparse_02_b200.attention import BlockSparseAttention

    rank, world, local = dist_env()
    if rank != 0:
        return 0  # a single-GPU measurement: under torchrun rank 0 runs it alone
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    length = w.N
    x = W.make_inputs(w, seed=rank_seed(rank))
    to_t = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    qtok_h = np.ascontiguousarray(x["q"][:, :, length - 1, :])
    q = to_t(qtok_h).to(dev)
    kc, vc = to_t(x["k"]).to(dev), to_t(x["v"]).to(dev)
    stream = torch.cuda.Stream(device=dev)
    att = BlockSparseAttention.from_workload(w, device=dev, stream=stream,
                                             select_mode=SELECT_MODES[args.select_mode],
                                             select_tau=args.tau if args.select_mode == "threshold" else 0.0)
    kp = att.pooled_key_cache()
    idx = torch.empty((w.B, w.Hq, att.width), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.B, w.Hq), dtype=torch.int32, device=dev)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # larger than L2
    clean = torch.ones(256 << 20, dtype=torch.uint8, device=dev)   # read after the flush
    with torch.cuda.stream(stream):
        att.pool_keys(kc, kp, 0, (length - 1) // w.block)
        for _ in range(args.warmup):
            att.decode(q, kc, vc, kp, length, out, None, idx, cnt)
    torch.cuda.synchronize(dev)
    from dynamic_block_sparse_02_b200 import binding as B
    status = B.dsa_check_status(att.ws, stream)
    if status != B.DSA_OK:
        raise RuntimeError("device error during warm-up: " + B.status_string(status))
    # Each timed step starts from a cold L2: a 256 MB write (the flush), then a
    # 256 MB read, which evicts the flush's dirty lines so that the step's reads
    # do not pay for their write-back. The write-only flush is timed too.
    def timed(read_after):
        ms = []
        for _ in range(args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                flush.fill_(1)
                if read_after:
                    clean.max()
                e0.record(stream)
                att.decode(q, kc, vc, kp, length, out, None, idx, cnt)
                e1.record(stream)
            torch.cuda.synchronize(dev)
            ms.append(e0.elapsed_time(e1))
        return statistics.median(ms)

    sampler = ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else 0)
    if not args.no_clocks:
        sampler.start()
    step_ms = timed(True)
    clocks = sampler.stop()
    dirty_ms = timed(False)
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    nbytes = decode_bytes(w, idx_h, cnt_h, length)
    peaks, peak_kind = load_peaks()
    gbs = nbytes / (step_ms / 1e3) / 1e9
    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        from threadpoolctl import threadpool_limits
        with threadpool_limits(1):  # one core: the step is one row per head
            t0 = time.perf_counter()
            steps = 0
            while True:  # whole decode steps until about cpu_budget seconds of CPU work
                oracle.decode(qtok_h, x["k"], x["v"], length, w.block, w.k_free, w.local_window, w.n_sink,
                              mode=args.select_mode, tau=args.tau if args.select_mode == "threshold" else 0.0)
                steps += 1
                if time.perf_counter() - t0 >= args.cpu_budget or steps >= 200:
                    break
            spent = time.perf_counter() - t0
        cpu = {"value": steps * w.B / spent, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": f"{steps} full decode steps on one core, BLAS on one thread ({spent:.1f} s)"}
    cfg = config_dict(w)
    cfg["l2"] = ("L2 flushed before every timed step: 256 MB write, then 256 MB read "
                 "(clean cold L2); ms_per_step_dirty_l2 = the same after the write alone")
    cfg.update({"context": length, "select_mode": args.select_mode})
    line = {
        "metric": DECODE_METRIC, "value": w.B / (step_ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                     "frac": gbs / float(peaks["hbm_gbs"]),
                     "traffic": recorded_decode_traffic(w.name, args.select_mode),
                     "kernel": "decode (dsa_decode_fwd)", "peak_kind": f"{peak_kind} copy bandwidth",
                     "algorithmic_bytes": nbytes},
        "cpu_baseline": cpu,
        "ms_per_step_dirty_l2": dirty_ms,
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


BACKWARD_METRIC = "sparse-attn backward tokens/s at 32K (dQ, dK, dV over the kept blocks)"


def backward_flops(cnt_sum: int, block: int, d: int) -> float:
    """Algorithmic FLOPs of the backward: 10 * bs^2 * d per kept block (the five
    products S = Q K^T, dP = dO V^T, dV = P^T dO, dK = dS^T Q, dQ = dS K over
    full tiles). The kernels recompute S and dP in both the dQ and the dK/dV
    pass; that recomputation is not counted."""
    return 10.0 * block * block * d * cnt_sum


def run_backward(args, w):
    import torch
    from dynamic_block_sparse_02_b200 import binding as B
    from dynamic_block_sparse_02_b200.attention import BlockSparseAttention

    rank, world, local = dist_env()
    if rank != 0:
        return 0  # a single-GPU measurement: under torchrun rank 0 runs it alone
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    x = W.make_inputs(w, seed=rank_seed(rank))
    g = np.random.default_rng(1000 + rank)
    do_h = W.f32_to_bf16_bits(g.standard_normal(x["q"].shape).astype(np.float32))
    to_t = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    q, k, v, dout = (to_t(a).to(dev) for a in (x["q"], x["k"], x["v"], do_h))
    stream = torch.cuda.Stream(device=dev)
    att = BlockSparseAttention.from_workload(w, attn_kernel=args.attn_kernel, device=dev, stream=stream)
    idx, cnt = att.empty_selection()
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    # the tcgen05 backward (64x64 blocks, unless the warp-MMA kernel is asked
    # for) launches prep, colbits, pairs, dQ and dK/dV; the warp-MMA path prep,
    # colbits, dQ and dK/dV
    tc_bwd = w.block == 64 and args.attn_kernel != 2
    with torch.cuda.stream(stream):
        att.forward(q, k, v, out, lse, idx, cnt)  # the selection and forward the backward follows
        for _ in range(args.warmup):
            att.sparse_attn_backward(q, k, v, out, lse, dout, idx, cnt, dq, dk, dv)
    torch.cuda.synchronize(dev)
    status = B.dsa_check_status(att.ws, stream)
    if status != B.DSA_OK:
        raise RuntimeError("device error during warm-up: " + B.status_string(status))
    kept = int(cnt.sum().item())
    sampler = ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else 0)
    if not args.no_clocks:
        sampler.start()
    ms = []
    for _ in range(args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            att.sparse_attn_backward(q, k, v, out, lse, dout, idx, cnt, dq, dk, dv)
            e1.record(stream)
        torch.cuda.synchronize(dev)
        ms.append(e0.elapsed_time(e1))
    clocks = sampler.stop()
    step_ms = statistics.median(ms)
    peaks, peak_kind = load_peaks()
    flops = backward_flops(kept, w.block, w.d)
    tfs = flops / (step_ms / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"])  # millisecond launches: the burst peak applies
    cpu = None
    if not args.no_cpu_baseline:
        from oracle.parallel import OraclePool
        idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
        items = [(0, h, i) for h in range(w.Hq) for i in range(w.nb - 1, -1, -97)][:args.bwd_sample]
        with OraclePool(dict(q=x["q"], k=x["k"], v=x["v"], dout=do_h, idx=idx_h, cnt=cnt_h)) as pool:
            t0 = time.perf_counter()
            pool.backward(items, w.block)
            spent = time.perf_counter() - t0
            cores = pool.workers
        share = float(sum(cnt_h[it] for it in items)) / float(cnt_h.sum())
        cpu = {"value": w.B * w.N * share / spent, "unit": "tokens/s", "cores": cores,
               "kind": "oracle",
               "sample": f"{len(items)} query blocks of the workload ({share:.3%} of its kept blocks, "
                         f"{spent:.1f} s wall on {cores} worker processes), scaled by kept blocks"}
    cfg = config_dict(w)
    cfg["l2"] = "inputs larger than L2 (q, dout, out 268 MB each), no flush"
    cfg["selection"] = "the forward's own top-k lists"
    line = {
        "metric": BACKWARD_METRIC, "value": w.B * w.N / (step_ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
        "roofline": {"bound": "tensor", "achieved": tfs, "peak": peak, "unit": "TFLOP/s", "frac": tfs / peak,
                     "traffic": None,
                     "kernel": "backward step (prep, colbits, pairs, dQ and dK/dV passes on tcgen05)" if tc_bwd
                     else "backward step (prep, colbits, dQ and dK/dV on mma.sync)",
                     "peak_kind": f"{peak_kind} bf16 dense, burst", "algorithmic_flops": flops,
                     "frac_of_sustained": tfs / float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))},
        "kept_blocks": kept,
        "cpu_baseline": cpu,
        "gpu_launches": (5 if tc_bwd else 4) * args.steps,
        "attn_kernel": {0: "auto", 1: "tcgen05", 2: "mma.sync"}[args.attn_kernel],
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--attn-kernel", type=int, default=0, choices=[0, 1, 2])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--select-mode", choices=sorted(SELECT_MODES), default="topk",
                    help="selection rule (default: per-head top-k)")
    ap.add_argument("--tau", type=float, default=0.05, help="threshold of --select-mode threshold")
    ap.add_argument("--decode", action="store_true",
                    help="time one decode step against a full KV cache instead of the prefill step")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward over the kept blocks instead of the prefill step")
    ap.add_argument("--bwd-sample", type=int, default=1024, help="query blocks in the oracle's timed sample")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.decode:
        return run_decode(args, w)
    if args.backward:
        return run_backward(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
