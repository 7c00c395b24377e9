"""Synthetic workloads: named shapes and seeded bf16 input generators.

This module holds no part of the attention method's arithmetic. It only
describes problem shapes and selection settings, and draws the seeded Q/K/V
tensors that both the CUDA path and the fp64 oracle consume.

Inputs are bf16 bit patterns (numpy ``uint16``), produced by drawing float32
samples from numpy's PCG64 generator and rounding them to bf16 with
round-to-nearest-even. The pages name only sequence lengths for their
workloads (2k/8k in "Sparse attention vs Flash Attention v2", section 2.1; 32k
in the "DeepSeek NSA" article, section 5; 128K in the zyentor.com forum
thread); their datasets (CNN/DailyMail, PG-19, QASPER, ...) are not available,
so these N(0,1) tensors stand in for them.
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Dict, Optional, Tuple

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    """One problem shape plus its block-selection settings.

    Field names follow the C-ABI's ``dsa_params`` struct.
    """

    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    block: int
    k_free: int                 # top-k picks beyond the forced set (all heads)
    local_window: int           # forced blocks {i-w+1 .. i}
    n_sink: int                 # forced blocks {0 .. n_sink-1}
    k_choices: Optional[Tuple[int, ...]] = None  # per-head k drawn from these
    structured_keys: bool = False  # add a shared unit direction to 5% of key blocks
    scale: float = 0.0          # 0 -> 1/sqrt(d)

    @property
    def nb(self) -> int:
        return self.N // self.block

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five synthetic configurations. Sizes and selection settings follow the
# block-sparse passages: 64x64 tiles decided per block (zblog.xzdbk.com,
# "hardware-friendly sparse computation"), 32x32 tiles with a light per-block
# activation estimate ("DeepSeek NSA", section 2.1), 128x128 tiles
# ("engineering advice" list of the same zblog page), and top-k with a local
# window plus global tokens (zblog, "Top-k local-global hybrid").
WORKLOADS: Dict[str, Workload] = {
    # B=1, 2 heads (MHA), d=64, 512 tokens, 64x64 blocks, top-k = 4 blocks
    # including the forced diagonal -> 3 free picks.
    "tiny": Workload("tiny", 1, 2, 2, 512, 64, 64, k_free=3, local_window=1, n_sink=0),
    # Llama-8B-shaped prefill: 32 query / 8 KV heads, d=128, 8K tokens,
    # 16 free picks + diagonal + block 0 as sink.
    "8k-gqa": Workload("8k-gqa", 1, 32, 8, 8192, 128, 64, k_free=16, local_window=1, n_sink=1),
    # 32K prefill: 64 free picks + 2-block local window {i-1, i} + sink block 0.
    "32k-gqa": Workload("32k-gqa", 1, 32, 8, 32768, 128, 64, k_free=64, local_window=2, n_sink=1),
    # 128K with structured keys, 128x128 blocks, 64 free picks + diagonal.
    "128k-structured": Workload("128k-structured", 1, 32, 8, 131072, 128, 128, k_free=64,
                                local_window=1, n_sink=0, structured_keys=True),
    # Batched fine-grained: B=4, 16 heads (MHA), d=64, 16K tokens, 32x32
    # blocks, per-head k from {8,16,32,64} + diagonal.
    "batched-32": Workload("batched-32", 4, 16, 16, 16384, 64, 32, k_free=64, local_window=1,
                           n_sink=0, k_choices=(8, 16, 32, 64)),
}

# Order used wherever "all configurations" are listed.
WORKLOAD_ORDER = ("tiny", "8k-gqa", "32k-gqa", "128k-structured", "batched-32")


def _seed(name: str, tensor: str, base: int) -> np.random.Generator:
    """A generator whose stream depends only on (workload name, tensor, base seed)."""
    ss = np.random.SeedSequence([base, zlib.crc32(name.encode()), zlib.crc32(tensor.encode())])
    return np.random.Generator(np.random.PCG64(ss))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round-to-nearest-even); return the bit patterns.

    Inputs are finite by construction, so NaN handling is not needed.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def _normal_bf16(gen: np.random.Generator, shape) -> np.ndarray:
    """N(0,1) samples rounded to bf16, drawn one leading slice at a time to bound memory."""
    out = np.empty(shape, dtype=np.uint16)
    lead = out.reshape(-1, shape[-2], shape[-1])
    for s in range(lead.shape[0]):
        lead[s] = f32_to_bf16_bits(gen.standard_normal(size=lead.shape[1:], dtype=np.float32))
    return out


def per_head_k(w: Workload, seed: int = 0) -> Optional[np.ndarray]:
    """Per-query-head budgets drawn from ``w.k_choices`` (one per head, shared across the batch)."""
    if w.k_choices is None:
        return None
    gen = _seed(w.name, "k_per_head", seed)
    return np.asarray(gen.choice(np.asarray(w.k_choices), size=w.Hq), dtype=np.int32)


def make_inputs(w: Workload, seed: int = 0, tensors=("q", "k", "v")) -> Dict[str, np.ndarray]:
    """Seeded bf16 Q [B,Hq,N,d], K/V [B,Hkv,N,d] as uint16 bit patterns.

    For ``structured_keys`` workloads, a seeded unit vector u (shared by all
    heads and blocks) times an amplitude a ~ U(2,4) is added to every key row
    of round(0.05 * nb) seeded key blocks per (batch, KV head), before the bf16
    rounding.
    """
    out: Dict[str, np.ndarray] = {}
    if "q" in tensors:
        out["q"] = _normal_bf16(_seed(w.name, "q", seed), (w.B, w.Hq, w.N, w.d))
    if "v" in tensors:
        out["v"] = _normal_bf16(_seed(w.name, "v", seed), (w.B, w.Hkv, w.N, w.d))
    if "k" in tensors:
        if not w.structured_keys:
            out["k"] = _normal_bf16(_seed(w.name, "k", seed), (w.B, w.Hkv, w.N, w.d))
        else:
            gk = _seed(w.name, "k", seed)
            gs = _seed(w.name, "k-structure", seed)
            u = gs.standard_normal(w.d)
            u = (u / np.linalg.norm(u)).astype(np.float32)
            n_boost = int(round(0.05 * w.nb))
            k = np.empty((w.B, w.Hkv, w.N, w.d), dtype=np.uint16)
            for b in range(w.B):
                for h in range(w.Hkv):
                    x = gk.standard_normal(size=(w.N, w.d), dtype=np.float32)
                    blocks = gs.choice(w.nb, size=n_boost, replace=False)
                    amps = gs.uniform(2.0, 4.0, size=n_boost).astype(np.float32)
                    xb = x.reshape(w.nb, w.block, w.d)
                    xb[blocks] += amps[:, None, None] * u[None, None, :]
                    k[b, h] = f32_to_bf16_bits(x)
            out["k"] = k
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32 (used for host-side checks)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
