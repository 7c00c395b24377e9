"""User-level wrapper: one block-sparse attention problem with its workspace.

The C library never allocates; this wrapper allocates the workspace once with
torch (caller-owned memory, as the C ABI expects) and forwards every call to
the C ABI through ``binding``.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import binding as B


class BlockSparseAttention:
    """Dynamic top-k block-sparse causal attention for one fixed problem shape.

    ``forward(q, k, v)`` takes bf16 CUDA tensors Q [B,Hq,N,d], K/V [B,Hkv,N,d]
    and returns O [B,Hq,N,d] (bf16), plus the log-sum-exp and the kept block
    lists when asked.
    """

    def __init__(self, B_: int, Hq: int, Hkv: int, N: int, d: int, block: int, k_free: int = 0,
                 k_per_head: Optional[Sequence[int]] = None, local_window: int = 1,
                 n_sink: int = 0, scale: float = 0.0, attn_kernel: int = B.DSA_ATTN_AUTO,
                 select_mode: int = B.DSA_SELECT_TOPK, select_tau: float = 0.0, device=None,
                 stream=None):
        self.params = B.Params(B_, Hq, Hkv, N, d, block, k_free, k_per_head, local_window, n_sink,
                               scale, attn_kernel, select_mode, select_tau)
        self.shape = (B_, Hq, Hkv, N, d, block)
        self.device = torch.device(device) if device is not None else torch.device("cuda")
        self.ws_bytes = B.dsa_workspace_size(self.params)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.device)
        self.width = B.dsa_kmax(self.params)
        self.stream = stream
        B.dsa_workspace_init(self.ws, self.ws_bytes, stream)

    @classmethod
    def from_workload(cls, w, k_per_head=None, attn_kernel=B.DSA_ATTN_AUTO, device=None,
                      select_mode=B.DSA_SELECT_TOPK, **over):
        kw = dict(B_=w.B, Hq=w.Hq, Hkv=w.Hkv, N=w.N, d=w.d, block=w.block, k_free=w.k_free,
                  k_per_head=k_per_head, local_window=w.local_window, n_sink=w.n_sink,
                  scale=w.scale, attn_kernel=attn_kernel, select_mode=select_mode, device=device)
        kw.update(over)
        return cls(**kw)

    @property
    def nb(self) -> int:
        return self.shape[3] // self.shape[5]

    def empty_out(self):
        Bn, Hq, _, N, d, _ = self.shape
        return torch.empty((Bn, Hq, N, d), dtype=torch.bfloat16, device=self.device)

    def empty_lse(self):
        Bn, Hq, _, N, _, _ = self.shape
        return torch.empty((Bn, Hq, N), dtype=torch.float32, device=self.device)

    def empty_selection(self):
        Bn, Hq = self.shape[0], self.shape[1]
        idx = torch.empty((Bn, Hq, self.nb, self.width), dtype=torch.int32, device=self.device)
        cnt = torch.empty((Bn, Hq, self.nb), dtype=torch.int32, device=self.device)
        return idx, cnt

    def forward(self, q, k, v, out=None, lse=None, idx=None, cnt=None):
        """Pool, score, select and attend (dsa_forward). Returns out (and lse/idx/cnt if given)."""
        out = self.empty_out() if out is None else out
        B.dsa_forward(self.params, q, k, v, out, lse, idx, cnt, self.ws, self.ws_bytes, self.stream)
        return out

    def block_scores(self, q, k, scores=None):
        Bn, Hq = self.shape[0], self.shape[1]
        if scores is None:
            scores = torch.empty((Bn, Hq, self.nb, self.nb), dtype=torch.float32, device=self.device)
        B.dsa_block_scores(self.params, q, k, scores, self.ws, self.ws_bytes, self.stream)
        return scores

    def select_blocks(self, q, k, idx=None, cnt=None):
        """Pool, score and select in one call (dsa_select_blocks)."""
        if idx is None:
            idx, cnt = self.empty_selection()
        B.dsa_select_blocks(self.params, q, k, idx, cnt, self.ws, self.ws_bytes, self.stream)
        return idx, cnt

    def topk_select(self, scores, idx=None, cnt=None):
        if idx is None:
            idx, cnt = self.empty_selection()
        B.dsa_topk_select(self.params, scores, idx, cnt, self.stream)
        return idx, cnt

    def sparse_attn(self, q, k, v, idx, cnt, out=None, lse=None):
        out = self.empty_out() if out is None else out
        B.dsa_sparse_attn_fwd(self.params, q, k, v, idx, cnt, out, lse, self.ws, self.ws_bytes,
                              self.stream)
        return out

    def sparse_attn_backward(self, q, k, v, out, lse, dout, idx, cnt, dq=None, dk=None, dv=None):
        """Gradients of sparse_attn over the kept blocks (dsa_sparse_attn_bwd); out and
        lse are the forward's outputs for the same idx/cnt. Returns (dq, dk, dv)."""
        dq = torch.empty_like(q) if dq is None else dq
        dk = torch.empty_like(k) if dk is None else dk
        dv = torch.empty_like(v) if dv is None else dv
        B.dsa_sparse_attn_bwd(self.params, q, k, v, out, lse, dout, idx, cnt, dq, dk, dv, self.ws,
                              self.ws_bytes, self.stream)
        return dq, dk, dv

    def pooled_key_cache(self):
        """An fp32 [B, Hkv, N/block, d] buffer for the pooled key cache."""
        Bn, _, Hkv, N, d, bs = self.shape
        return torch.empty((Bn, Hkv, N // bs, d), dtype=torch.float32, device=self.device)

    def pool_keys(self, k_cache, kp_cache, j_begin: int, j_end: int):
        """Pool key blocks [j_begin, j_end) of the cache into kp_cache (dsa_pool_keys)."""
        B.dsa_pool_keys(self.params, k_cache, kp_cache, j_begin, j_end, self.stream)
        return kp_cache

    def decode(self, q, k_cache, v_cache, kp_cache, length: int, out=None, lse=None, idx=None,
               cnt=None):
        """One decode step (dsa_decode_fwd): q [B, Hq, d] at position length - 1."""
        Bn, Hq, _, _, d, _ = self.shape
        if out is None:
            out = torch.empty((Bn, Hq, d), dtype=torch.bfloat16, device=self.device)
        B.dsa_decode_fwd(self.params, q, k_cache, v_cache, kp_cache, length, out, lse, idx, cnt,
                         self.ws, self.ws_bytes, self.stream)
        return out

    def set_wait_limit(self, ns: int) -> None:
        """Time limit (ns) of the kernels' bounded waits; 0 = the default."""
        B.dsa_workspace_set_wait_limit(self.ws, self.ws_bytes, ns, self.stream)

    def check_status(self) -> int:
        return B.dsa_check_status(self.ws, self.stream)
