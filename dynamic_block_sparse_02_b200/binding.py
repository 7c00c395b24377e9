"""Thin Python binding of libdsa (the C ABI in include/dsa.h).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels. Tensor arguments may be torch tensors (their device
pointer is passed after shape, dtype, contiguity and device checks) or raw
integer addresses. There is no CPU fallback: if libdsa.so is missing the
import fails.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libdsa.so is not built ({LIB_PATH}); run "
                      "`python -m dynamic_block_sparse_02_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

# dsa_status values
DSA_OK = 0
DSA_ERR_INVALID_ARG = 1
DSA_ERR_UNSUPPORTED = 2
DSA_ERR_WORKSPACE = 3
DSA_ERR_CUDA = 4
DSA_ERR_DEVICE_TIMEOUT = 5
DSA_ERR_DEVICE_BOUNDS = 6

# dsa_attn_kernel values
DSA_ATTN_AUTO = 0
DSA_ATTN_TCGEN05 = 1
DSA_ATTN_MMA_SYNC = 2

# dsa_select_mode values
DSA_SELECT_TOPK = 0
DSA_SELECT_GROUP_TOPK = 1
DSA_SELECT_THRESHOLD = 2

# Every function the header declares, with its C signature.
_vp, _sz, _i32p, _f32p = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p


class dsa_params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("N", ctypes.c_int), ("d", ctypes.c_int), ("block", ctypes.c_int),
                ("k_free", ctypes.c_int), ("k_per_head", ctypes.POINTER(ctypes.c_int32)),
                ("local_window", ctypes.c_int), ("n_sink", ctypes.c_int),
                ("scale", ctypes.c_float), ("attn_kernel", ctypes.c_int),
                ("select_mode", ctypes.c_int), ("select_tau", ctypes.c_float)]


_P = ctypes.POINTER(dsa_params)
SIGNATURES = {
    "dsa_kmax": (_sz, [_P]),
    "dsa_attn_uses_tcgen05": (ctypes.c_int, [_P]),
    "dsa_workspace_size": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_size_t)]),
    "dsa_workspace_init": (ctypes.c_int, [_vp, _sz, _vp]),
    "dsa_workspace_set_wait_limit": (ctypes.c_int, [_vp, _sz, ctypes.c_ulonglong, _vp]),
    "dsa_block_scores": (ctypes.c_int, [_P, _vp, _vp, _f32p, _vp, _sz, _vp]),
    "dsa_topk_select": (ctypes.c_int, [_P, _f32p, _i32p, _i32p, _vp]),
    "dsa_select_blocks": (ctypes.c_int, [_P, _vp, _vp, _i32p, _i32p, _vp, _sz, _vp]),
    "dsa_select_blocks_static": (ctypes.c_int, [_P, _vp, _vp, _i32p, _i32p, _vp]),
    "dsa_sparse_attn_fwd": (ctypes.c_int, [_P, _vp, _vp, _vp, _i32p, _i32p, _vp, _f32p, _vp, _sz, _vp]),
    "dsa_sparse_attn_bwd": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _f32p, _vp, _i32p, _i32p, _vp, _vp,
                                           _vp, _vp, _sz, _vp]),
    "dsa_forward": (ctypes.c_int, [_P, _vp, _vp, _vp, _vp, _f32p, _i32p, _i32p, _vp, _sz, _vp]),
    "dsa_pool_keys": (ctypes.c_int, [_P, _vp, _f32p, ctypes.c_int, ctypes.c_int, _vp]),
    "dsa_decode_fwd": (ctypes.c_int, [_P, _vp, _vp, _vp, _f32p, ctypes.c_int, _vp, _f32p, _i32p, _i32p,
                                      _vp, _sz, _vp]),
    "dsa_check_status": (ctypes.c_int, [_vp, _vp]),
    "dsa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}
for _name, (_res, _args) in SIGNATURES.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class DsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def status_string(status: int) -> str:
    return _lib.dsa_status_string(int(status)).decode()


class Params:
    """Python-side holder of a dsa_params struct (keeps k_per_head alive)."""

    def __init__(self, B, Hq, Hkv, N, d, block, k_free=0, k_per_head: Optional[Sequence[int]] = None,
                 local_window=1, n_sink=0, scale=0.0, attn_kernel=DSA_ATTN_AUTO,
                 select_mode=DSA_SELECT_TOPK, select_tau=0.0):
        self._kph = None
        kph_ptr = None
        if k_per_head is not None:
            self._kph = (ctypes.c_int32 * len(k_per_head))(*[int(x) for x in k_per_head])
            kph_ptr = ctypes.cast(self._kph, ctypes.POINTER(ctypes.c_int32))
        self.c = dsa_params(int(B), int(Hq), int(Hkv), int(N), int(d), int(block), int(k_free),
                            kph_ptr, int(local_window), int(n_sink), float(scale), int(attn_kernel),
                            int(select_mode), float(select_tau))

    @classmethod
    def from_workload(cls, w, k_per_head=None, attn_kernel=DSA_ATTN_AUTO, select_mode=DSA_SELECT_TOPK,
                      **over):
        kw = dict(B=w.B, Hq=w.Hq, Hkv=w.Hkv, N=w.N, d=w.d, block=w.block, k_free=w.k_free,
                  k_per_head=k_per_head, local_window=w.local_window, n_sink=w.n_sink,
                  scale=w.scale, attn_kernel=attn_kernel, select_mode=select_mode)
        kw.update(over)
        return cls(**kw)

    @property
    def ref(self):
        return ctypes.byref(self.c)

    @property
    def nb(self) -> int:
        return self.c.N // self.c.block if self.c.block else 0


def _ptr(x) -> Optional[int]:
    """Device address of a tensor argument (None passes NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    if x.device.type != "cuda":
        raise ValueError("tensor arguments must be CUDA device tensors")
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        try:
            import torch
            return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
        except Exception:
            return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != DSA_OK:
        raise DsaError(status, where)


def dsa_kmax(p: Params) -> int:
    return int(_lib.dsa_kmax(p.ref))


def dsa_attn_uses_tcgen05(p: Params) -> int:
    return int(_lib.dsa_attn_uses_tcgen05(p.ref))


def dsa_workspace_size(p: Params) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.dsa_workspace_size(p.ref, ctypes.byref(n)), "dsa_workspace_size")
    return int(n.value)


def dsa_workspace_init(ws, ws_bytes: int, stream=None) -> None:
    _check(_lib.dsa_workspace_init(_ptr(ws), ws_bytes, _stream(stream)), "dsa_workspace_init")


def dsa_workspace_set_wait_limit(ws, ws_bytes: int, ns: int, stream=None) -> None:
    _check(_lib.dsa_workspace_set_wait_limit(_ptr(ws), ws_bytes, int(ns), _stream(stream)),
           "dsa_workspace_set_wait_limit")


def dsa_block_scores(p: Params, q, k, scores, ws, ws_bytes: int, stream=None) -> None:
    _check(_lib.dsa_block_scores(p.ref, _ptr(q), _ptr(k), _ptr(scores), _ptr(ws), ws_bytes,
                                 _stream(stream)), "dsa_block_scores")


def dsa_topk_select(p: Params, scores, idx, cnt, stream=None) -> None:
    _check(_lib.dsa_topk_select(p.ref, _ptr(scores), _ptr(idx), _ptr(cnt), _stream(stream)),
           "dsa_topk_select")


def dsa_select_blocks(p: Params, q, k, idx, cnt, ws, ws_bytes: int, stream=None) -> None:
    _check(_lib.dsa_select_blocks(p.ref, _ptr(q), _ptr(k), _ptr(idx), _ptr(cnt), _ptr(ws),
                                  ws_bytes, _stream(stream)), "dsa_select_blocks")


def dsa_select_blocks_static(p: Params, q, k, idx, cnt, stream=None) -> None:
    _check(_lib.dsa_select_blocks_static(p.ref, _ptr(q), _ptr(k), _ptr(idx), _ptr(cnt),
                                         _stream(stream)), "dsa_select_blocks_static")


def dsa_sparse_attn_fwd(p: Params, q, k, v, idx, cnt, out, lse, ws, ws_bytes: int,
                        stream=None) -> None:
    _check(_lib.dsa_sparse_attn_fwd(p.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(cnt),
                                    _ptr(out), _ptr(lse), _ptr(ws), ws_bytes, _stream(stream)),
           "dsa_sparse_attn_fwd")


def dsa_sparse_attn_bwd(p: Params, q, k, v, out, lse, dout, idx, cnt, dq, dk, dv, ws, ws_bytes: int,
                        stream=None) -> None:
    _check(_lib.dsa_sparse_attn_bwd(p.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout),
                                    _ptr(idx), _ptr(cnt), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
                                    ws_bytes, _stream(stream)),
           "dsa_sparse_attn_bwd")


def dsa_forward(p: Params, q, k, v, out, lse, idx, cnt, ws, ws_bytes: int, stream=None) -> None:
    _check(_lib.dsa_forward(p.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(idx),
                            _ptr(cnt), _ptr(ws), ws_bytes, _stream(stream)), "dsa_forward")


def dsa_pool_keys(p: Params, k, kp, j_begin: int, j_end: int, stream=None) -> None:
    _check(_lib.dsa_pool_keys(p.ref, _ptr(k), _ptr(kp), int(j_begin), int(j_end), _stream(stream)),
           "dsa_pool_keys")


def dsa_decode_fwd(p: Params, q, k, v, kp, length: int, out, lse, idx, cnt, ws, ws_bytes: int,
                   stream=None) -> None:
    _check(_lib.dsa_decode_fwd(p.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(kp), int(length), _ptr(out),
                               _ptr(lse), _ptr(idx), _ptr(cnt), _ptr(ws), ws_bytes, _stream(stream)),
           "dsa_decode_fwd")


def dsa_check_status(ws, stream=None) -> int:
    """Synchronise, read and clear the device error flag; return the dsa_status value."""
    return int(_lib.dsa_check_status(_ptr(ws), _stream(stream)))


def raw(name: str):
    """The raw ctypes function of a C-ABI symbol (for argument-error tests)."""
    return getattr(_lib, name)
