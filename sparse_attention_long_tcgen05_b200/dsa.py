"""ctypes binding of libdsa.so (include/dsa.h): argument marshalling only.

Every function here forwards torch tensors' device pointers and the current
CUDA stream to the C ABI of the same name and raises DsaError on a non-OK
status. Every step of the DSA forward path runs in the library's CUDA
kernels; there is no Python or CPU fallback. Importing this module loads the
library and fails loudly if it has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")

DSA_OK = 0
DSA_ERR_INVALID_ARG = 1
DSA_ERR_UNSUPPORTED = 2
DSA_ERR_WORKSPACE_TOO_SMALL = 3
DSA_ERR_CUDA = 4
DSA_ERR_DEVICE_BOUNDS = 5
DSA_ERR_TIMEOUT = 6

DSA_F32, DSA_E4M3, DSA_BF16 = 0, 1, 2
DSA_KV_CONTIGUOUS, DSA_KV_PAGED = 0, 1
DSA_OP_INDEXER_SCORES, DSA_OP_TOPK, DSA_OP_SPARSE_MQA, DSA_OP_FORWARD = 0, 1, 2, 3

DSA_OP_SELECT = 4

EXPORTED = ["dsa_indexer_scores", "dsa_topk", "dsa_sparse_mqa_fwd", "dsa_select", "dsa_forward",
            "dsa_workspace_size", "dsa_check_status", "dsa_status_string",
            "dsa_last_cuda_error", "dsa_launch_counter", "dsa_version", "dsa_select_noalloc",
            "dsa_set_wait_limit_ns", "dsa_dense_mqa_fwd", "dsa_select_scored", "dsa_indexer_kl",
            "dsa_sparse_mqa_bwd"]


class DsaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: status {status} ({status_string(status)})")


class KvLayout(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("block_table", ctypes.c_void_p), ("ld_block_table", ctypes.c_int64),
                ("max_pages", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("ctx_lens", ctypes.c_void_p), ("q_seq", ctypes.c_void_p),
                ("q_pos", ctypes.c_void_p), ("n_seq", ctypes.c_int32)]


class IndexerIn(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("n_q", ctypes.c_int32), ("n_keys", ctypes.c_int32),
                ("heads", ctypes.c_int32), ("dim", ctypes.c_int32),
                ("q", ctypes.c_void_p), ("ld_q", ctypes.c_int64), ("q_scale", ctypes.c_void_p),
                ("k", ctypes.c_void_p), ("ld_k", ctypes.c_int64), ("k_scale", ctypes.c_void_p),
                ("w", ctypes.c_void_p), ("ld_w", ctypes.c_int64), ("kv", KvLayout)]


class AttnIn(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("n_q", ctypes.c_int32), ("n_keys", ctypes.c_int32),
                ("heads", ctypes.c_int32), ("d_qk", ctypes.c_int32), ("d_v", ctypes.c_int32),
                ("scale", ctypes.c_float),
                ("q", ctypes.c_void_p), ("ld_q", ctypes.c_int64),
                ("kv", ctypes.c_void_p), ("ld_kv", ctypes.c_int64),
                ("v", ctypes.c_void_p), ("ld_v", ctypes.c_int64),
                ("kv_layout", KvLayout)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m sparse_attention_long_tcgen05_b200._build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "dsa_indexer_scores": [ctypes.POINTER(IndexerIn), P, I32, P, I64, I32, P, SZ, P],
        "dsa_topk": [P, I64, P, I32, I32, P, I64, P],
        "dsa_sparse_mqa_fwd": [ctypes.POINTER(AttnIn), P, I64, I32, P, P, P, SZ, P],
        "dsa_select": [ctypes.POINTER(IndexerIn), I32, P, I64, P, SZ, P],
        "dsa_dense_mqa_fwd": [ctypes.POINTER(AttnIn), P, P, P],
        "dsa_select_scored": [ctypes.POINTER(IndexerIn), I32, P, I64, P, I64, P, SZ, P],
        "dsa_indexer_kl": [ctypes.POINTER(AttnIn), P, I64, I32, P, P, I64, P, P, I64, P],
        "dsa_sparse_mqa_bwd": [ctypes.POINTER(AttnIn), P, I64, I32, P, P, P, P, P, I64, P, P],
        "dsa_forward": [ctypes.POINTER(IndexerIn), ctypes.POINTER(AttnIn), I32, P, P, P, P, SZ, P],
        "dsa_launch_counter": [],
        "dsa_set_wait_limit_ns": [I64],
        "dsa_select_noalloc": [ctypes.POINTER(IndexerIn), I32, P, I64, P],
        "dsa_workspace_size": [I32, ctypes.POINTER(IndexerIn), ctypes.POINTER(AttnIn), I32, I32,
                               I32, ctypes.POINTER(SZ)],
        "dsa_check_status": [P],
        "dsa_status_string": [ctypes.c_int],
        "dsa_last_cuda_error": [],
        "dsa_version": [],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = {"dsa_status_string": ctypes.c_char_p,
                     "dsa_launch_counter": ctypes.c_int64}.get(name, ctypes.c_int32)
    return lib


LIB = _load()


def status_string(status: int) -> str:
    return LIB.dsa_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, what: str):
    if status != DSA_OK:
        raise DsaError(status, what + (f" (cudaError {LIB.dsa_last_cuda_error()})"
                                       if status == DSA_ERR_CUDA else ""))


# ------------------------------------------------------------ struct builders

class _Keep:
    """A C struct plus the tensors whose pointers it holds."""

    def __init__(self, struct, tensors):
        self.struct = struct
        self.tensors = tensors


def paged_layout(block_table: torch.Tensor, ctx_lens: torch.Tensor, num_pages: int,
                 q_seq: Optional[torch.Tensor] = None,
                 q_pos: Optional[torch.Tensor] = None) -> KvLayout:
    """PAGED key side: block_table [n_seq, max_pages] and ctx_lens [n_seq]
    int32; optional q_seq / q_pos [n_q] int32 (sequence and position of each
    query; by default query b is the newest token of sequence b). The caller
    keeps the tensors alive while the layout is in use."""
    return KvLayout(DSA_KV_PAGED, 64, block_table.data_ptr(), block_table.stride(0),
                    block_table.shape[1], num_pages, ctx_lens.data_ptr(),
                    q_seq.data_ptr() if q_seq is not None else None,
                    q_pos.data_ptr() if q_pos is not None else None, ctx_lens.shape[0])


def indexer_in(q, k, w, q_scale=None, k_scale=None, n_keys=None, kv: Optional[KvLayout] = None):
    """q [n_q, H_I, d_I] (uint8 e4m3 codes or float32), k [n_keys, d_I] or paged
    [pages, 64, d_I], w [n_q, H_I]; scales [n_q] / [n_keys or pages*64]."""
    fp8 = q.dtype == torch.uint8
    n_q, heads, dim = q.shape
    kv = kv if kv is not None else KvLayout(DSA_KV_CONTIGUOUS, 0, None, 0, 0, 0, None)
    ld_k = k.stride(-2)
    s = IndexerIn(DSA_E4M3 if fp8 else DSA_F32, n_q,
                  (n_keys if n_keys is not None else k.shape[0]) if kv.kind == DSA_KV_CONTIGUOUS
                  else 0,
                  heads, dim, q.data_ptr(), q.stride(0),
                  q_scale.data_ptr() if q_scale is not None else None,
                  k.data_ptr(), ld_k, k_scale.data_ptr() if k_scale is not None else None,
                  w.data_ptr(), w.stride(0), kv)
    return _Keep(s, [q, k, w, q_scale, k_scale])


def attn_in(q, kv, scale, d_v, v=None, kv_layout: Optional[KvLayout] = None):
    """q [n_q, H, d_qk], kv [n_keys, d_qk] or paged [pages, 64, d_qk] (bf16 or
    float32), optional separate v [n_keys, d_v] (float32 only)."""
    bf16 = q.dtype == torch.bfloat16
    n_q, heads, d_qk = q.shape
    lay = kv_layout if kv_layout is not None else KvLayout(DSA_KV_CONTIGUOUS, 0, None, 0, 0, 0,
                                                           None)
    s = AttnIn(DSA_BF16 if bf16 else DSA_F32, n_q,
               kv.shape[0] if lay.kind == DSA_KV_CONTIGUOUS else 0,
               heads, d_qk, d_v, float(scale), q.data_ptr(), q.stride(0), kv.data_ptr(),
               kv.stride(-2), v.data_ptr() if v is not None else None,
               v.stride(0) if v is not None else 0, lay)
    return _Keep(s, [q, kv, v])


# ------------------------------------------------------------ the C ABI calls

def dsa_workspace_size(op, ind: Optional[_Keep] = None, attn: Optional[_Keep] = None,
                       n_rows: int = 0, n_cols: int = 0, k: int = 0) -> int:
    out = ctypes.c_size_t(0)
    _check(LIB.dsa_workspace_size(op, ctypes.byref(ind.struct) if ind else None,
                                  ctypes.byref(attn.struct) if attn else None,
                                  n_rows, n_cols, k, ctypes.byref(out)), "dsa_workspace_size")
    return out.value


def dsa_indexer_scores(ind: _Keep, rows: Optional[torch.Tensor], n_rows: int,
                       scores: torch.Tensor, n_cols: int, ws: Optional[torch.Tensor] = None,
                       stream=None):
    _check(LIB.dsa_indexer_scores(ctypes.byref(ind.struct), _ptr(rows), n_rows, _ptr(scores),
                                  scores.stride(0), n_cols, _ptr(ws),
                                  0 if ws is None else ws.numel() * ws.element_size(),
                                  _stream(stream)), "dsa_indexer_scores")


def dsa_topk(scores: torch.Tensor, row_pos: torch.Tensor, k: int, idx: torch.Tensor,
             stream=None):
    _check(LIB.dsa_topk(_ptr(scores), scores.stride(0), _ptr(row_pos), scores.shape[0], k,
                        _ptr(idx), idx.stride(0), _stream(stream)), "dsa_topk")


def dsa_sparse_mqa_fwd(attn: _Keep, idx: torch.Tensor, k: int, out: torch.Tensor,
                       lse: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                       stream=None):
    _check(LIB.dsa_sparse_mqa_fwd(ctypes.byref(attn.struct), _ptr(idx), idx.stride(0), k,
                                  _ptr(out), _ptr(lse), _ptr(ws),
                                  0 if ws is None else ws.numel() * ws.element_size(),
                                  _stream(stream)), "dsa_sparse_mqa_fwd")


def dsa_dense_mqa_fwd(attn: _Keep, out: torch.Tensor, lse: Optional[torch.Tensor] = None,
                      stream=None):
    _check(LIB.dsa_dense_mqa_fwd(ctypes.byref(attn.struct), _ptr(out), _ptr(lse),
                                 _stream(stream)), "dsa_dense_mqa_fwd")


def dsa_select_scored(ind: _Keep, k: int, idx: torch.Tensor, sel_scores: torch.Tensor,
                      ws: torch.Tensor, stream=None):
    _check(LIB.dsa_select_scored(ctypes.byref(ind.struct), k, _ptr(idx), idx.stride(0),
                                 _ptr(sel_scores), sel_scores.stride(0), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream)),
           "dsa_select_scored")


def dsa_indexer_kl(attn: _Keep, idx: torch.Tensor, k: int, lse: torch.Tensor,
                   sel_scores: torch.Tensor, loss: torch.Tensor, grad: torch.Tensor,
                   stream=None):
    _check(LIB.dsa_indexer_kl(ctypes.byref(attn.struct), _ptr(idx), idx.stride(0), k, _ptr(lse),
                              _ptr(sel_scores), sel_scores.stride(0), _ptr(loss), _ptr(grad),
                              grad.stride(0), _stream(stream)), "dsa_indexer_kl")


def dsa_sparse_mqa_bwd(attn: _Keep, idx: torch.Tensor, k: int, out: torch.Tensor,
                       lse: torch.Tensor, d_out: torch.Tensor, d_q: torch.Tensor,
                       d_kv: torch.Tensor, delta: torch.Tensor, stream=None):
    """Gradient of dsa_sparse_mqa_fwd: writes d_q and delta, ADDS into d_kv."""
    _check(LIB.dsa_sparse_mqa_bwd(ctypes.byref(attn.struct), _ptr(idx), idx.stride(0), k,
                                  _ptr(out), _ptr(lse), _ptr(d_out), _ptr(d_q), _ptr(d_kv),
                                  d_kv.stride(0), _ptr(delta), _stream(stream)),
           "dsa_sparse_mqa_bwd")


def dsa_select(ind: _Keep, k: int, idx: torch.Tensor, ws: torch.Tensor, stream=None):
    _check(LIB.dsa_select(ctypes.byref(ind.struct), k, _ptr(idx), idx.stride(0), _ptr(ws),
                          ws.numel() * ws.element_size(), _stream(stream)), "dsa_select")


def dsa_select_noalloc(ind: _Keep, k: int, idx: torch.Tensor, stream=None):
    """dsa_select without a workspace, for callers that cannot allocate device
    memory: the library's fixed 16 MiB per-GPU scratch holds the score rows.
    Calls on one device must not overlap (they share that scratch)."""
    _check(LIB.dsa_select_noalloc(ctypes.byref(ind.struct), k, _ptr(idx), idx.stride(0),
                                  _stream(stream)), "dsa_select_noalloc")


def dsa_set_wait_limit_ns(ns: int):
    """Bound of the indexer kernel's pipeline waits (ns <= 0: the 1 s default)."""
    _check(LIB.dsa_set_wait_limit_ns(int(ns)), "dsa_set_wait_limit_ns")


def dsa_launch_counter() -> int:
    return int(LIB.dsa_launch_counter())


def dsa_forward(ind: _Keep, attn: _Keep, k: int, idx_out: Optional[torch.Tensor],
                out: torch.Tensor, lse: Optional[torch.Tensor], ws: torch.Tensor, stream=None):
    _check(LIB.dsa_forward(ctypes.byref(ind.struct), ctypes.byref(attn.struct), k,
                           _ptr(idx_out), _ptr(out), _ptr(lse), _ptr(ws),
                           ws.numel() * ws.element_size(), _stream(stream)), "dsa_forward")


def dsa_check_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status."""
    return int(LIB.dsa_check_status(_stream(stream)))


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A 256-byte aligned device buffer of at least nbytes (torch allocations are)."""
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
