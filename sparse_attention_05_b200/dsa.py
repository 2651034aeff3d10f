"""Thin Python binding of the C ABI in include/dsa.h (libdsa.so).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. Tensors are PyTorch CUDA tensors (device memory and streams come from
PyTorch); each call is enqueued on the current PyTorch stream unless a stream
is given. There is no CPU or PyTorch fallback: a missing library raises.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa.so")

DSA_KV_CONTIGUOUS = 0
DSA_KV_PAGED = 1

H_IDX, D_IDX, HEADS, D_QK, D_V, MAX_K = 64, 128, 128, 576, 512, 2048

STATUS = {
    0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED_SHAPE", 3: "DSA_ERR_CUDA",
    4: "DSA_ERR_DEVICE_TIMEOUT", 5: "DSA_ERR_BOUNDS", 6: "DSA_ERR_WORKSPACE",
}


class DSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class KvDescC(ctypes.Structure):
    _fields_ = [
        ("layout", ctypes.c_int32), ("batch", ctypes.c_int32), ("max_ctx", ctypes.c_int32),
        ("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int32),
        ("max_pages", ctypes.c_int32), ("block_table", ctypes.c_void_p),
        ("seqlens", ctypes.c_void_p),
    ]


class QDescC(ctypes.Structure):
    _fields_ = [("num_q", ctypes.c_int32), ("q_per_seq", ctypes.c_int32),
                ("row_begin", ctypes.c_int32), ("row_count", ctypes.c_int32),
                ("q_start", ctypes.c_void_p)]


_P = ctypes.c_void_p
_lib = None

# name -> (restype, argtypes): mirrors include/dsa.h
SIGNATURES = {
    "dsa_indexer_scores": (ctypes.c_int, [_P, _P, _P, _P, ctypes.POINTER(KvDescC),
                                          ctypes.POINTER(QDescC), _P, ctypes.c_int64, _P]),
    "dsa_topk": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.POINTER(KvDescC),
                                ctypes.POINTER(QDescC), ctypes.c_int32, _P, _P]),
    "dsa_topk_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(KvDescC), ctypes.POINTER(QDescC),
                                                  ctypes.c_int32]),
    "dsa_topk_ws": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.POINTER(KvDescC),
                                   ctypes.POINTER(QDescC), ctypes.c_int32, _P, ctypes.c_size_t,
                                   _P, _P]),
    "dsa_sparse_mla_fwd": (ctypes.c_int, [_P, _P, ctypes.POINTER(KvDescC), ctypes.POINTER(QDescC),
                                          _P, ctypes.c_int32, ctypes.c_float, _P, _P, _P]),
    "dsa_sparse_mla_fwd_ws": (ctypes.c_int, [_P, _P, ctypes.POINTER(KvDescC),
                                             ctypes.POINTER(QDescC), _P, ctypes.c_int32,
                                             ctypes.c_float, _P, ctypes.c_size_t, _P, _P, _P]),
    "dsa_sparse_mla_workspace_size": (ctypes.c_size_t, []),
    "dsa_indexer_kl": (ctypes.c_int, [_P, _P, ctypes.POINTER(KvDescC), ctypes.POINTER(QDescC),
                                      _P, ctypes.c_int32, ctypes.c_float, _P, _P, ctypes.c_int64,
                                      _P, _P]),
    "dsa_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(KvDescC), ctypes.POINTER(QDescC),
                                             ctypes.c_int32]),
    "dsa_forward": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.POINTER(KvDescC),
                                   ctypes.POINTER(QDescC), ctypes.c_int32, ctypes.c_float, _P,
                                   ctypes.c_size_t, _P, _P, _P, _P]),
    "dsa_forward_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.POINTER(KvDescC),
                                           ctypes.POINTER(QDescC), ctypes.c_int32, ctypes.c_float,
                                           _P, _P, _P, _P]),
    "dsa_mla_up_project": (ctypes.c_int, [_P, _P, _P, ctypes.POINTER(KvDescC), _P, _P, _P,
                                          ctypes.c_int64, _P]),
    "dsa_selection_mask": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.POINTER(KvDescC),
                                          ctypes.POINTER(QDescC), _P, ctypes.c_int64, _P]),
    "dsa_masked_mha": (ctypes.c_int, [_P, _P, _P, _P, ctypes.c_int64, ctypes.POINTER(KvDescC),
                                      ctypes.POINTER(QDescC), _P, ctypes.c_int64, ctypes.c_int32,
                                      ctypes.c_float, _P, _P, _P]),
    "dsa_mha_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(KvDescC), ctypes.POINTER(QDescC),
                                                 ctypes.c_int32]),
    "dsa_mha_prefill": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, ctypes.POINTER(KvDescC),
                                       ctypes.POINTER(QDescC), ctypes.c_int32, ctypes.c_float, _P,
                                       ctypes.c_size_t, _P, _P, _P, _P]),
    "dsa_fused_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(KvDescC), ctypes.POINTER(QDescC),
                                                   ctypes.c_int32]),
    "dsa_select_fused": (ctypes.c_int, [_P, _P, _P, _P, ctypes.POINTER(KvDescC),
                                        ctypes.POINTER(QDescC), ctypes.c_int32, ctypes.c_int32, _P,
                                        ctypes.c_size_t, _P, _P]),
    "dsa_forward_fused": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.POINTER(KvDescC),
                                         ctypes.POINTER(QDescC), ctypes.c_int32, ctypes.c_float,
                                         ctypes.c_int32, _P, ctypes.c_size_t, _P, _P, _P, _P]),
    "dsa_get_device_error": (ctypes.c_int, [_P]),
    "dsa_set_wait_timeout_ns": (ctypes.c_uint64, [ctypes.c_uint64]),
    "dsa_selftest_wait_timeout": (ctypes.c_int, [_P]),
    "dsa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}


def lib() -> ctypes.CDLL:
    """Load libdsa.so (built in-tree by ``sparse_attention_05_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libdsa.so not built ({LIB_PATH}); run "
                               "python -m sparse_attention_05_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise DSAError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the DSA library must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the DSA library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


@dataclasses.dataclass
class KvLayout:
    """Geometry of the per-token caches (dsa_kv_desc_t)."""
    batch: int
    max_ctx: int
    seqlens: Optional[torch.Tensor] = None         # int32 [batch] on the device
    block_table: Optional[torch.Tensor] = None     # int32 [batch, max_pages] (paged)
    page_size: int = 64
    num_pages: int = 0

    @property
    def paged(self) -> bool:
        return self.block_table is not None

    def c(self) -> KvDescC:
        d = KvDescC()
        d.layout = DSA_KV_PAGED if self.paged else DSA_KV_CONTIGUOUS
        d.batch, d.max_ctx = self.batch, self.max_ctx
        d.page_size = self.page_size if self.paged else 0
        d.num_pages = self.num_pages if self.paged else 0
        d.max_pages = self.block_table.shape[1] if self.paged else 0
        d.block_table = _ptr(self.block_table).value if self.paged else None
        d.seqlens = _ptr(self.seqlens).value if self.seqlens is not None else None
        return d

    @staticmethod
    def of(problem) -> "KvLayout":
        """Geometry of a synth.Problem whose tensors live on the GPU."""
        return KvLayout(batch=problem.batch, max_ctx=problem.max_ctx, seqlens=problem.seqlens,
                        block_table=problem.block_table if problem.paged else None,
                        page_size=problem.page_size,
                        num_pages=problem.k_idx.shape[0] if problem.paged else 0)


def _qdesc(num_q: int, q_per_seq: int, rows: Optional[Tuple[int, int]] = None,
           q_start: Optional[torch.Tensor] = None) -> QDescC:
    """rows = (row_begin, row_count) window within each sequence (None = all);
    q_start = int32 [batch + 1] device offsets of a ragged batch's query rows
    (sequence b owns rows q_start[b] .. q_start[b+1] - 1; q_per_seq = the largest
    count), None for a uniform batch."""
    r0, rc = rows if rows is not None else (0, 0)
    if q_start is not None and (q_start.dtype != torch.int32 or q_start.dim() != 1):
        raise ValueError("q_start must be a 1-D int32 tensor of batch + 1 offsets")
    return QDescC(num_q, q_per_seq, r0, rc, _ptr(q_start).value if q_start is not None else None)


def round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


def _window(kv: KvLayout, q_per_seq: int, rows) -> int:
    """Rows per sequence covered by the window."""
    r0, rc = rows if rows is not None else (0, 0)
    return rc if rc else q_per_seq - r0


def dsa_indexer_scores(q_idx, w, k_idx, k_scale, kv: KvLayout, q_per_seq: int,
                       scores: Optional[torch.Tensor] = None, rows=None,
                       stream=None, q_start=None) -> torch.Tensor:
    """Scores [batch * window_rows, ld] (window rows stored compactly)."""
    T = q_idx.shape[0]
    if scores is None:
        scores = torch.empty(kv.batch * _window(kv, q_per_seq, rows), round_up(kv.max_ctx, 128),
                             dtype=torch.float32, device=q_idx.device)
    kvd, qd = kv.c(), _qdesc(T, q_per_seq, rows, q_start)
    _check(lib().dsa_indexer_scores(_ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(k_scale),
                                    ctypes.byref(kvd), ctypes.byref(qd), _ptr(scores),
                                    scores.shape[1], _stream(stream)), "dsa_indexer_scores")
    return scores


def dsa_topk(scores, kv: KvLayout, q_per_seq: int, k: int,
             idx: Optional[torch.Tensor] = None, rows=None, stream=None, q_start=None,
             num_q: Optional[int] = None) -> torch.Tensor:
    """Selected positions [T, k] (rows outside the window are left untouched). A
    ragged batch (q_start) needs ``idx`` or ``num_q`` for T."""
    if q_start is None:
        T = kv.batch * q_per_seq
    elif num_q is not None:
        T = num_q
    elif idx is not None:
        T = idx.shape[0]
    else:
        raise ValueError("dsa_topk on a ragged batch needs idx or num_q")
    if idx is None:
        idx = torch.empty(T, k, dtype=torch.int32, device=scores.device)
    kvd, qd = kv.c(), _qdesc(T, q_per_seq, rows, q_start)
    _check(lib().dsa_topk(_ptr(scores), scores.shape[1], ctypes.byref(kvd), ctypes.byref(qd), k,
                          _ptr(idx), _stream(stream)), "dsa_topk")
    return idx


def dsa_topk_workspace_size(kv: KvLayout, num_q: int, q_per_seq: int, k: int, rows=None,
                            q_start=None) -> int:
    kvd, qd = kv.c(), _qdesc(num_q, q_per_seq, rows, q_start)
    return int(lib().dsa_topk_workspace_size(ctypes.byref(kvd), ctypes.byref(qd), k))


def dsa_topk_ws(scores, kv: KvLayout, q_per_seq: int, k: int, workspace=None,
                idx: Optional[torch.Tensor] = None, rows=None, stream=None, q_start=None,
                num_q: Optional[int] = None) -> torch.Tensor:
    """dsa_topk with scratch for sweeping long rows with several CTAs (include/dsa.h);
    ``workspace`` is a 256-B aligned device tensor (a fresh one of
    dsa_topk_workspace_size() bytes when None). Same selection as dsa_topk."""
    if q_start is None:
        T = kv.batch * q_per_seq
    elif num_q is not None:
        T = num_q
    elif idx is not None:
        T = idx.shape[0]
    else:
        raise ValueError("dsa_topk_ws on a ragged batch needs idx or num_q")
    if idx is None:
        idx = torch.empty(T, k, dtype=torch.int32, device=scores.device)
    if workspace is None:
        workspace = torch.empty(max(256, dsa_topk_workspace_size(kv, T, q_per_seq, k, rows,
                                                                 q_start)),
                                dtype=torch.uint8, device=scores.device)
    kvd, qd = kv.c(), _qdesc(T, q_per_seq, rows, q_start)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().dsa_topk_ws(_ptr(scores), scores.shape[1], ctypes.byref(kvd), ctypes.byref(qd),
                             k, _ptr(workspace), nbytes, _ptr(idx), _stream(stream)),
           "dsa_topk_ws")
    return idx


def dsa_sparse_mla_fwd(q, kv_cache, kv: KvLayout, q_per_seq: int, idx, scale: float,
                       out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                       rows=None, stream=None, q_start=None) -> Tuple[torch.Tensor, torch.Tensor]:
    T = q.shape[0]
    if out is None:
        out = torch.empty(T, HEADS, D_V, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(T, HEADS, dtype=torch.float32, device=q.device)
    kvd, qd = kv.c(), _qdesc(T, q_per_seq, rows, q_start)
    _check(lib().dsa_sparse_mla_fwd(_ptr(q), _ptr(kv_cache), ctypes.byref(kvd), ctypes.byref(qd),
                                    _ptr(idx), idx.shape[1], float(scale), _ptr(out), _ptr(lse),
                                    _stream(stream)), "dsa_sparse_mla_fwd")
    return out, lse


def dsa_sparse_mla_workspace_size() -> int:
    return int(lib().dsa_sparse_mla_workspace_size())


def dsa_sparse_mla_fwd_ws(q, kv_cache, kv: KvLayout, q_per_seq: int, idx, scale: float,
                          workspace: Optional[torch.Tensor] = None,
                          out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                          rows=None, stream=None, q_start=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """dsa_sparse_mla_fwd with scratch for splitting the rows of a partly filled
    last wave (include/dsa.h); ``workspace`` is any 256-B aligned device tensor
    (a fresh one of dsa_sparse_mla_workspace_size() bytes when None)."""
    T = q.shape[0]
    if workspace is None:
        workspace = torch.empty(dsa_sparse_mla_workspace_size(), dtype=torch.uint8,
                                device=q.device)
    if out is None:
        out = torch.empty(T, HEADS, D_V, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(T, HEADS, dtype=torch.float32, device=q.device)
    kvd, qd = kv.c(), _qdesc(T, q_per_seq, rows, q_start)
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().dsa_sparse_mla_fwd_ws(_ptr(q), _ptr(kv_cache), ctypes.byref(kvd),
                                       ctypes.byref(qd), _ptr(idx), idx.shape[1], float(scale),
                                       _ptr(workspace), nbytes, _ptr(out), _ptr(lse),
                                       _stream(stream)), "dsa_sparse_mla_fwd_ws")
    return out, lse


def dsa_indexer_kl(q, kv_cache, kv: KvLayout, q_per_seq: int, idx, scale: float, lse, scores,
                   kl: Optional[torch.Tensor] = None, rows=None, stream=None, q_start=None) -> torch.Tensor:
    """KL(p || softmax(I)) per row of the window (include/dsa.h): idx [T][k], lse
    [T][128] from dsa_sparse_mla_fwd, scores [batch * window rows][ld]."""
    T = q.shape[0]
    if kl is None:
        kl = torch.empty(kv.batch * _window(kv, q_per_seq, rows), dtype=torch.float32,
                         device=q.device)
    kvd, qd = kv.c(), _qdesc(T, q_per_seq, rows, q_start)
    _check(lib().dsa_indexer_kl(_ptr(q), _ptr(kv_cache), ctypes.byref(kvd), ctypes.byref(qd),
                                _ptr(idx), idx.shape[1], float(scale), _ptr(lse), _ptr(scores),
                                scores.shape[1], _ptr(kl), _stream(stream)), "dsa_indexer_kl")
    return kl


def dsa_workspace_size(kv: KvLayout, num_q: int, q_per_seq: int, k: int, rows=None,
                       q_start=None) -> int:
    kvd, qd = kv.c(), _qdesc(num_q, q_per_seq, rows, q_start)
    return int(lib().dsa_workspace_size(ctypes.byref(kvd), ctypes.byref(qd), k))


def dsa_forward(q_idx, w, k_idx, k_scale, q, kv_cache, kv: KvLayout, q_per_seq: int, k: int,
                scale: float, workspace: Optional[torch.Tensor] = None,
                idx_out: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                lse: Optional[torch.Tensor] = None, rows=None, stream=None, q_start=None):
    T = q.shape[0]
    if workspace is None:
        nbytes = dsa_workspace_size(kv, T, q_per_seq, k, rows, q_start)
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty(T, HEADS, D_V, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(T, HEADS, dtype=torch.float32, device=q.device)
    kvd, qd = kv.c(), _qdesc(T, q_per_seq, rows, q_start)
    _check(lib().dsa_forward(_ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(k_scale), _ptr(q),
                             _ptr(kv_cache), ctypes.byref(kvd), ctypes.byref(qd), k, float(scale),
                             _ptr(workspace), workspace.numel(), _ptr(idx_out), _ptr(out),
                             _ptr(lse), _stream(stream)), "dsa_forward")
    return out, lse, idx_out


def dsa_forward_noalloc(q_idx, w, k_idx, k_scale, q, kv_cache, kv: KvLayout, q_per_seq: int,
                        k: int, scale: float, idx_out: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                        rows=None, stream=None, q_start=None):
    """dsa_forward on the library's own fixed scratch array: the caller passes
    inputs and outputs only (see include/dsa.h for the limits)."""
    T = q.shape[0]
    if out is None:
        out = torch.empty(T, HEADS, D_V, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(T, HEADS, dtype=torch.float32, device=q.device)
    kvd, qd = kv.c(), _qdesc(T, q_per_seq, rows, q_start)
    _check(lib().dsa_forward_noalloc(_ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(k_scale), _ptr(q),
                                     _ptr(kv_cache), ctypes.byref(kvd), ctypes.byref(qd), k,
                                     float(scale), _ptr(idx_out), _ptr(out), _ptr(lse),
                                     _stream(stream)), "dsa_forward_noalloc")
    return out, lse, idx_out


# ---- fused indexer -> top-k (no stored score rows) -------------------------------------


def dsa_fused_workspace_size(kv: KvLayout, num_q: int, q_per_seq: int, k: int, rows=None,
                             q_start=None) -> int:
    kvd, qd = kv.c(), _qdesc(num_q, q_per_seq, rows, q_start)
    return int(lib().dsa_fused_workspace_size(ctypes.byref(kvd), ctypes.byref(qd), k))


def dsa_select_fused(q_idx, w, k_idx, k_scale, kv: KvLayout, q_per_seq: int, k: int,
                     cand_cap: int = 0, idx=None, workspace=None, rows=None, stream=None, q_start=None):
    """Selected positions [T, k] without stored score rows (include/dsa.h)."""
    T = q_idx.shape[0]
    if idx is None:
        idx = torch.empty(T, k, dtype=torch.int32, device=q_idx.device)
    if workspace is None:
        nbytes = dsa_fused_workspace_size(kv, T, q_per_seq, k, rows, q_start)
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q_idx.device)
    kvd, qd = kv.c(), _qdesc(T, q_per_seq, rows, q_start)
    _check(lib().dsa_select_fused(_ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(k_scale),
                                  ctypes.byref(kvd), ctypes.byref(qd), k, int(cand_cap),
                                  _ptr(workspace), workspace.numel(), _ptr(idx), _stream(stream)),
           "dsa_select_fused")
    return idx


def dsa_forward_fused(q_idx, w, k_idx, k_scale, q, kv_cache, kv: KvLayout, q_per_seq: int,
                      k: int, scale: float, cand_cap: int = 0, workspace=None, idx_out=None,
                      out=None, lse=None, rows=None, stream=None, q_start=None):
    T = q.shape[0]
    if workspace is None:
        nbytes = dsa_fused_workspace_size(kv, T, q_per_seq, k, rows, q_start)
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty(T, HEADS, D_V, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(T, HEADS, dtype=torch.float32, device=q.device)
    kvd, qd = kv.c(), _qdesc(T, q_per_seq, rows, q_start)
    _check(lib().dsa_forward_fused(_ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(k_scale), _ptr(q),
                                   _ptr(kv_cache), ctypes.byref(kvd), ctypes.byref(qd), k,
                                   float(scale), int(cand_cap), _ptr(workspace),
                                   workspace.numel(), _ptr(idx_out), _ptr(out), _ptr(lse),
                                   _stream(stream)), "dsa_forward_fused")
    return out, lse, idx_out


# ---- MLA in MHA mode (masked-MHA emulation of DSA for short prefill) -------------------

MHA_DN, MHA_DR, MHA_DV = 128, 64, 128


def mha_ctx_pad(kv: KvLayout) -> int:
    """Key slots per (sequence, head) of the decompressed keys and values."""
    return round_up(kv.max_ctx, 128)


def dsa_mla_up_project(kv_cache, w_uk, w_uv, kv: KvLayout, k_nope=None, k_rope=None, v=None,
                       stream=None):
    """Decompressed MHA-mode keys / values (include/dsa.h): k_nope [B,128,ctx_pad,128],
    k_rope [B,ctx_pad,64], v [B,128,ctx_pad,128], all bf16."""
    cp = mha_ctx_pad(kv)
    dev = kv_cache.device
    if k_nope is None:
        k_nope = torch.empty(kv.batch, HEADS, cp, MHA_DN, dtype=torch.bfloat16, device=dev)
    if k_rope is None:
        k_rope = torch.empty(kv.batch, cp, MHA_DR, dtype=torch.bfloat16, device=dev)
    if v is None:
        v = torch.empty(kv.batch, HEADS, cp, MHA_DV, dtype=torch.bfloat16, device=dev)
    kvd = kv.c()
    _check(lib().dsa_mla_up_project(_ptr(kv_cache), _ptr(w_uk), _ptr(w_uv), ctypes.byref(kvd),
                                    _ptr(k_nope), _ptr(k_rope), _ptr(v), k_nope.shape[2],
                                    _stream(stream)), "dsa_mla_up_project")
    return k_nope, k_rope, v


def dsa_selection_mask(idx, kv: KvLayout, q_per_seq: int, mask=None, rows=None, stream=None,
                       q_start=None):
    """Selection bits [T, mask_ld] uint32 (stored as int32) of the window's rows."""
    T, k = idx.shape
    if mask is None:
        mask = torch.zeros(T, mha_ctx_pad(kv) // 32, dtype=torch.int32, device=idx.device)
    kvd, qd = kv.c(), _qdesc(T, q_per_seq, rows, q_start)
    _check(lib().dsa_selection_mask(_ptr(idx), k, ctypes.byref(kvd), ctypes.byref(qd),
                                    _ptr(mask), mask.shape[1], _stream(stream)),
           "dsa_selection_mask")
    return mask


def dsa_masked_mha(q_mha, k_nope, k_rope, v, kv: KvLayout, q_per_seq: int, scale: float,
                   mask=None, k: int = 0, out=None, lse=None, rows=None, stream=None, q_start=None):
    """Masked MHA (include/dsa.h): out [T,128,128] bf16, lse [T,128] fp32."""
    T = q_mha.shape[0]
    if out is None:
        out = torch.empty(T, HEADS, MHA_DV, dtype=torch.bfloat16, device=q_mha.device)
    if lse is None:
        lse = torch.empty(T, HEADS, dtype=torch.float32, device=q_mha.device)
    kvd, qd = kv.c(), _qdesc(T, q_per_seq, rows, q_start)
    _check(lib().dsa_masked_mha(_ptr(q_mha), _ptr(k_nope), _ptr(k_rope), _ptr(v),
                                k_nope.shape[2], ctypes.byref(kvd), ctypes.byref(qd), _ptr(mask),
                                mask.shape[1] if mask is not None else 0, int(k), float(scale),
                                _ptr(out), _ptr(lse), _stream(stream)), "dsa_masked_mha")
    return out, lse


def dsa_mha_workspace_size(kv: KvLayout, num_q: int, q_per_seq: int, k: int, rows=None,
                           q_start=None) -> int:
    kvd, qd = kv.c(), _qdesc(num_q, q_per_seq, rows, q_start)
    return int(lib().dsa_mha_workspace_size(ctypes.byref(kvd), ctypes.byref(qd), k))


def dsa_mha_prefill(q_idx, w, k_idx, k_scale, q_mha, kv_cache, w_uk, w_uv, kv: KvLayout,
                    q_per_seq: int, k: int, scale: float, workspace=None, idx_out=None,
                    out=None, lse=None, rows=None, stream=None, q_start=None):
    """Short-prefill DSA in MHA mode: indexer -> top-k -> masks -> up-projection ->
    masked MHA, one call (include/dsa.h)."""
    T = q_mha.shape[0]
    if workspace is None:
        nbytes = dsa_mha_workspace_size(kv, T, q_per_seq, k, rows, q_start)
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q_mha.device)
    if out is None:
        out = torch.empty(T, HEADS, MHA_DV, dtype=torch.bfloat16, device=q_mha.device)
    if lse is None:
        lse = torch.empty(T, HEADS, dtype=torch.float32, device=q_mha.device)
    kvd, qd = kv.c(), _qdesc(T, q_per_seq, rows, q_start)
    _check(lib().dsa_mha_prefill(_ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(k_scale), _ptr(q_mha),
                                 _ptr(kv_cache), _ptr(w_uk), _ptr(w_uv), ctypes.byref(kvd),
                                 ctypes.byref(qd), k, float(scale), _ptr(workspace),
                                 workspace.numel(), _ptr(idx_out), _ptr(out), _ptr(lse),
                                 _stream(stream)), "dsa_mha_prefill")
    return out, lse, idx_out


def dsa_get_device_error(stream=None) -> int:
    return int(lib().dsa_get_device_error(_stream(stream)))


def dsa_set_wait_timeout_ns(ns: int) -> int:
    return int(lib().dsa_set_wait_timeout_ns(ns))


def dsa_selftest_wait_timeout(stream=None) -> int:
    return int(lib().dsa_selftest_wait_timeout(_stream(stream)))


def dsa_status_string(status: int) -> str:
    return lib().dsa_status_string(status).decode()
