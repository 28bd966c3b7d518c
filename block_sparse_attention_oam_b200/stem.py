"""Thin ctypes binding of libstem (include/stem.h).

Argument marshalling only: torch tensors provide device memory and the current
CUDA stream; every step of the path runs in libstem's CUDA kernels.  There is no
fallback: if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import re
from typing import Optional, Sequence

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libstem.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "stem.h")

STEM_OK, STEM_ERR_INVALID, STEM_ERR_UNSUPPORTED, STEM_ERR_WORKSPACE, STEM_ERR_CUDA, STEM_ERR_TIMEOUT, STEM_ERR_BOUNDS = range(7)
DT_BF16, DT_FP8 = 0, 1
PAGE_SIZE = 64


class StemError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"libstem status {status}: {message}")
        self.status = status


class _Problem(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int),
        ("cu_seqlens", ctypes.POINTER(ctypes.c_int32)),
        ("num_q_heads", ctypes.c_int),
        ("num_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("block_size", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("q_scale", ctypes.c_float),
        ("k_scale", ctypes.c_float),
        ("v_scale", ctypes.c_float),
        ("softmax_scale", ctypes.c_float),
        ("beta", ctypes.c_float),
        ("keep", ctypes.c_double),
        ("mu", ctypes.c_double),
        ("shared_lists", ctypes.c_int),
    ]


class _Paged(ctypes.Structure):
    _fields_ = [
        ("k_cache", ctypes.c_void_p),
        ("v_cache", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p),
        ("page_size", ctypes.c_int),
        ("max_pages_per_seq", ctypes.c_int),
        ("num_slots", ctypes.c_int),
    ]


class _Sizes(ctypes.Structure):
    _fields_ = [
        ("num_rows", ctypes.c_int64),
        ("scores_per_head", ctypes.c_int64),
        ("nnz_per_head", ctypes.c_int64),
        ("total_tokens", ctypes.c_int64),
        ("workspace_bytes", ctypes.c_size_t),
        ("list_heads", ctypes.c_int64),
    ]


_lib = None
_P = ctypes.c_void_p


def lib() -> ctypes.CDLL:
    """Load libstem.so (built in-tree by build.py).  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m block_sparse_attention_oam_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    pp = ctypes.POINTER(_Problem)
    pg = ctypes.POINTER(_Paged)
    sig = {
        "stem_query_sizes": ([pp, ctypes.POINTER(_Sizes)], ctypes.c_int),
        "stem_workspace_size": ([pp], ctypes.c_size_t),
        "stem_tpd_plan": ([ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.POINTER(ctypes.c_double),
                           ctypes.POINTER(ctypes.c_int64)], ctypes.c_int),
        "stem_score": ([pp, _P, _P, _P, pg, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
        "stem_select": ([pp, _P, _P, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
        "stem_score_select": ([pp, _P, _P, _P, pg, _P, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
        "bsa_prefill": ([pp, _P, _P, _P, pg, _P, _P, _P, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
        "bsa_dense_prefill": ([pp, _P, _P, _P, pg, _P, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
        "stem_attention": ([pp, _P, _P, _P, pg, _P, _P, _P, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
        "stem_attention_noalloc": ([pp, _P, _P, _P, pg, _P, _P, _P, _P, _P, _P], ctypes.c_int),
        "stem_attention_host": ([pp, _P, _P, _P, _P, _P, _P, pg, _P, _P, _P, _P, _P, ctypes.c_int, _P,
                                 ctypes.c_size_t, _P], ctypes.c_int),
        "stem_query_status": ([_P, _P], ctypes.c_int),
        "stem_reset_status": ([_P, _P], ctypes.c_int),
        "stem_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "stem_last_error": ([], ctypes.c_char_p),
        "stem_debug_inject": ([ctypes.c_int], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def header_functions() -> list:
    """Names of the functions include/stem.h declares."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*STEM_API\s+(?:const\s+)?[A-Za-z_][\w]*\s*\*?\s+\**([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)


def _check(status: int) -> None:
    if status != STEM_OK:
        msg = lib().stem_last_error().decode()
        raise StemError(status, msg or lib().stem_status_string(status).decode())


@dataclasses.dataclass
class Problem:
    cu_seqlens: Sequence[int]
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str = "bf16"
    q_scale: float = 1.0
    k_scale: float = 1.0
    v_scale: float = 1.0
    softmax_scale: float = 0.0
    beta: float = 0.2
    keep: float = 0.25
    mu: float = 0.7
    shared_lists: bool = False   # one selection per KV group (an extension, not in the pages)

    def __post_init__(self):
        self._cu = np.ascontiguousarray(np.asarray(self.cu_seqlens, dtype=np.int32))
        self._c = _Problem(len(self._cu) - 1, self._cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                           self.num_q_heads, self.num_kv_heads, self.head_dim, self.block_size,
                           DT_FP8 if self.dtype == "fp8_e4m3" else DT_BF16,
                           self.q_scale, self.k_scale, self.v_scale, self.softmax_scale, self.beta,
                           self.keep, self.mu, 1 if self.shared_lists else 0)

    @property
    def c(self):
        return ctypes.byref(self._c)

    def sizes(self) -> dict:
        s = _Sizes()
        _check(lib().stem_query_sizes(self.c, ctypes.byref(s)))
        return dict(num_rows=s.num_rows, scores_per_head=s.scores_per_head, nnz_per_head=s.nnz_per_head,
                    total_tokens=s.total_tokens, workspace_bytes=s.workspace_bytes, list_heads=s.list_heads)


@dataclasses.dataclass
class PagedKV:
    k_cache: torch.Tensor       # [num_slots, 64, Hkv, d]
    v_cache: torch.Tensor
    block_table: torch.Tensor   # int32 [num_seqs, max_pages] on the device

    def c(self):
        return ctypes.byref(_Paged(self.k_cache.data_ptr(), self.v_cache.data_ptr(), self.block_table.data_ptr(),
                                   PAGE_SIZE, self.block_table.shape[1], self.k_cache.shape[0]))


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("libstem takes dense row-major tensors; got a non-contiguous one")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _paged(paged: Optional[PagedKV]):
    return None if paged is None else paged.c()


def tpd_plan(n_blocks: int, keep: float, mu: float):
    r = ctypes.c_double()
    t = ctypes.c_int64()
    _check(lib().stem_tpd_plan(n_blocks, keep, mu, ctypes.byref(r), ctypes.byref(t)))
    return r.value, t.value


def workspace(prob: Problem, device="cuda") -> torch.Tensor:
    n = prob.sizes()["workspace_bytes"]
    ws = torch.zeros(n, dtype=torch.uint8, device=device)
    return ws


def stem_score(prob: Problem, q, k, v, paged: Optional[PagedKV] = None, scores=None, ws=None, stream=None):
    sz = prob.sizes()
    if scores is None:
        scores = torch.empty((prob.num_q_heads, sz["scores_per_head"]), dtype=torch.float32, device=q.device)
    ws = workspace(prob, q.device) if ws is None else ws
    _check(lib().stem_score(prob.c, _ptr(q), _ptr(k), _ptr(v), _paged(paged), _ptr(scores), _ptr(ws),
                            ws.numel(), _stream(stream)))
    return scores


def stem_select(prob: Problem, scores, row_ptr=None, col_idx=None, ws=None, stream=None):
    sz = prob.sizes()
    dev = scores.device
    if row_ptr is None:
        row_ptr = torch.empty(sz["num_rows"] + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        col_idx = torch.empty((sz["list_heads"], sz["nnz_per_head"]), dtype=torch.int32, device=dev)
    ws = workspace(prob, dev) if ws is None else ws
    _check(lib().stem_select(prob.c, _ptr(scores), _ptr(row_ptr), _ptr(col_idx), _ptr(ws), ws.numel(),
                             _stream(stream)))
    return row_ptr, col_idx


def stem_score_select(prob: Problem, q, k, v, paged: Optional[PagedKV] = None, row_ptr=None, col_idx=None, ws=None,
                      stream=None):
    """Pool, score and select in one pass (no score matrix): returns (row_ptr, col_idx)."""
    sz = prob.sizes()
    dev = q.device
    if row_ptr is None:
        row_ptr = torch.empty(sz["num_rows"] + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        col_idx = torch.empty((sz["list_heads"], sz["nnz_per_head"]), dtype=torch.int32, device=dev)
    ws = workspace(prob, dev) if ws is None else ws
    _check(lib().stem_score_select(prob.c, _ptr(q), _ptr(k), _ptr(v), _paged(paged), _ptr(row_ptr), _ptr(col_idx),
                                   _ptr(ws), ws.numel(), _stream(stream)))
    return row_ptr, col_idx


def _out(prob, q, out):
    if out is None:
        out = torch.empty((q.shape[0], prob.num_q_heads, prob.head_dim), dtype=torch.bfloat16, device=q.device)
    return out


def bsa_prefill(prob: Problem, q, k, v, row_ptr, col_idx, paged: Optional[PagedKV] = None, out=None, lse=None,
                ws=None, stream=None):
    out = _out(prob, q, out)
    ws = workspace(prob, q.device) if ws is None else ws
    _check(lib().bsa_prefill(prob.c, _ptr(q), _ptr(k), _ptr(v), _paged(paged), _ptr(row_ptr), _ptr(col_idx),
                             _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def bsa_dense_prefill(prob: Problem, q, k, v, paged: Optional[PagedKV] = None, out=None, lse=None, ws=None,
                      stream=None):
    out = _out(prob, q, out)
    ws = workspace(prob, q.device) if ws is None else ws
    _check(lib().bsa_dense_prefill(prob.c, _ptr(q), _ptr(k), _ptr(v), _paged(paged), _ptr(out), _ptr(lse),
                                   _ptr(ws), ws.numel(), _stream(stream)))
    return out


def stem_attention(prob: Problem, q, k, v, paged: Optional[PagedKV] = None, out=None, lse=None, row_ptr=None,
                   col_idx=None, ws=None, stream=None):
    out = _out(prob, q, out)
    ws = workspace(prob, q.device) if ws is None else ws
    _check(lib().stem_attention(prob.c, _ptr(q), _ptr(k), _ptr(v), _paged(paged), _ptr(out), _ptr(lse),
                                _ptr(row_ptr), _ptr(col_idx), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def capture_attention(prob: Problem, q, k, v, paged: Optional[PagedKV] = None, out=None, lse=None, row_ptr=None,
                      col_idx=None, ws=None):
    """Capture one stem_attention call (pooling, scoring, selection, BSA: every kernel of
    the path) into a CUDA graph on these buffers.  `graph.replay()` re-runs the whole path
    on whatever the buffers hold at replay time, with one launch from the host.  The
    problem (sequence lengths, heads, knobs) is fixed by the capture.  Returns (graph, out)."""
    out = _out(prob, q, out)
    ws = workspace(prob, q.device) if ws is None else ws
    side = torch.cuda.Stream(device=q.device)
    side.wait_stream(torch.cuda.current_stream(q.device))
    with torch.cuda.stream(side):  # one eager call first: kernel attributes and the budget plan
        stem_attention(prob, q, k, v, paged, out, lse, row_ptr, col_idx, ws)
    torch.cuda.current_stream(q.device).wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        stem_attention(prob, q, k, v, paged, out, lse, row_ptr, col_idx, ws)
    return graph, out


def stem_attention_host(prob: Problem, q_host, k_host, v_host, q, k, v, paged: Optional[PagedKV] = None,
                        out_host=None, out=None, lse=None, row_ptr=None, col_idx=None, out_groups: int = 0, ws=None,
                        stream=None):
    """The whole path from host tensors: q_host / k_host / v_host (CPU, ideally pinned)
    go to the device and O comes back into out_host (CPU bf16 [T, Hq, d]), one group of
    kv-heads at a time, the copies of each group overlapping the work of the others.
    q / k / v / out (a paged cache: paged.k_cache / paged.v_cache) are device scratch
    of the full sizes, overwritten with the inputs staged group by group.  Returns
    out_host; the work is asynchronous on `stream` (synchronise before reading it)."""
    out = _out(prob, q, out)
    if out_host is None:
        out_host = torch.empty(tuple(out.shape), dtype=torch.bfloat16, pin_memory=True)
    for t, name in ((q_host, "q_host"), (k_host, "k_host"), (v_host, "v_host"), (out_host, "out_host")):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous host tensor")
    ws = workspace(prob, q.device) if ws is None else ws
    _check(lib().stem_attention_host(prob.c, _ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(q), _ptr(k), _ptr(v),
                                     _paged(paged), _ptr(out_host), _ptr(out), _ptr(lse), _ptr(row_ptr),
                                     _ptr(col_idx), int(out_groups), _ptr(ws), ws.numel(), _stream(stream)))
    return out_host


def stem_attention_noalloc(prob: Problem, q, k, v, paged: Optional[PagedKV] = None, out=None, lse=None,
                           row_ptr=None, col_idx=None, status=None, stream=None):
    """stem_attention with the library's static scratch instead of a workspace
    (for callers that cannot allocate device memory).  `status`: optional device
    int32 tensor of one element that receives the call's device status word."""
    out = _out(prob, q, out)
    _check(lib().stem_attention_noalloc(prob.c, _ptr(q), _ptr(k), _ptr(v), _paged(paged), _ptr(out), _ptr(lse),
                                        _ptr(row_ptr), _ptr(col_idx), _ptr(status), _stream(stream)))
    return out


def debug_inject(mode: int) -> None:
    """Failure-detection test hook: mode 1 makes the next BSA launch stall one CTA
    until its bounded wait reports STEM_ERR_TIMEOUT."""
    _check(lib().stem_debug_inject(mode))


def query_status(ws, stream=None) -> int:
    """Synchronise, read and clear the device status word; raises on a device error."""
    st = lib().stem_query_status(_ptr(ws), _stream(stream))
    _check(st)
    return st


def problem_for(wl, inputs=None, keep=None) -> Problem:
    """Problem description of a workload (workloads.Workload) and its inputs."""
    cu = np.zeros(len(wl.seqlens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(wl.seqlens)
    kw = {}
    if inputs is not None and wl.dtype == "fp8_e4m3":
        kw = dict(q_scale=inputs.q_scale, k_scale=inputs.k_scale, v_scale=inputs.v_scale)
    return Problem(cu, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block, wl.dtype, beta=wl.beta,
                   keep=wl.keep if keep is None else keep, mu=wl.mu, shared_lists=wl.shared_lists, **kw)
