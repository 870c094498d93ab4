"""indexed_sparse_attention_paged_b200 -- Python binding of libsia (include/sia.h).

Indexed sparse attention over paged caches on B200 (sm_100a): a lightweight indexer scores
every causal history position from a paged index-K cache as
``I[t,s] = sum_h w[t,h] * ReLU(q[t,h] . k[s])`` and keeps each query's Top-K positions; an
MLA-style attention then gathers only those latent rows from the paged main KV cache.

This module only marshals arguments: it checks tensor dtypes, shapes and devices, allocates
outputs and workspaces with torch when the caller passes none, and calls the C ABI.  Every
step of the computation runs in the CUDA kernels of ``libsia.so``; there is no CPU or
PyTorch fallback, and importing the binding fails loudly when the library is missing.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

from . import workloads  # noqa: F401  (seeded inputs for tests and the benchmark)

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsia.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "sia.h")

SIA_OK, SIA_ERR_INVALID_ARGUMENT, SIA_ERR_UNSUPPORTED, SIA_ERR_CUDA, SIA_ERR_WORKSPACE = range(5)
SIA_DEV_BAD_PAGE, SIA_DEV_BAD_POSITION, SIA_DEV_TIMEOUT, SIA_DEV_INTERNAL = 0x1, 0x2, 0x4, 0x8
SIA_BF16, SIA_FP8_E4M3, SIA_MXFP8 = 0, 1, 2
SIA_KEY_BF16, SIA_KEY_FP8_POW2, SIA_KEY_MXFP8 = 0, 1, 2
SIA_KV_BF16, SIA_KV_FP8_BLOCK128 = 0, 1


class SiaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


class IndexArgs(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("max_pages_per_seq", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("q", ctypes.c_void_p), ("q_scale", ctypes.c_void_p), ("w", ctypes.c_void_p),
                ("k_cache", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
                ("page_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("q_pos", ctypes.c_void_p), ("topk_out", ctypes.c_void_p),
                ("scores_out", ctypes.c_void_p), ("q_mx", ctypes.c_void_p), ("k_mx", ctypes.c_void_p)]


class AttendArgs(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("d_latent", ctypes.c_int32), ("d_rope", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float),
                ("q", ctypes.c_void_p), ("kv_cache", ctypes.c_void_p),
                ("page_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("topk", ctypes.c_void_p), ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("kv_scale", ctypes.c_void_p)]


class AppendArgs(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("d_kv", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("max_pages_per_seq", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("key_format", ctypes.c_int32), ("kv_format", ctypes.c_int32),
                ("new_k", ctypes.c_void_p), ("new_kv", ctypes.c_void_p),
                ("page_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("k_cache", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
                ("kv_cache", ctypes.c_void_p), ("kv_scale", ctypes.c_void_p)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libsia.so (built by ``build()``); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError("libsia.so not found at %s: run `python -m indexed_sparse_attention_paged_b200.build`"
                          % path)
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.sia_index_workspace_size.restype = ctypes.c_size_t
    lib.sia_index_workspace_size.argtypes = [ctypes.POINTER(IndexArgs)]
    lib.sia_attend_workspace_size.restype = ctypes.c_size_t
    lib.sia_attend_workspace_size.argtypes = [ctypes.POINTER(AttendArgs)]
    lib.sia_workspace_size.restype = ctypes.c_size_t
    lib.sia_workspace_size.argtypes = [ctypes.POINTER(IndexArgs), ctypes.POINTER(AttendArgs)]
    lib.sia_sparse_index_topk.restype = ctypes.c_int
    lib.sia_sparse_index_topk.argtypes = [ctypes.POINTER(IndexArgs), P, ctypes.c_size_t, P, P]
    lib.sia_index_scores.restype = ctypes.c_int
    lib.sia_index_scores.argtypes = [ctypes.POINTER(IndexArgs), P, P]
    lib.sia_sparse_index_topk_noalloc.restype = ctypes.c_int
    lib.sia_sparse_index_topk_noalloc.argtypes = [ctypes.POINTER(IndexArgs), P, P]
    lib.sia_sparse_mla_attend.restype = ctypes.c_int
    lib.sia_sparse_mla_attend.argtypes = [ctypes.POINTER(AttendArgs), P, ctypes.c_size_t, P, P]
    lib.sia_fused_decode.restype = ctypes.c_int
    lib.sia_fused_decode.argtypes = [ctypes.POINTER(IndexArgs), ctypes.POINTER(AttendArgs), P,
                                     ctypes.c_size_t, P, P]
    lib.sia_status_string.restype = ctypes.c_char_p
    lib.sia_status_string.argtypes = [ctypes.c_int]
    lib.sia_last_error.restype = ctypes.c_char_p
    lib.sia_version.restype = ctypes.c_int32
    lib.sia_cache_append.restype = ctypes.c_int
    lib.sia_cache_append.argtypes = [ctypes.POINTER(AppendArgs), P, P]
    lib.sia_set_wait_limit_ns.restype = ctypes.c_uint64
    lib.sia_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    _lib = lib
    return lib


def header_functions(path: str = HEADER_PATH):
    """Names of the functions include/sia.h declares."""
    with open(path) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(sia_\w+)\s*\(", text, re.M)))


def set_wait_limit_ns(ns: int) -> int:
    """Bound of every in-kernel wait of later calls (0 = the default two seconds); returns the
    previous bound.  Only for testing the timeout path."""
    return int(load_library().sia_set_wait_limit_ns(int(ns)))


def _check(status: int):
    if status != SIA_OK:
        lib = load_library()
        raise SiaError(status, "%s: %s" % (lib.sia_status_string(status).decode(),
                                           lib.sia_last_error().decode()))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype=None, dim=None, device=None):
    if t is None:
        raise ValueError("%s is required" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError("%s must have dtype %s (got %s)" % (name, dtype, t.dtype))
    if dim is not None and t.dim() != dim:
        raise ValueError("%s must have %d dims (got %d)" % (name, dim, t.dim()))
    if device is not None and t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))
    return t


def index_args(q, w, k_cache, page_table, seq_lens, *, top_k, q_scale=None, k_scale=None,
               q_pos=None, topk_out=None, scores_out=None, q_mx=None, k_mx=None) -> IndexArgs:
    """Fill the stage-1 argument struct from tensors (see sia_index_args in include/sia.h).
    With q_mx and k_mx (E8M0 codes, uint8 or float8_e8m0fnu, one per 32 elements) the e4m3 q and
    k_cache are the MXFP8 index path."""
    _need(q, "q", (torch.bfloat16, torch.float8_e4m3fn), 4)
    dev = q.device
    B, J, H, D = q.shape
    fp8 = q.dtype == torch.float8_e4m3fn
    _need(k_cache, "k_cache", q.dtype, 3, dev)
    _need(w, "w", torch.float32, 3, dev)
    _need(page_table, "page_table", torch.int32, 2, dev)
    _need(seq_lens, "seq_lens", torch.int32, 1, dev)
    if q_scale is not None:
        _need(q_scale, "q_scale", torch.float32, 2, dev)
    if k_scale is not None:
        _need(k_scale, "k_scale", torch.float32, 2, dev)
    if q_pos is not None:
        _need(q_pos, "q_pos", torch.int32, 2, dev)
    if topk_out is not None:
        _need(topk_out, "topk_out", torch.int32, 3, dev)
    if scores_out is not None:
        _need(scores_out, "scores_out", torch.float32, 3, dev)
    mx = q_mx is not None or k_mx is not None
    if mx:
        if not fp8:
            raise ValueError("the MXFP8 path takes e4m3 q and k_cache")
        _need(q_mx, "q_mx", (torch.uint8, torch.float8_e8m0fnu), 4, dev)
        _need(k_mx, "k_mx", (torch.uint8, torch.float8_e8m0fnu), 3, dev)
        if tuple(q_mx.shape) != (B, J, H, D // 32) or tuple(k_mx.shape) != (k_cache.shape[0], k_cache.shape[1], D // 32):
            raise ValueError("one E8M0 scale per 32 elements of q and of each key is expected")
    a = IndexArgs()
    a.batch, a.n_q, a.n_heads, a.head_dim = B, J, H, D
    a.page_size = k_cache.shape[1]
    a.max_pages_per_seq = page_table.shape[1]
    a.num_pages = k_cache.shape[0]
    a.top_k = int(top_k)
    a.dtype = SIA_MXFP8 if mx else (SIA_FP8_E4M3 if fp8 else SIA_BF16)
    a.q, a.q_scale, a.w = _ptr(q), _ptr(q_scale), _ptr(w)
    a.k_cache, a.k_scale = _ptr(k_cache), _ptr(k_scale)
    a.page_table, a.seq_lens, a.q_pos = _ptr(page_table), _ptr(seq_lens), _ptr(q_pos)
    a.topk_out, a.scores_out = _ptr(topk_out), _ptr(scores_out)
    a.q_mx, a.k_mx = _ptr(q_mx), _ptr(k_mx)
    return a


def attend_args(q, kv_cache, page_table, seq_lens, topk, *, d_latent, softmax_scale, out=None,
                lse=None, kv_scale=None) -> AttendArgs:
    """Fill the stage-2 argument struct from tensors (see sia_attend_args in include/sia.h).
    With kv_scale (fp32 [pages, P, ceil(DC/128)]) kv_cache holds FP8 E4M3 codes."""
    _need(q, "q", torch.bfloat16, 4)
    dev = q.device
    B, J, H, DC = q.shape
    if kv_scale is None:
        _need(kv_cache, "kv_cache", torch.bfloat16, 3, dev)
    else:
        _need(kv_cache, "kv_cache", (torch.float8_e4m3fn, torch.uint8), 3, dev)
        _need(kv_scale, "kv_scale", torch.float32, 3, dev)
        if tuple(kv_scale.shape) != (kv_cache.shape[0], kv_cache.shape[1], (DC + 127) // 128):
            raise ValueError("kv_scale must be [num_pages, page_size, ceil(DC / 128)]")
    _need(page_table, "page_table", torch.int32, 2, dev)
    _need(seq_lens, "seq_lens", torch.int32, 1, dev)
    _need(topk, "topk", torch.int32, 3, dev)
    if out is not None:
        _need(out, "out", torch.bfloat16, 4, dev)
    if lse is not None:
        _need(lse, "lse", torch.float32, 3, dev)
    a = AttendArgs()
    a.batch, a.n_q, a.n_heads = B, J, H
    a.d_latent, a.d_rope = int(d_latent), DC - int(d_latent)
    a.page_size = kv_cache.shape[1]
    a.max_pages_per_seq = page_table.shape[1]
    a.num_pages = kv_cache.shape[0]
    a.top_k = topk.shape[-1]
    a.softmax_scale = float(softmax_scale)
    a.q, a.kv_cache = _ptr(q), _ptr(kv_cache)
    a.page_table, a.seq_lens, a.topk = _ptr(page_table), _ptr(seq_lens), _ptr(topk)
    a.out, a.lse = _ptr(out), _ptr(lse)
    a.kv_scale = _ptr(kv_scale)
    return a


def _workspace(nbytes: int, device, workspace):
    if nbytes == 0:
        return workspace
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError("workspace needs %d bytes" % nbytes)
        return workspace
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _ws_ptr(ws):
    return (ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size()) if ws is not None else (None, 0)


def sparse_index_topk(q, w, k_cache, page_table, seq_lens, *, top_k, q_scale=None, k_scale=None,
                      q_pos=None, topk_out=None, scores_out=None, workspace=None, dev_status=None,
                      stream=None, q_mx=None, k_mx=None):
    """Stage 1: Top-K positions per query, int32 [B, J, top_k] (ascending, -1 padded)."""
    lib = load_library()
    B, J = q.shape[:2]
    if topk_out is None:
        topk_out = torch.empty((B, J, int(top_k)), dtype=torch.int32, device=q.device)
    a = index_args(q, w, k_cache, page_table, seq_lens, top_k=top_k, q_scale=q_scale,
                   k_scale=k_scale, q_pos=q_pos, topk_out=topk_out, scores_out=scores_out,
                   q_mx=q_mx, k_mx=k_mx)
    ws = _workspace(lib.sia_index_workspace_size(ctypes.byref(a)), q.device, workspace)
    wp, wn = _ws_ptr(ws)
    _check(lib.sia_sparse_index_topk(ctypes.byref(a), wp, wn, _ptr(dev_status), _stream_ptr(stream)))
    return topk_out


def index_scores(q, w, k_cache, page_table, seq_lens, *, scores_out, q_scale=None, k_scale=None,
                 q_pos=None, dev_status=None, stream=None, q_mx=None, k_mx=None):
    """The scoring step alone: I[t, s] for every causal position into `scores_out`
    (fp32 [B, J, max_pages_per_seq * page_size]; positions past a query's own are untouched)."""
    lib = load_library()
    a = index_args(q, w, k_cache, page_table, seq_lens, top_k=1, q_scale=q_scale, k_scale=k_scale,
                   q_pos=q_pos, topk_out=None, scores_out=scores_out, q_mx=q_mx, k_mx=k_mx)
    _check(lib.sia_index_scores(ctypes.byref(a), _ptr(dev_status), _stream_ptr(stream)))
    return scores_out


def sparse_index_topk_noalloc(q, w, k_cache, page_table, seq_lens, *, top_k, topk_out, q_scale=None,
                              k_scale=None, q_pos=None, dev_status=None, stream=None):
    """Stage 1 through the entry point that allocates nothing (its score scratch is a fixed
    16 MiB array inside the library, shared by every call).  `topk_out` must be given."""
    lib = load_library()
    a = index_args(q, w, k_cache, page_table, seq_lens, top_k=top_k, q_scale=q_scale,
                   k_scale=k_scale, q_pos=q_pos, topk_out=topk_out)
    _check(lib.sia_sparse_index_topk_noalloc(ctypes.byref(a), _ptr(dev_status), _stream_ptr(stream)))
    return topk_out


def sparse_mla_attend(q, kv_cache, page_table, seq_lens, topk, *, d_latent, softmax_scale,
                      out=None, lse=None, workspace=None, dev_status=None, stream=None, kv_scale=None):
    """Stage 2: bf16 [B, J, H, d_latent] attention output (and lse when given a buffer)."""
    lib = load_library()
    B, J, H, _ = q.shape
    if out is None:
        out = torch.empty((B, J, H, int(d_latent)), dtype=torch.bfloat16, device=q.device)
    a = attend_args(q, kv_cache, page_table, seq_lens, topk, d_latent=d_latent,
                    softmax_scale=softmax_scale, out=out, lse=lse, kv_scale=kv_scale)
    ws = _workspace(lib.sia_attend_workspace_size(ctypes.byref(a)), q.device, workspace)
    wp, wn = _ws_ptr(ws)
    _check(lib.sia_sparse_mla_attend(ctypes.byref(a), wp, wn, _ptr(dev_status), _stream_ptr(stream)))
    return out


def cache_append(new_k, new_kv, page_table, seq_lens, k_cache, kv_cache, *, key_format=SIA_KEY_BF16,
                 kv_format=None, k_scale=None, kv_scale=None, dev_status=None, stream=None):
    """Write the J new tokens of every sequence (bf16 new_k [B,J,D], new_kv [B,J,DC]) into the
    paged caches in place, quantising as the formats say (see sia_cache_append in
    include/sia.h).  kv_format defaults to FP8 when kv_scale is given, else bf16."""
    lib = load_library()
    _need(new_k, "new_k", torch.bfloat16, 3)
    dev = new_k.device
    _need(new_kv, "new_kv", torch.bfloat16, 3, dev)
    _need(page_table, "page_table", torch.int32, 2, dev)
    _need(seq_lens, "seq_lens", torch.int32, 1, dev)
    key_dtype = torch.bfloat16 if key_format == SIA_KEY_BF16 else torch.float8_e4m3fn
    _need(k_cache, "k_cache", (key_dtype, torch.uint8) if key_dtype != torch.bfloat16 else key_dtype, 3, dev)
    if kv_format is None:
        kv_format = SIA_KV_BF16 if kv_scale is None else SIA_KV_FP8_BLOCK128
    kv_dtype = torch.bfloat16 if kv_format == SIA_KV_BF16 else (torch.float8_e4m3fn, torch.uint8)
    _need(kv_cache, "kv_cache", kv_dtype, 3, dev)
    if k_scale is not None:
        _need(k_scale, "k_scale", torch.float32 if key_format == SIA_KEY_FP8_POW2 else
              (torch.uint8, torch.float8_e8m0fnu), None, dev)
    if kv_scale is not None:
        _need(kv_scale, "kv_scale", torch.float32, 3, dev)
    B, J, D = new_k.shape
    a = AppendArgs()
    a.batch, a.n_q, a.head_dim, a.d_kv = B, J, D, new_kv.shape[2]
    a.page_size, a.max_pages_per_seq, a.num_pages = k_cache.shape[1], page_table.shape[1], k_cache.shape[0]
    a.key_format, a.kv_format = int(key_format), int(kv_format)
    a.new_k, a.new_kv = _ptr(new_k), _ptr(new_kv)
    a.page_table, a.seq_lens = _ptr(page_table), _ptr(seq_lens)
    a.k_cache, a.k_scale, a.kv_cache, a.kv_scale = _ptr(k_cache), _ptr(k_scale), _ptr(kv_cache), _ptr(kv_scale)
    _check(lib.sia_cache_append(ctypes.byref(a), _ptr(dev_status), _stream_ptr(stream)))


def fused_decode_workspace_size(ia: IndexArgs, aa: AttendArgs) -> int:
    return load_library().sia_workspace_size(ctypes.byref(ia), ctypes.byref(aa))


def fused_decode(q_idx, w, k_cache, q_attn, kv_cache, page_table, seq_lens, *, top_k, d_latent,
                 softmax_scale, q_scale=None, k_scale=None, q_pos=None, topk_out=None, out=None,
                 lse=None, workspace=None, dev_status=None, stream=None, kv_scale=None, q_mx=None,
                 k_mx=None):
    """Both stages in one call: returns (out bf16 [B,J,H,d_latent], topk int32 [B,J,K])."""
    lib = load_library()
    B, J = q_idx.shape[:2]
    H = q_attn.shape[2]
    if topk_out is None:
        topk_out = torch.empty((B, J, int(top_k)), dtype=torch.int32, device=q_idx.device)
    if out is None:
        out = torch.empty((B, J, H, int(d_latent)), dtype=torch.bfloat16, device=q_idx.device)
    ia = index_args(q_idx, w, k_cache, page_table, seq_lens, top_k=top_k, q_scale=q_scale,
                    k_scale=k_scale, q_pos=q_pos, topk_out=topk_out, q_mx=q_mx, k_mx=k_mx)
    aa = attend_args(q_attn, kv_cache, page_table, seq_lens, topk_out, d_latent=d_latent,
                     softmax_scale=softmax_scale, out=out, lse=lse, kv_scale=kv_scale)
    ws = _workspace(lib.sia_workspace_size(ctypes.byref(ia), ctypes.byref(aa)), q_idx.device, workspace)
    wp, wn = _ws_ptr(ws)
    _check(lib.sia_fused_decode(ctypes.byref(ia), ctypes.byref(aa), wp, wn, _ptr(dev_status),
                                _stream_ptr(stream)))
    return out, topk_out


class FusedDecodePlan:
    """A fused-decode call with every buffer allocated once (workspace, outputs), so that each
    step is one C-ABI call with no allocation -- what the benchmark times and what a serving loop
    would capture in a CUDA graph."""

    def __init__(self, inputs: dict, device, *, with_lse: bool = True, out=None, lse=None, topk=None):
        wl = inputs["workload"]
        self.inputs = inputs
        B, J = inputs["batch"], inputs["n_q"]
        self.topk = topk if topk is not None else torch.empty((B, J, wl.top_k), dtype=torch.int32, device=device)
        self.out = out if out is not None else torch.empty((B, J, wl.attn_heads, wl.d_latent), dtype=torch.bfloat16,
                                                           device=device)
        if lse is not None:
            self.lse = lse
        else:
            self.lse = torch.empty((B, J, wl.attn_heads), dtype=torch.float32, device=device) if with_lse else None
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.ia = index_args(inputs["q_idx"], inputs["w"], inputs["k_cache"], inputs["page_table"],
                             inputs["seq_lens"], top_k=wl.top_k, k_scale=inputs["k_scale"],
                             q_pos=inputs.get("q_pos"), topk_out=self.topk, q_mx=inputs.get("q_mx"),
                             k_mx=inputs.get("k_mx"))
        self.aa = attend_args(inputs["q_attn"], inputs["kv_cache"], inputs["page_table"],
                              inputs["seq_lens"], self.topk, d_latent=wl.d_latent,
                              softmax_scale=wl.softmax_scale, out=self.out, lse=self.lse,
                              kv_scale=inputs.get("kv_scale"))
        lib = load_library()
        n = lib.sia_workspace_size(ctypes.byref(self.ia), ctypes.byref(self.aa))
        self.ws = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
        self._ws = _ws_ptr(self.ws)
        self._lib = lib

    def __call__(self, stream=None):
        _check(self._lib.sia_fused_decode(ctypes.byref(self.ia), ctypes.byref(self.aa), self._ws[0],
                                          self._ws[1], _ptr(self.status), _stream_ptr(stream)))
        return self.out
