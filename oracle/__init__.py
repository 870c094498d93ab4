"""Plain CPU oracle for indexed sparse attention over paged caches.

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the cpu-baseline /
reference legs of ``bench.py`` may import this package; the product path never does.  The
arithmetic lives in ``sia_oracle.c`` (plain C, fp64), which shares nothing with the CUDA
library; this module only compiles it with gcc and marshals numpy arrays into it.

Each wrapper names the step of the naive five-step decode chain ("Day 0 Inference Adaptation
and Performance Optimization for Hybrid Sparse Attention LLMs", section "Operator Fusion and
Multi-Stream Scheduling") that it computes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sia_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile sia_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP, strict fp)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.oracle_bf16_value.restype = ctypes.c_double
            lib.oracle_bf16_value.argtypes = [ctypes.c_uint16]
            lib.oracle_e4m3_value.restype = ctypes.c_double
            lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
            lib.oracle_e8m0_value.restype = ctypes.c_double
            lib.oracle_e8m0_value.argtypes = [ctypes.c_uint8]
            lib.oracle_index_scores_mx.restype = I
            lib.oracle_index_scores_mx.argtypes = [I, I, I, I, I, I, I, P, P, P, P, P, P, P, P, P,
                                                   I, P, P]
            lib.oracle_index_scores.restype = I
            lib.oracle_index_scores.argtypes = [I, I, I, I, I, I, I, I, P, P, P, P, P, P, P, P,
                                                P, I, P, P]
            lib.oracle_topk_row.restype = I
            lib.oracle_topk_row.argtypes = [P, I, I, P]
            lib.oracle_topk.restype = I
            lib.oracle_topk.argtypes = [P, P, ctypes.c_long, I, P, I, I, P]
            lib.oracle_sparse_attend.restype = I
            lib.oracle_sparse_attend.argtypes = [I, I, I, I, I, I, I, I, ctypes.c_double, P, P,
                                                 P, P, P, I, P, I, P, P]
            lib.oracle_sparse_attend_fp8kv.restype = I
            lib.oracle_sparse_attend_fp8kv.argtypes = [I, I, I, I, I, I, I, I, ctypes.c_double, P,
                                                       P, P, P, P, P, I, P, I, P, P]
            lib.oracle_dense_masked_attend.restype = I
            lib.oracle_dense_masked_attend.argtypes = [I, I, I, I, I, I, I, I, ctypes.c_double,
                                                       P, P, P, P, P, P, P, P]
            lib.oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
            lib.oracle_cache_append.restype = I
            lib.oracle_cache_append.argtypes = [I, I, I, I, I, I, I, P, P, P, I, P, P, P, I, P, P]
            lib.oracle_num_threads.restype = I
            lib.oracle_set_num_threads.argtypes = [I]
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def _raw16(a):
    """bf16 data as its uint16 bit patterns (accepts a torch tensor or a numpy array)."""
    if hasattr(a, "view") and hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        import torch
        return np.ascontiguousarray(a.contiguous().view(torch.int16).numpy().view(np.uint16))
    return np.ascontiguousarray(a, dtype=np.uint16)


def _raw8(a):
    """e4m3 data as its uint8 codes (accepts a torch float8 tensor or a numpy array)."""
    if hasattr(a, "view") and hasattr(a, "dtype") and "float8" in str(a.dtype):
        import torch
        return np.ascontiguousarray(a.contiguous().view(torch.uint8).numpy())
    return np.ascontiguousarray(a, dtype=np.uint8)


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def bf16_value(bits: int) -> float:
    return _load().oracle_bf16_value(int(bits))


def e4m3_value(code: int) -> float:
    return _load().oracle_e4m3_value(int(code))


def e4m3_encode(x: float) -> int:
    """e4m3 code of an fp32 value: nearest grid value, ties to even, saturating at 448."""
    return _load().oracle_e4m3_encode(float(x))


def cache_append(new_k, new_kv, page_table, seq_lens, k_cache, kv_cache, *, page_size,
                 k_mode="bf16", k_scale=None, kv_scale=None):
    """The step before scoring: write the J new tokens of every sequence into the paged caches
    (token j of sequence b at position seq_lens[b] - J + j), in place.

    new_k [B,J,D] and new_kv [B,J,DC] are float values (fp32, or bf16 tensors).  k_mode:
    "bf16" (k_cache uint16 bits), "fp8" (e4m3 codes + per-token power-of-two fp32 scale in
    k_scale [pages,P]) or "mx" (e4m3 codes + E8M0 codes in k_scale uint8 [pages,P,D/32]).
    kv_scale None: kv_cache holds bf16 bits; else e4m3 codes + fp32 scale per 128-element
    block (kv_scale [pages,P,ceil(DC/128)]).  Every array is a contiguous numpy array, updated
    in place.  Returns the status.
    """
    nk = np.ascontiguousarray(np.asarray(new_k.float() if hasattr(new_k, "float") else new_k,
                                         dtype=np.float32))
    nv = np.ascontiguousarray(np.asarray(new_kv.float() if hasattr(new_kv, "float") else new_kv,
                                         dtype=np.float32))
    B, J, D = nk.shape
    DC = nv.shape[2]
    mode = {"bf16": 0, "fp8": 1, "mx": 2}[k_mode]
    for a in (k_cache, kv_cache, k_scale, kv_scale):
        if a is not None and not (isinstance(a, np.ndarray) and a.flags.c_contiguous):
            raise ValueError("caches and scales must be contiguous numpy arrays")
    pt, sl = _c(page_table, np.int32), _c(seq_lens, np.int32)
    return _load().oracle_cache_append(B, J, D, DC, page_size, pt.shape[1], k_cache.shape[0],
                                       _ptr(pt), _ptr(sl), _ptr(nk), mode, _ptr(k_cache),
                                       _ptr(k_scale), _ptr(nv), 0 if kv_scale is None else 1,
                                       _ptr(kv_cache), _ptr(kv_scale))


def e8m0_value(code: int) -> float:
    return _load().oracle_e8m0_value(int(code))


def _rows_arg(rows):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(rows, dtype=np.int32)
    return r, int(r.size)


def index_scores(q, w, k_cache, page_table, seq_lens, *, page_size, fp8=False, q_scale=None,
                 k_scale=None, q_pos=None, rows=None):
    """Steps 1-2 (score, head-weighted sum) over the causal history of every query.

    q [B,J,H,D] (bf16 bits or e4m3 codes), w [B,J,H] fp32, k_cache [num_pages,P,D],
    page_table [B,max_pages] int32, seq_lens [B] int32.  Returns (scores fp64 [B,J,Lpad] with
    NaN past the query position, n_visible int32 [B,J], status).
    """
    B, J, H, D = q.shape
    num_pages = k_cache.shape[0]
    max_pages = page_table.shape[1]
    raw = _raw8 if fp8 else _raw16
    qa, ka = raw(q), raw(k_cache)
    wa = _c(w, np.float32)
    pt, sl = _c(page_table, np.int32), _c(seq_lens, np.int32)
    qp = _c(q_pos, np.int32)
    qs, ks = _c(q_scale, np.float32), _c(k_scale, np.float32)
    r, nr = _rows_arg(rows)
    Lpad = max_pages * page_size
    scores = np.full((B, J, Lpad), np.nan, dtype=np.float64)
    nvis = np.zeros((B, J), dtype=np.int32)
    st = _load().oracle_index_scores(B, J, H, D, page_size, max_pages, num_pages, int(bool(fp8)),
                                     _ptr(qa), _ptr(qs), _ptr(wa), _ptr(ka), _ptr(ks), _ptr(pt),
                                     _ptr(sl), _ptr(qp), _ptr(r), nr, _ptr(scores), _ptr(nvis))
    return scores, nvis, st


def topk_row(scores_row, n_visible, k):
    """Step 3 for one query: ascending positions of the K best scores, -1 padded."""
    s = np.ascontiguousarray(scores_row, dtype=np.float64)
    out = np.empty(k, dtype=np.int32)
    _load().oracle_topk_row(_ptr(s), int(n_visible), int(k), _ptr(out))
    return out


def topk(scores, n_visible, k, rows=None):
    """Step 3 for every (b, j): scores [B,J,Lpad] fp64 -> int32 [B,J,K]."""
    B, J, Lpad = scores.shape
    s = np.ascontiguousarray(scores, dtype=np.float64)
    nv = _c(n_visible, np.int32)
    r, nr = _rows_arg(rows)
    out = np.full((B, J, k), -1, dtype=np.int32)
    _load().oracle_topk(_ptr(s), _ptr(nv), Lpad, int(k), _ptr(r), nr, B * J, _ptr(out))
    return out


def index_scores_mx(q, q_mx, w, k_cache, k_mx, page_table, seq_lens, *, page_size, q_pos=None,
                    rows=None):
    """Steps 1-2 on the MXFP8 index path: e4m3 codes with one E8M0 scale per 32 elements.

    q [B,J,H,D] e4m3, q_mx [B,J,H,D/32] E8M0 (uint8 codes or torch float8_e8m0fnu), w [B,J,H]
    fp32, k_cache [num_pages,P,D] e4m3, k_mx [num_pages,P,D/32] E8M0.  Returns (scores fp64
    [B,J,Lpad] with NaN past the query position, n_visible int32 [B,J], status).
    """
    B, J, H, D = q.shape
    num_pages = k_cache.shape[0]
    max_pages = page_table.shape[1]
    qa, ka, qm, km = _raw8(q), _raw8(k_cache), _raw8(q_mx), _raw8(k_mx)
    if qm.shape != (B, J, H, D // 32) or km.shape != (num_pages, k_cache.shape[1], D // 32):
        raise ValueError("one E8M0 scale per 32 elements of q and of each key is expected")
    wa = _c(w, np.float32)
    pt, sl = _c(page_table, np.int32), _c(seq_lens, np.int32)
    qp = _c(q_pos, np.int32)
    r, nr = _rows_arg(rows)
    Lpad = max_pages * page_size
    scores = np.full((B, J, Lpad), np.nan, dtype=np.float64)
    nvis = np.zeros((B, J), dtype=np.int32)
    st = _load().oracle_index_scores_mx(B, J, H, D, page_size, max_pages, num_pages, _ptr(qa),
                                        _ptr(qm), _ptr(wa), _ptr(ka), _ptr(km), _ptr(pt), _ptr(sl),
                                        _ptr(qp), _ptr(r), nr, _ptr(scores), _ptr(nvis))
    return scores, nvis, st


def index_topk(q, w, k_cache, page_table, seq_lens, *, page_size, top_k, fp8=False,
               q_scale=None, k_scale=None, q_pos=None, rows=None):
    """Steps 1-3: (topk int32 [B,J,K], scores fp64 [B,J,Lpad], status)."""
    scores, nvis, st = index_scores(q, w, k_cache, page_table, seq_lens, page_size=page_size,
                                    fp8=fp8, q_scale=q_scale, k_scale=k_scale, q_pos=q_pos,
                                    rows=rows)
    return topk(scores, nvis, top_k, rows=rows), scores, st


def sparse_attend(q, kv_cache, page_table, seq_lens, topk_idx, *, page_size, d_latent, scale,
                  rows=None, kv_scale=None):
    """Steps 4-5: gather the selected latent rows and attend (fp64).

    q [B,J,H,DL+DR] bf16, kv_cache [num_pages,P,DL+DR] bf16, topk [B,J,K] int32.  With
    kv_scale (fp32 [num_pages,P,ceil((DL+DR)/128)]) the cache holds e4m3 codes instead and each
    element is its decoded code times the scale of its 128-element block of the token's row.
    Returns (out fp64 [B,J,H,DL], lse fp64 [B,J,H], status).
    """
    B, J, H, DC = q.shape
    DL = int(d_latent)
    DR = DC - DL
    K = topk_idx.shape[-1]
    qa = _raw16(q)
    pt, sl = _c(page_table, np.int32), _c(seq_lens, np.int32)
    tk = _c(topk_idx, np.int32)
    r, nr = _rows_arg(rows)
    out = np.zeros((B, J, H, DL), dtype=np.float64)
    lse = np.full((B, J, H), np.nan, dtype=np.float64)
    if kv_scale is None:
        kva = _raw16(kv_cache)
        st = _load().oracle_sparse_attend(B, J, H, DL, DR, page_size, page_table.shape[1],
                                          kv_cache.shape[0], float(scale), _ptr(qa), _ptr(kva),
                                          _ptr(pt), _ptr(sl), _ptr(tk), K, _ptr(r), nr, _ptr(out),
                                          _ptr(lse))
    else:
        kva = _raw8(kv_cache)
        nblk = (DC + 127) // 128
        ks = _c(kv_scale, np.float32)
        if ks.shape != (kv_cache.shape[0], kv_cache.shape[1], nblk):
            raise ValueError("kv_scale must be [num_pages, P, %d]" % nblk)
        st = _load().oracle_sparse_attend_fp8kv(B, J, H, DL, DR, page_size, page_table.shape[1],
                                                kv_cache.shape[0], float(scale), _ptr(qa),
                                                _ptr(kva), _ptr(ks), _ptr(pt), _ptr(sl), _ptr(tk), K,
                                                _ptr(r), nr, _ptr(out), _ptr(lse))
    return out, lse, st


def dense_masked_attend(q, kv_cache, page_table, seq_lens, allowed, *, page_size, d_latent,
                        scale, q_pos=None):
    """Independent dense formulation: causal attention with -inf outside `allowed`.

    allowed: bool/uint8 [B,J,Lpad].  Returns (out fp64 [B,J,H,DL], lse fp64 [B,J,H], status).
    """
    B, J, H, DC = q.shape
    DL = int(d_latent)
    DR = DC - DL
    qa, kva = _raw16(q), _raw16(kv_cache)
    pt, sl = _c(page_table, np.int32), _c(seq_lens, np.int32)
    qp = _c(q_pos, np.int32)
    al = np.ascontiguousarray(allowed, dtype=np.uint8)
    out = np.zeros((B, J, H, DL), dtype=np.float64)
    lse = np.full((B, J, H), np.nan, dtype=np.float64)
    st = _load().oracle_dense_masked_attend(B, J, H, DL, DR, page_size, page_table.shape[1],
                                            kv_cache.shape[0], float(scale), _ptr(qa), _ptr(kva),
                                            _ptr(pt), _ptr(sl), _ptr(qp), _ptr(al), _ptr(out),
                                            _ptr(lse))
    return out, lse, st
