"""Seeded synthetic workloads shaped like the pages' decode / prefill / speculative cases.

This module only draws random inputs (on the CPU, with ``torch.Generator``) and holds none of
the method's arithmetic.  Both the CUDA path and the CPU oracle are fed from it, so they see
identical bytes.

Input recipe:
  * index q and index k: integers drawn uniformly from [-3, 3], stored as bf16 or as FP8 E4M3
    (exact either way);
  * head weights w: integers drawn uniformly from [-2, 2], fp32;
  * per-token index-k scale (FP8 cases): 2**e with e drawn uniformly from [-4, 4];
  * attention q and latent KV rows: N(0, 1) rounded to bf16;
  * page ids: one random permutation of the whole page pool, handed out sequence by sequence
    (the page table is therefore "shuffled"); unused page-table slots hold -1;
  * variable context lengths (quantised decode): uniform integers in [1024, 32768].
Seed = 1000 + the workload's number, so every run draws the same tensors.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    number: int
    name: str
    batch: int
    n_q: int                 # query tokens per sequence (J)
    context: int             # context length; 0 = drawn per sequence from [len_lo, len_hi]
    page_size: int
    idx_heads: int
    idx_dim: int
    idx_fp8: bool
    top_k: int
    attn_heads: int
    d_latent: int
    d_rope: int
    len_lo: int = 0
    len_hi: int = 0
    causal_prefill: bool = False   # query j sits at position j (a chunk of T tokens)

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.d_latent + self.d_rope)


WORKLOADS = {
    1: Workload(1, "tiny_decode_b1_ctx256", 1, 1, 256, 16, 4, 32, False, 16, 8, 64, 16),
    2: Workload(2, "decode_b32_ctx8k", 32, 1, 8192, 64, 64, 128, False, 2048, 128, 512, 64),
    3: Workload(3, "fp8_index_decode_b128_ctx1k_32k", 128, 1, 0, 64, 64, 128, True, 2048, 128,
                512, 64, len_lo=1024, len_hi=32768),
    4: Workload(4, "causal_prefill_t16k", 1, 16384, 16384, 64, 64, 128, False, 2048, 128, 512, 64,
                causal_prefill=True),
    5: Workload(5, "spec_decode_b8_ctx128k_j2", 8, 2, 131072, 64, 64, 128, True, 2048, 128, 512,
                64),
}


def _randint(gen, lo, hi, shape):
    """Integers uniform in [lo, hi] (both ends included)."""
    return torch.randint(lo, hi + 1, shape, generator=gen, dtype=torch.int32)


def _randn_bf16(gen, shape, chunk_rows=1 << 16):
    """N(0,1) rounded to bf16, drawn in chunks along dim 0 to bound host memory."""
    out = torch.empty(shape, dtype=torch.bfloat16)
    flat = out.view(shape[0], -1)
    for s in range(0, shape[0], chunk_rows):
        e = min(shape[0], s + chunk_rows)
        flat[s:e] = torch.randn((e - s, flat.shape[1]), generator=gen, dtype=torch.float32).to(torch.bfloat16)
    return out


def make_inputs(wl: Workload, seed: Optional[int] = None, *, batch: Optional[int] = None,
                context: Optional[int] = None, n_q: Optional[int] = None,
                seq_lens: Optional[list] = None) -> dict:
    """Draw one workload's inputs as CPU tensors.

    `batch`, `context`, `n_q` and `seq_lens` override the workload's sizes (used to make the
    small and ragged parity cases); the drawing recipe stays the same.
    """
    seed = 1000 + wl.number if seed is None else seed
    gen = torch.Generator().manual_seed(seed)
    B = wl.batch if batch is None else batch
    J = wl.n_q if n_q is None else n_q
    P = wl.page_size
    if seq_lens is not None:
        lens = torch.tensor(seq_lens, dtype=torch.int32)
        B = lens.numel()
    elif wl.context == 0 and context is None:
        lens = _randint(gen, wl.len_lo, wl.len_hi, (B,))
    else:
        L = wl.context if context is None else context
        lens = torch.full((B,), L, dtype=torch.int32)
    pages_per_seq = [(int(l) + P - 1) // P for l in lens]
    max_pages = max(1, max(pages_per_seq))
    num_pages = max(1, sum(pages_per_seq))
    perm = torch.randperm(num_pages, generator=gen).to(torch.int32)
    page_table = torch.full((B, max_pages), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(pages_per_seq):
        page_table[b, :n] = perm[off:off + n]
        off += n

    Hi, Di = wl.idx_heads, wl.idx_dim
    q_idx = _randint(gen, -3, 3, (B, J, Hi, Di)).to(torch.float32)
    k_idx = _randint(gen, -3, 3, (num_pages, P, Di)).to(torch.float32)
    w = _randint(gen, -2, 2, (B, J, Hi)).to(torch.float32)
    if wl.idx_fp8:
        q_idx = q_idx.to(torch.float8_e4m3fn)
        k_idx = k_idx.to(torch.float8_e4m3fn)
        k_scale = torch.pow(2.0, _randint(gen, -4, 4, (num_pages, P)).to(torch.float32))
    else:
        q_idx = q_idx.to(torch.bfloat16)
        k_idx = k_idx.to(torch.bfloat16)
        k_scale = None

    Ha, DC = wl.attn_heads, wl.d_latent + wl.d_rope
    q_attn = _randn_bf16(gen, (B * J * Ha, DC)).view(B, J, Ha, DC)
    kv_cache = _randn_bf16(gen, (num_pages * P, DC)).view(num_pages, P, DC)

    # query j of sequence b sits at position seq_len - J + j (for the prefill chunk J = L, so
    # query j sits at position j); no explicit position array is needed
    return dict(workload=wl, batch=B, n_q=J, seq_lens=lens, page_table=page_table,
                num_pages=num_pages, max_pages=max_pages, q_idx=q_idx, w=w, k_cache=k_idx,
                k_scale=k_scale, q_pos=None, q_attn=q_attn, kv_cache=kv_cache)


def fp8_main_cache(inputs: dict, seed: Optional[int] = None, pow2_scales: bool = False) -> dict:
    """The same workload with its main latent cache drawn in the FP8 format instead: e4m3 codes
    (N(0, 100^2) samples cast to e4m3, saturating at 448, so that the codes use the format's
    range) and one fp32 scale per 128-element block of each row (uniform in [1/110, 1/90), or a
    power of two 2^e with e uniform in [-7, -6]).  The decoded values have about the spread of
    the bf16 cache's N(0, 1)."""
    wl = inputs["workload"]
    seed = 2000 + wl.number if seed is None else seed
    gen = torch.Generator().manual_seed(seed)
    pages, P, DC = inputs["kv_cache"].shape
    nblk = (DC + 127) // 128
    codes = torch.empty((pages, P, DC), dtype=torch.float8_e4m3fn)
    flat = codes.view(pages * P, DC)
    for s0 in range(0, pages * P, 1 << 16):
        e = min(pages * P, s0 + (1 << 16))
        flat[s0:e] = (torch.randn((e - s0, DC), generator=gen) * 100.0).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    if pow2_scales:
        scale = torch.pow(2.0, _randint(gen, -7, -6, (pages, P, nblk)).to(torch.float32))
    else:
        scale = torch.rand((pages, P, nblk), generator=gen) * (1.0 / 90 - 1.0 / 110) + 1.0 / 110
    out = dict(inputs)
    out["kv_cache"] = codes
    out["kv_scale"] = scale
    return out


def to_device(inputs: dict, device) -> dict:
    out = {}
    for k, v in inputs.items():
        out[k] = v.to(device) if isinstance(v, torch.Tensor) else v
    return out
