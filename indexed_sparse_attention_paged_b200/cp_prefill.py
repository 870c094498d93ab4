"""Context-parallel prefill of one long chunk across ranks, with the Zigzag pairing.

"Day0 Inference Adaptation and Performance Optimization for New-Architecture LLMs" (section 5.2)
and "Day0 Inference Adaptation and Performance Optimization for a New Hybrid-Attention LLM
Architecture" (section 4.3) split a long prefill chunk over N cards for context parallelism: the
chunk's T tokens are cut into 2N shards and card i takes shards i and 2N-1-i, so that every card
gets one shard from the light (early) end of the causal triangle and one from the heavy (late)
end; the index keys and latent KV that every card needs are exchanged with one all-gather, and the
per-card results are put back in token order at the end.

The steps on each rank (one process per GPU, torch.distributed for the collectives):
  1. all-gather the rank's new index keys and latent rows (padded to the largest rank share, so
     one fixed-size collective each) and reassemble them in token order;
  2. write all T tokens into this rank's own paged caches (sia_cache_append: the chunk is
     sequence 0 with seq_len = T, so token t goes to position t);
  3. score and rank only the rank's own queries (sia_sparse_index_topk with q_pos = their token
     positions; each query sees the causal history 0..t of the whole chunk), then attend
     (sia_sparse_mla_attend);
  4. all-gather the outputs and restore the token order.

Every step of the computation runs in libsia's CUDA kernels; this module only moves tensors.
The three compute calls go through a backend object so that the host logic (shards, gathers,
order) can also be driven on CPU ranks in tests.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def zigzag_shards(T: int, N: int) -> List[Tuple[int, int]]:
    """The 2N contiguous shards of a T-token chunk, as even as possible (the pages leave ragged
    chunks open; here the first T mod 2N shards take one token more)."""
    if N < 1 or T < 0:
        raise ValueError("need N >= 1 and T >= 0")
    S = 2 * N
    base, extra = divmod(T, S)
    out, start = [], 0
    for s in range(S):
        end = start + base + (1 if s < extra else 0)
        out.append((start, end))
        start = end
    return out


def rank_shards(N: int, rank: int) -> Tuple[int, int]:
    """The two shards card `rank` takes: rank and 2N - 1 - rank."""
    if not 0 <= rank < N:
        raise ValueError("rank %d outside [0, %d)" % (rank, N))
    return rank, 2 * N - 1 - rank


def rank_tokens(T: int, N: int, rank: int) -> torch.Tensor:
    """Token positions of card `rank`'s queries, in the order its outputs are produced: its
    first shard, then its second."""
    sh = zigzag_shards(T, N)
    a, b = rank_shards(N, rank)
    return torch.cat([torch.arange(*sh[a]), torch.arange(*sh[b])]).to(torch.int32)


def restore_order(parts: Sequence[torch.Tensor], T: int, N: int) -> torch.Tensor:
    """Put per-rank results (rank r's rows in rank_tokens order) back in token order."""
    if len(parts) != N:
        raise ValueError("one part per rank is expected")
    out = torch.empty((T,) + tuple(parts[0].shape[1:]), dtype=parts[0].dtype, device=parts[0].device)
    for r, p in enumerate(parts):
        idx = rank_tokens(T, N, r).to(torch.long).to(p.device)
        if p.shape[0] != idx.numel():
            raise ValueError("rank %d part has %d rows, expected %d" % (r, p.shape[0], idx.numel()))
        out[idx] = p
    return out


def _all_gather_padded(x: torch.Tensor, counts: Sequence[int], group) -> List[torch.Tensor]:
    """All-gather rank shares of different lengths along dim 0 with one fixed-size collective
    (each share padded to the largest)."""
    N = len(counts)
    m = max(counts)
    pad = torch.zeros((m,) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    pad[: x.shape[0]] = x
    if N == 1:
        return [pad[: counts[0]]]
    if dist.get_backend(group) == "nccl":
        buf = torch.empty((N * m,) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
        dist.all_gather_into_tensor(buf, pad, group=group)
        return [buf[r * m: r * m + counts[r]] for r in range(N)]
    # other backends (gloo on CPU ranks): a list all-gather of the raw bytes, since gloo does not
    # take every element type (bf16, fp8, int16)
    raw = pad.reshape(m, -1).view(torch.uint8)
    bufs = [torch.empty_like(raw) for _ in range(N)]
    dist.all_gather(bufs, raw, group=group)
    return [b.view(x.dtype).reshape(pad.shape)[: counts[r]] for r, b in enumerate(bufs)]


class CudaBackend:
    """The three compute calls of a rank, through libsia's C ABI on the rank's GPU."""

    def __init__(self, *, page_size: int, top_k: int, d_latent: int, softmax_scale: float):
        import indexed_sparse_attention_paged_b200 as sia
        self.sia = sia
        self.page_size, self.top_k, self.d_latent, self.softmax_scale = page_size, top_k, d_latent, softmax_scale

    def append(self, new_k, new_kv, page_table, seq_lens, k_cache, kv_cache):
        self.sia.cache_append(new_k, new_kv, page_table, seq_lens, k_cache, kv_cache)

    def index_topk(self, q_idx, w, k_cache, page_table, seq_lens, q_pos):
        return self.sia.sparse_index_topk(q_idx, w, k_cache, page_table, seq_lens, top_k=self.top_k, q_pos=q_pos)

    def attend(self, q_attn, kv_cache, page_table, seq_lens, topk):
        return self.sia.sparse_mla_attend(q_attn, kv_cache, page_table, seq_lens, topk, d_latent=self.d_latent,
                                          softmax_scale=self.softmax_scale)


class ZigzagPrefill:
    """One rank's part of a context-parallel prefill chunk (see the module docstring)."""

    def __init__(self, backend, group=None):
        self.backend = backend
        self.group = group
        self.N = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if self.N > 1 else 0

    def run(self, T: int, new_k: torch.Tensor, new_kv: torch.Tensor, q_idx: torch.Tensor, w: torch.Tensor,
            q_attn: torch.Tensor, page_table: torch.Tensor, k_cache: torch.Tensor, kv_cache: torch.Tensor,
            gather_output: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
        """new_k [n_r, D] / new_kv [n_r, DC] (bf16): this rank's tokens' new cache rows;
        q_idx [n_r, H, D], w [n_r, H], q_attn [n_r, Ha, DC]: its queries (rank_tokens order).
        page_table [1, max_pages] int32 and this rank's caches k_cache [pages, P, D],
        kv_cache [pages, P, DC] (bf16).  Returns (this rank's outputs [n_r, Ha, d_latent], the
        whole chunk's outputs in token order [T, Ha, d_latent] or None)."""
        N, r = self.N, self.rank
        mine = rank_tokens(T, N, r)
        n_r = mine.numel()
        for name, t in (("new_k", new_k), ("new_kv", new_kv), ("q_idx", q_idx), ("w", w), ("q_attn", q_attn)):
            if t.shape[0] != n_r:
                raise ValueError("%s has %d rows; rank %d owns %d tokens" % (name, t.shape[0], r, n_r))
        counts = [rank_tokens(T, N, i).numel() for i in range(N)]
        # 1. one all-gather per cache, then token order
        ks = _all_gather_padded(new_k, counts, self.group)
        vs = _all_gather_padded(new_kv, counts, self.group)
        full_k = restore_order(ks, T, N)
        full_kv = restore_order(vs, T, N)
        out = self.rank_compute(T, N, r, full_k, full_kv, q_idx, w, q_attn, page_table, k_cache, kv_cache)
        if not gather_output:
            return out, None
        # 4. every rank's outputs, back in token order
        parts = _all_gather_padded(out, counts, self.group)
        return out, restore_order(parts, T, N)

    def rank_compute(self, T, N, r, full_k, full_kv, q_idx, w, q_attn, page_table, k_cache, kv_cache):
        """Steps 2-3 for rank r of N, given the whole chunk's new rows in token order."""
        dev = full_k.device
        # 2. the whole chunk into this rank's paged caches: sequence 0, seq_len = T
        seq_lens = torch.tensor([T], dtype=torch.int32, device=dev)
        self.backend.append(full_k.unsqueeze(0).contiguous(), full_kv.unsqueeze(0).contiguous(), page_table,
                            seq_lens, k_cache, kv_cache)
        # 3. this rank's queries only, each at its own token position
        q_pos = rank_tokens(T, N, r).to(dev).unsqueeze(0).contiguous()
        topk = self.backend.index_topk(q_idx.unsqueeze(0).contiguous(), w.unsqueeze(0).contiguous(), k_cache,
                                       page_table, seq_lens, q_pos)
        return self.backend.attend(q_attn.unsqueeze(0).contiguous(), kv_cache, page_table, seq_lens, topk)[0]
