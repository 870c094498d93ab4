"""Host logic of the Zigzag context-parallel prefill (indexed_sparse_attention_paged_b200.
cp_prefill) on CPU ranks: the shards and positions each rank takes match the pages' pairing (as
the oracle restates it), and two or three gloo ranks that exchange their new cache rows with the
all-gather, compute their own queries and restore the token order reproduce the whole chunk
computed in one piece.  The compute calls here go through a test-side backend built on the oracle;
on a GPU the same host logic drives libsia's kernels (tests/test_cp_prefill_gpu.py)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from oracle import zigzag
from indexed_sparse_attention_paged_b200 import cp_prefill, workloads


@pytest.mark.parametrize("T,N", [(0, 2), (5, 2), (17, 4), (64, 8), (1000, 3), (16384, 8)])
def test_rank_tokens_follow_the_pairing(T, N):
    got = [cp_prefill.rank_tokens(T, N, r).tolist() for r in range(N)]
    assert got == zigzag.card_positions(T, N)
    assert [cp_prefill.rank_shards(N, r) for r in range(N)] == [tuple(p) for p in zigzag.assignment(N)]


def test_restore_order_inverts_the_split():
    T, N = 37, 3
    parts = [cp_prefill.rank_tokens(T, N, r).float().unsqueeze(1) * 10 for r in range(N)]
    out = cp_prefill.restore_order(parts, T, N)
    assert torch.equal(out[:, 0], torch.arange(T).float() * 10)


class OracleBackend:
    """Test-side stand-in for the CUDA backend: the same three calls through the oracle."""

    def __init__(self, page_size, top_k, d_latent, scale):
        self.P, self.K, self.DL, self.scale = page_size, top_k, d_latent, scale

    def append(self, new_k, new_kv, page_table, seq_lens, k_cache, kv_cache):
        kn = k_cache.view(torch.int16).numpy().view(np.uint16)
        vn = kv_cache.view(torch.int16).numpy().view(np.uint16)
        assert oracle.cache_append(new_k, new_kv, page_table.numpy(), seq_lens.numpy(), kn, vn, page_size=self.P) == 0

    def index_topk(self, q_idx, w, k_cache, page_table, seq_lens, q_pos):
        topk, _, st = oracle.index_topk(q_idx, w.numpy(), k_cache, page_table.numpy(), seq_lens.numpy(),
                                        page_size=self.P, top_k=self.K,
                                        q_pos=None if q_pos is None else q_pos.numpy())
        assert st == 0
        return torch.from_numpy(topk)

    def attend(self, q_attn, kv_cache, page_table, seq_lens, topk):
        out, _, st = oracle.sparse_attend(q_attn, kv_cache, page_table.numpy(), seq_lens.numpy(), topk.numpy(),
                                          page_size=self.P, d_latent=self.DL, scale=self.scale)
        assert st == 0
        return torch.from_numpy(out)


def chunk(T, seed=31):
    """A prefill chunk of T tokens shaped like the tiny workload (page size 16, indexer 4 x 32,
    8 attention heads over 64 + 16): the new cache rows and the queries of every token."""
    wl = workloads.WORKLOADS[1]
    h = workloads.make_inputs(wl, seed=seed, seq_lens=[T], n_q=T)
    g = torch.Generator().manual_seed(seed + 1)
    new_k = torch.randint(-3, 4, (T, wl.idx_dim), generator=g).to(torch.bfloat16)
    new_kv = torch.randn((T, wl.d_latent + wl.d_rope), generator=g).to(torch.bfloat16)
    return wl, h, new_k, new_kv


def reference(T, top_k):
    """The whole chunk in one piece: every token appended, every query ranked and attended."""
    wl, h, new_k, new_kv = chunk(T)
    be = OracleBackend(wl.page_size, top_k, wl.d_latent, wl.softmax_scale)
    k = torch.zeros_like(h["k_cache"])
    kv = torch.zeros_like(h["kv_cache"])
    sl = torch.tensor([T], dtype=torch.int32)
    be.append(new_k.unsqueeze(0), new_kv.unsqueeze(0), h["page_table"], sl, k, kv)
    topk = be.index_topk(h["q_idx"], h["w"], k, h["page_table"], sl, None)
    return be.attend(h["q_attn"], kv, h["page_table"], sl, topk)[0]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, T, top_k, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl, h, new_k, new_kv = chunk(T)
        mine = cp_prefill.rank_tokens(T, world, rank).long()
        be = OracleBackend(wl.page_size, top_k, wl.d_latent, wl.softmax_scale)
        k = torch.zeros_like(h["k_cache"])
        kv = torch.zeros_like(h["kv_cache"])
        cp = cp_prefill.ZigzagPrefill(be)
        assert (cp.N, cp.rank) == (world, rank)
        own, full = cp.run(T, new_k[mine], new_kv[mine], h["q_idx"][0, mine], h["w"][0, mine],
                           h["q_attn"][0, mine], h["page_table"], k, kv)
        q.put((rank, own, full))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("T,world", [(96, 2), (100, 3)])
def test_gloo_ranks_reproduce_the_whole_chunk(T, world):
    top_k = 24
    ref = reference(T, top_k)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, T, top_k, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict()
    for _ in range(world):
        r, own, full = q.get(timeout=240)
        got[r] = (own, full)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        own, full = got[r]
        assert torch.equal(full, ref)                       # every rank holds the whole chunk's result
        assert torch.equal(own, ref[cp_prefill.rank_tokens(T, world, r).long()])
