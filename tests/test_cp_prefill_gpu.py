"""The Zigzag context-parallel prefill's per-rank compute on a B200 (libsia kernels): with one
GPU, the ranks of an N-card split are emulated one after another (each writes the whole chunk
into its own caches and computes its own queries at their positions; no rank waits on another),
and their outputs, put back in token order, must match the oracle's whole-chunk result.  A
world-size-1 NCCL process group also drives the full run() path (all-gathers included)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from indexed_sparse_attention_paged_b200 import cp_prefill, workloads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _chunk(T, seed=41):
    wl = workloads.WORKLOADS[2]
    h = workloads.make_inputs(wl, seed=seed, seq_lens=[T], n_q=T)
    g = torch.Generator().manual_seed(seed + 1)
    new_k = torch.randint(-3, 4, (T, wl.idx_dim), generator=g).to(torch.bfloat16)
    new_kv = torch.randn((T, wl.d_latent + wl.d_rope), generator=g).to(torch.bfloat16)
    return wl, h, new_k, new_kv


def _oracle_chunk(wl, h, new_k, new_kv, T, top_k):
    k = np.zeros(tuple(h["k_cache"].shape), np.uint16)
    kv = np.zeros(tuple(h["kv_cache"].shape), np.uint16)
    pt, sl = h["page_table"].numpy(), np.array([T], np.int32)
    assert oracle.cache_append(new_k.unsqueeze(0), new_kv.unsqueeze(0), pt, sl, k, kv, page_size=wl.page_size) == 0
    kt = torch.from_numpy(k.view(np.int16)).view(torch.bfloat16)
    kvt = torch.from_numpy(kv.view(np.int16)).view(torch.bfloat16)
    topk, _, st = oracle.index_topk(h["q_idx"], h["w"].numpy(), kt, pt, sl, page_size=wl.page_size, top_k=top_k)
    assert st == 0
    out, _, st = oracle.sparse_attend(h["q_attn"], kvt, pt, sl, topk, page_size=wl.page_size, d_latent=wl.d_latent,
                                      scale=wl.softmax_scale)
    assert st == 0
    return out[0]


@pytest.mark.parametrize("T,N,top_k", [(1000, 2, 256), (1500, 4, 512)])
def test_emulated_ranks_reproduce_the_whole_chunk(T, N, top_k):
    wl, h, new_k, new_kv = _chunk(T)
    be = cp_prefill.CudaBackend(page_size=wl.page_size, top_k=top_k, d_latent=wl.d_latent,
                                softmax_scale=wl.softmax_scale)
    cp = cp_prefill.ZigzagPrefill(be)
    d = workloads.to_device(h, DEV)
    parts = []
    for r in range(N):
        mine = cp_prefill.rank_tokens(T, N, r).long()
        k = torch.zeros_like(d["k_cache"])
        kv = torch.zeros_like(d["kv_cache"])
        out = cp.rank_compute(T, N, r, new_k.to(DEV), new_kv.to(DEV), d["q_idx"][0, mine.to(DEV)],
                              d["w"][0, mine.to(DEV)], d["q_attn"][0, mine.to(DEV)], d["page_table"], k, kv)
        parts.append(out)
    got = cp_prefill.restore_order(parts, T, N).float().cpu().numpy()
    torch.cuda.synchronize()
    ref = _oracle_chunk(wl, h, new_k, new_kv, T, top_k)
    # the first queries of a chunk attend to a handful of rows: their outputs reach magnitudes
    # where the bf16 output's own rounding (up to 2^-9 |ref|) adds to the 1e-2
    assert np.all(np.abs(got - ref) <= 1e-2 + 2.0 ** -9 * np.abs(ref))


def test_world_size_one_nccl_run():
    T, top_k = 700, 128
    wl, h, new_k, new_kv = _chunk(T, seed=43)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device(DEV))
    try:
        be = cp_prefill.CudaBackend(page_size=wl.page_size, top_k=top_k, d_latent=wl.d_latent,
                                    softmax_scale=wl.softmax_scale)
        d = workloads.to_device(h, DEV)
        k = torch.zeros_like(d["k_cache"])
        kv = torch.zeros_like(d["kv_cache"])
        own, full = cp_prefill.ZigzagPrefill(be).run(T, new_k.to(DEV), new_kv.to(DEV), d["q_idx"][0], d["w"][0],
                                                    d["q_attn"][0], d["page_table"], k, kv)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref = _oracle_chunk(wl, h, new_k, new_kv, T, top_k)
    assert np.all(np.abs(full.float().cpu().numpy() - ref) <= 1e-2 + 2.0 ** -9 * np.abs(ref))
    assert torch.equal(own, full)
