"""The index + Top-K entry point that allocates nothing (sia_sparse_index_topk_noalloc), for
callers that cannot allocate device memory while they run: its score scratch is a fixed array
inside the library instead of a caller-provided workspace.  Its Top-K lists must equal those of
the regular entry point exactly, on consecutive calls with different inputs (the shared scratch
keeps the previous call's scores, which must not leak into the next result)."""
import ctypes

import pytest
import torch

import indexed_sparse_attention_paged_b200 as sia
from indexed_sparse_attention_paged_b200 import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _regular_and_noalloc(h):
    wl = h["workload"]
    d = workloads.to_device(h, DEV)
    ref = sia.sparse_index_topk(d["q_idx"], d["w"], d["k_cache"], d["page_table"], d["seq_lens"],
                                top_k=wl.top_k, k_scale=d["k_scale"])
    out = torch.full_like(ref, -7)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    sia.sparse_index_topk_noalloc(d["q_idx"], d["w"], d["k_cache"], d["page_table"], d["seq_lens"],
                                  top_k=wl.top_k, k_scale=d["k_scale"], topk_out=out, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return ref, out


def test_noalloc_entry_point_matches_the_regular_one_on_two_calls_in_a_row():
    first = workloads.make_inputs(workloads.WORKLOADS[2], seq_lens=[3000, 8192, 1500])
    second = workloads.make_inputs(workloads.WORKLOADS[3], seq_lens=[2000, 700, 5000, 4096])
    for h in (first, second):
        ref, out = _regular_and_noalloc(h)
        assert torch.equal(out, ref)


def test_noalloc_entry_point_refuses_more_than_its_scratch():
    lib = sia.load_library()
    # 64 x 1 x 128 pages x 1024 positions x 4 bytes = 32 MiB of scores > 16 MiB
    q = torch.zeros(64, 1, 64, 128, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(64, 1, 64, dtype=torch.float32, device=DEV)
    k = torch.zeros(8, 1024, 128, dtype=torch.bfloat16, device=DEV)
    pt = torch.zeros(64, 128, dtype=torch.int32, device=DEV)
    sl = torch.full((64,), 100, dtype=torch.int32, device=DEV)
    out = torch.empty(64, 1, 16, dtype=torch.int32, device=DEV)
    a = sia.index_args(q, w, k, pt, sl, top_k=16, topk_out=out)
    st = lib.sia_sparse_index_topk_noalloc(ctypes.byref(a), None,
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == sia.SIA_ERR_WORKSPACE
    assert b"workspace" in lib.sia_last_error()
