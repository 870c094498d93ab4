"""The timeout path of the bounded in-kernel waits, made to run out on purpose with a tiny
bound (no GPU fault, no hang): every kernel of the call gives up at its first wait that does not
succeed at once, drains the copies and tensor-core operations it already issued, reports
SIA_DEV_TIMEOUT in the status word and returns; the context stays usable and the next call,
with the default bound, is exact again."""
import numpy as np
import pytest
import torch

import indexed_sparse_attention_paged_b200 as sia
import oracle
from indexed_sparse_attention_paged_b200 import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _fused(h, d, status):
    wl = h["workload"]
    return sia.fused_decode(d["q_idx"], d["w"], d["k_cache"], d["q_attn"], d["kv_cache"],
                            d["page_table"], d["seq_lens"], top_k=wl.top_k, d_latent=wl.d_latent,
                            softmax_scale=wl.softmax_scale, k_scale=d["k_scale"], dev_status=status)


def test_a_wait_that_runs_out_reports_timeout_and_the_next_call_is_exact():
    h = workloads.make_inputs(workloads.WORKLOADS[2], seq_lens=[3000, 5000, 2100])
    d = workloads.to_device(h, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    prev = sia.set_wait_limit_ns(1)
    try:
        _fused(h, d, status)
        torch.cuda.synchronize()
    finally:
        sia.set_wait_limit_ns(prev)
    assert int(status.item()) & sia.SIA_DEV_TIMEOUT
    assert not int(status.item()) & (sia.SIA_DEV_BAD_PAGE | sia.SIA_DEV_BAD_POSITION)

    status.zero_()
    out, topk = _fused(h, d, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    wl = h["workload"]
    ref_topk, _, _ = oracle.index_topk(h["q_idx"], h["w"].numpy(), h["k_cache"], h["page_table"].numpy(),
                                       h["seq_lens"].numpy(), page_size=wl.page_size, top_k=wl.top_k)
    assert np.array_equal(topk.cpu().numpy(), ref_topk)
    ref, _, _ = oracle.sparse_attend(h["q_attn"], h["kv_cache"], h["page_table"].numpy(),
                                     h["seq_lens"].numpy(), ref_topk, page_size=wl.page_size,
                                     d_latent=wl.d_latent, scale=wl.softmax_scale)
    assert np.abs(out.float().cpu().numpy() - ref).max() <= 1e-2

