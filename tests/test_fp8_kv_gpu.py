"""GPU parity of the sparse attention over an FP8 main cache (e4m3 codes, one fp32 scale per
128-element block of each row) against the oracle's fp64 dequantise-then-attend, and, with
power-of-two scales, bit-for-bit equality with the bf16 path on a bf16 cache holding the decoded
values (the dequantised element is then exact in bf16, so both paths feed identical operands to
the tensor cores).

Tolerance: the kernel rounds each decoded element (code x block scale) once to bf16 before the
products, a relative error of at most 2^-9; the output is a convex combination of the selected
rows, so that rounding moves it by at most 2^-9 max|c| on top of the bf16 path's 1e-2; the
bf16 output's own rounding (2^-9 |ref|) is added as in the other stress cases."""
import numpy as np
import pytest
import torch

import indexed_sparse_attention_paged_b200 as sia
import oracle
from indexed_sparse_attention_paged_b200 import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
ATOL = 1e-2


def fp8_tol(h):
    """1e-2 plus the bf16 rounding of the largest decoded element (see the module docstring)."""
    DC = h["kv_cache"].shape[2]
    dec = h["kv_cache"].float() * h["kv_scale"].repeat_interleave(128, dim=2)[:, :, :DC]
    return ATOL + 2.0 ** -9 * float(dec.abs().max())


def _topk(h, top_k, seed, fill=1.0):
    rng = np.random.default_rng(seed)
    B, J = h["batch"], h["n_q"]
    L = h["seq_lens"].numpy()
    out = np.full((B, J, top_k), -1, dtype=np.int32)
    for b in range(B):
        for j in range(J):
            p = L[b] - J + j
            n = min(top_k, p + 1, max(1, int(fill * top_k)))
            out[b, j, :n] = rng.choice(p + 1, size=n, replace=False)   # unsorted on purpose
    return out


def _run(h, topk_np, kv_scale=True):
    wl = h["workload"]
    d = workloads.to_device(h, DEV)
    topk = torch.from_numpy(topk_np).to(DEV)
    B, J = h["batch"], h["n_q"]
    lse = torch.empty((B, J, wl.attn_heads), device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = sia.sparse_mla_attend(d["q_attn"], d["kv_cache"], d["page_table"], d["seq_lens"], topk,
                                d_latent=wl.d_latent, softmax_scale=wl.softmax_scale, lse=lse,
                                dev_status=status, kv_scale=d.get("kv_scale") if kv_scale else None)
    torch.cuda.synchronize()
    return out, lse, int(status.item())


CASES = {
    "tiny_64_16": (1, dict(), 16, 1.0),
    "mla512_b1_splits": (2, dict(seq_lens=[5000]), 2048, 1.0),
    "mla512_ragged": (2, dict(seq_lens=[3000, 130, 700]), 512, 0.7),
    "mla512_j2": (2, dict(seq_lens=[900, 2500], n_q=2), 256, 1.0),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_fp8_main_cache_attention_matches_the_oracle(name):
    num, kw, top_k, fill = CASES[name]
    h = workloads.fp8_main_cache(workloads.make_inputs(workloads.WORKLOADS[num], **kw))
    tk = _topk(h, top_k, seed=11, fill=fill)
    out, lse, st = _run(h, tk)
    assert st == 0
    wl = h["workload"]
    ref, ref_lse, ost = oracle.sparse_attend(h["q_attn"], h["kv_cache"], h["page_table"].numpy(),
                                             h["seq_lens"].numpy(), tk, page_size=wl.page_size,
                                             d_latent=wl.d_latent, scale=wl.softmax_scale,
                                             kv_scale=h["kv_scale"].numpy())
    assert ost == 0
    err = np.abs(out.float().cpu().numpy() - ref)
    assert np.all(err <= fp8_tol(h) + 2.0 ** -9 * np.abs(ref)), err.max()
    g = lse.cpu().numpy()
    fin = np.isfinite(ref_lse)
    assert np.all(np.isfinite(g) == fin)
    assert np.all(np.abs(g[fin] - ref_lse[fin]) <= 1e-3 * np.maximum(1.0, np.abs(ref_lse[fin])))


@pytest.mark.parametrize("num,kw,top_k", [(2, dict(seq_lens=[4000, 2100]), 2048), (1, dict(), 16)])
def test_fp8_cache_with_power_of_two_scales_equals_the_bf16_path_bit_for_bit(num, kw, top_k):
    h8 = workloads.fp8_main_cache(workloads.make_inputs(workloads.WORKLOADS[num], **kw), pow2_scales=True)
    nblk = h8["kv_scale"].shape[2]
    DC = h8["kv_cache"].shape[2]
    per_elem = h8["kv_scale"].repeat_interleave(128, dim=2)[:, :, :DC]
    hb = dict(h8, kv_cache=(h8["kv_cache"].float() * per_elem).to(torch.bfloat16), kv_scale=None)
    assert torch.equal(hb["kv_cache"].float(), h8["kv_cache"].float() * per_elem)   # exact in bf16
    tk = _topk(h8, top_k, seed=12)
    o8, l8, s8 = _run(h8, tk)
    ob, lb, sb = _run(hb, tk, kv_scale=False)
    assert s8 == 0 and sb == 0
    assert torch.equal(o8, ob) and torch.equal(l8, lb)
    assert nblk == (DC + 127) // 128


def test_fused_decode_over_an_fp8_main_cache():
    wl = workloads.WORKLOADS[3]
    h = workloads.fp8_main_cache(workloads.make_inputs(wl, seq_lens=[1500, 3000, 2049]))
    d = workloads.to_device(h, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out, topk = sia.fused_decode(d["q_idx"], d["w"], d["k_cache"], d["q_attn"], d["kv_cache"],
                                 d["page_table"], d["seq_lens"], top_k=wl.top_k, d_latent=wl.d_latent,
                                 softmax_scale=wl.softmax_scale, k_scale=d["k_scale"],
                                 kv_scale=d["kv_scale"], dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_topk, _, _ = oracle.index_topk(h["q_idx"], h["w"].numpy(), h["k_cache"], h["page_table"].numpy(),
                                       h["seq_lens"].numpy(), page_size=wl.page_size, top_k=wl.top_k,
                                       fp8=True, k_scale=h["k_scale"].numpy())
    assert np.array_equal(topk.cpu().numpy(), ref_topk)
    ref, _, _ = oracle.sparse_attend(h["q_attn"], h["kv_cache"], h["page_table"].numpy(), h["seq_lens"].numpy(),
                                     ref_topk, page_size=wl.page_size, d_latent=wl.d_latent,
                                     scale=wl.softmax_scale, kv_scale=h["kv_scale"].numpy())
    assert np.all(np.abs(out.float().cpu().numpy() - ref) <= fp8_tol(h) + 2.0 ** -9 * np.abs(ref))
