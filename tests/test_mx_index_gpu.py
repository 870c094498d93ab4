"""GPU parity of the MXFP8 index path (E4M3 codes, one E8M0 scale per 32 elements of q and of
each key) against the oracle: scores bit for bit and Top-K lists exact, for integer-valued codes
whose scale exponents keep every partial sum exact in fp32; and the Top-K agreement of the MXFP8
path with the bf16 path on real-valued queries and keys quantised by the pages' rule."""
import numpy as np
import pytest
import torch

import indexed_sparse_attention_paged_b200 as sia
import oracle
from indexed_sparse_attention_paged_b200 import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _mx_inputs(seed, seq_lens, n_q=1, D=128, H=64, exp_lo=-1, exp_hi=1):
    """Workload-3 shapes with MX scales: codes are integers in [-3, 3], scale codes 127 + e with
    e uniform in [exp_lo, exp_hi]."""
    h = workloads.make_inputs(workloads.WORKLOADS[3], seed=seed, seq_lens=seq_lens, n_q=n_q)
    g = torch.Generator().manual_seed(seed + 1)
    B, J = h["batch"], h["n_q"]
    pages, P = h["k_cache"].shape[:2]
    q_mx = (127 + torch.randint(exp_lo, exp_hi + 1, (B, J, H, D // 32), generator=g, dtype=torch.int32)).to(torch.uint8)
    k_mx = (127 + torch.randint(exp_lo, exp_hi + 1, (pages, P, D // 32), generator=g, dtype=torch.int32)).to(torch.uint8)
    h["q_mx"], h["k_mx"], h["k_scale"] = q_mx, k_mx, None
    return h


def _run(h, top_k):
    d = workloads.to_device(h, DEV)
    B, J = h["batch"], h["n_q"]
    Lpad = h["max_pages"] * h["workload"].page_size
    scores = torch.full((B, J, Lpad), float("nan"), device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    topk = sia.sparse_index_topk(d["q_idx"], d["w"], d["k_cache"], d["page_table"], d["seq_lens"],
                                 top_k=top_k, q_mx=d["q_mx"], k_mx=d["k_mx"], scores_out=scores,
                                 dev_status=status)
    torch.cuda.synchronize()
    return topk.cpu().numpy(), scores.cpu().numpy(), int(status.item())


@pytest.mark.parametrize("seq_lens,n_q,top_k", [([513, 2000, 64], 1, 256), ([1500, 777], 2, 300),
                                                ([9000, 4100], 1, 2048)])
def test_mx_index_scores_and_topk_match_the_oracle_exactly(seq_lens, n_q, top_k):
    h = _mx_inputs(900 + len(seq_lens), seq_lens, n_q)
    got_topk, got, st = _run(h, top_k)
    assert st == 0
    ref, nvis, ost = oracle.index_scores_mx(h["q_idx"], h["q_mx"], h["w"].numpy(), h["k_cache"], h["k_mx"],
                                            h["page_table"].numpy(), h["seq_lens"].numpy(),
                                            page_size=h["workload"].page_size)
    assert ost == 0
    ref_topk = oracle.topk(ref, nvis, top_k)
    B, J = h["batch"], h["n_q"]
    for b in range(B):
        for j in range(J):
            n = int(nvis[b, j])
            bad = np.flatnonzero(got[b, j, :n] != ref[b, j, :n].astype(np.float32))
            assert bad.size == 0, "row (%d,%d): %d scores differ" % (b, j, bad.size)
            assert np.array_equal(got_topk[b, j], ref_topk[b, j])


def test_mx_wide_scale_exponents_stay_close_to_the_oracle():
    """Exponents over [-6, 6] on both sides: sums are no longer exact in fp32, so the scores are
    compared to within fp32 rounding and the list is checked to be a valid Top-K."""
    h = _mx_inputs(950, [3000, 1700], exp_lo=-6, exp_hi=6)
    got_topk, got, st = _run(h, 512)
    assert st == 0
    ref, nvis, _ = oracle.index_scores_mx(h["q_idx"], h["q_mx"], h["w"].numpy(), h["k_cache"], h["k_mx"],
                                          h["page_table"].numpy(), h["seq_lens"].numpy(),
                                          page_size=h["workload"].page_size)
    for b in range(h["batch"]):
        n = int(nvis[b, 0])
        r = ref[b, 0, :n]
        scale = np.max(np.abs(r)) + 1e-30
        assert np.max(np.abs(got[b, 0, :n] - r)) <= 1e-5 * scale
        sel = got_topk[b, 0][got_topk[b, 0] >= 0]
        mask = np.zeros(n, bool)
        mask[sel] = True
        assert sel.size == min(512, n)
        assert r[mask].min() >= r[~mask].max() - 2e-5 * scale


def _mx_quantise(x):
    """Real values [..., D] -> (e4m3 codes, E8M0 codes [..., D/32]) by the pages' MX rule, through
    the oracle's cache append (each vector written as the new key of a one-token sequence)."""
    flat = x.reshape(-1, x.shape[-1]).float()
    n, D = flat.shape
    pt = np.arange(n, dtype=np.int32).reshape(n, 1)
    sl = np.ones(n, dtype=np.int32)
    codes = np.zeros((n, 1, D), np.uint8)
    scales = np.zeros((n, 1, D // 32), np.uint8)
    kv = np.zeros((n, 1, 16), np.uint16)
    assert oracle.cache_append(flat.view(n, 1, D), torch.zeros(n, 1, 16), pt, sl, codes, kv, page_size=1,
                               k_mode="mx", k_scale=scales) == 0
    return (torch.from_numpy(codes.reshape(*x.shape)).view(torch.float8_e4m3fn),
            torch.from_numpy(scales.reshape(*x.shape[:-1], D // 32)))


def test_mx_topk_agrees_with_the_bf16_path_on_real_valued_inputs():
    h = workloads.make_inputs(workloads.WORKLOADS[2], seq_lens=[8192, 6000, 4096])
    g = torch.Generator().manual_seed(77)
    q = torch.randn(h["q_idx"].shape, generator=g).to(torch.bfloat16)
    k = torch.randn(h["k_cache"].shape, generator=g).to(torch.bfloat16)
    hb = dict(h, q_idx=q, k_cache=k)
    db = workloads.to_device(hb, DEV)
    tb = sia.sparse_index_topk(db["q_idx"], db["w"], db["k_cache"], db["page_table"], db["seq_lens"], top_k=2048)
    qc, qm = _mx_quantise(q)
    kc, km = _mx_quantise(k)
    tm = sia.sparse_index_topk(qc.to(DEV), db["w"], kc.to(DEV), db["page_table"], db["seq_lens"], top_k=2048,
                               q_mx=qm.to(DEV), k_mx=km.to(DEV))
    torch.cuda.synchronize()
    tb, tm = tb.cpu().numpy(), tm.cpu().numpy()
    recall = [len(np.intersect1d(tb[b, 0], tm[b, 0])) / 2048.0 for b in range(3)]
    print("MXFP8 vs bf16 Top-K recall per sequence:", recall)
    assert min(recall) >= 0.8
