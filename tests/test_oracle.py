"""Pins for the CPU oracle: each check is fixed by something other than the oracle itself
(hand-worked examples, closed forms, invariants, brute force, library routines)."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp, softmax

import oracle
from indexed_sparse_attention_paged_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- element decoding

def test_bf16_decode_matches_torch_for_every_pattern():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_value(int(b)) for b in bits[::7]])
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref[::7]))
    ok = ~np.isnan(ref[::7])
    np.testing.assert_array_equal(got[ok], ref[::7][ok])


def test_e4m3_decode_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_value(int(c)) for c in codes])
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    assert oracle.e4m3_value(0x7E) == 448.0          # largest finite value of the format
    assert oracle.e4m3_value(0x01) == 2.0 ** -9      # smallest subnormal


# ---------------------------------------------------------------- scores (steps 1-2)

def _golden_index():
    with open(os.path.join(GOLDEN, "worked_index_example.json")) as f:
        return json.load(f)


def test_scores_hand_worked_example():
    g = _golden_index()
    q = bf16(g["q"])
    k = bf16(g["k_cache"])
    w = np.array(g["w"], dtype=np.float32)
    pt = np.array(g["page_table"], dtype=np.int32)
    sl = np.array([g["seq_len"]], dtype=np.int32)
    scores, nvis, st = oracle.index_scores(q, w, k, pt, sl, page_size=g["page_size"])
    assert st == 0 and nvis[0, 0] == 3
    np.testing.assert_array_equal(scores[0, 0, :3], g["scores"])
    assert np.isnan(scores[0, 0, 3])          # past the query: not scored
    tk, _, _ = oracle.index_topk(q, w, k, pt, sl, page_size=g["page_size"], top_k=2)
    assert tk[0, 0].tolist() == g["top2"]
    tk, _, _ = oracle.index_topk(q, w, k, pt, sl, page_size=g["page_size"], top_k=4)
    assert tk[0, 0].tolist() == g["top4"]


def _small_index_case(seed, B=2, J=1, H=3, D=8, P=4, L=11, fp8=False):
    r = rng(seed)
    pages = (L + P - 1) // P
    num_pages = B * pages
    perm = r.permutation(num_pages).astype(np.int32)
    pt = perm.reshape(B, pages)
    q = r.integers(-3, 4, (B, J, H, D)).astype(np.float32)
    k = r.integers(-3, 4, (num_pages, P, D)).astype(np.float32)
    w = r.integers(-2, 3, (B, J, H)).astype(np.float32)
    sl = np.full(B, L, dtype=np.int32)
    return q, k, w, pt, sl


def _logical_k(k, pt, P, b, L):
    """Logical-order key rows of sequence b, read through the page table by hand."""
    return np.stack([k[pt[b, s // P], s % P] for s in range(L)])


def test_scores_closed_form_without_relu():
    # with w = 1 and non-negative q, k every dot is >= 0, ReLU is the identity and the head
    # sum factors: I[s] = (sum_h q_h) . k[s]
    q, k, w, pt, sl = _small_index_case(1)
    q, k, w = np.abs(q), np.abs(k), np.ones_like(w)
    scores, _, st = oracle.index_scores(bf16(q), w, bf16(k), pt, sl, page_size=4)
    assert st == 0
    for b in range(2):
        expect = _logical_k(k, pt, 4, b, 11) @ q[b, 0].sum(axis=0)
        np.testing.assert_array_equal(scores[b, 0, :11], expect)


def test_scores_single_head_weight_selects_relu_of_that_head():
    q, k, w, pt, sl = _small_index_case(2)
    for h in range(3):
        wh = np.zeros_like(w)
        wh[..., h] = 1.0
        scores, _, _ = oracle.index_scores(bf16(q), wh, bf16(k), pt, sl, page_size=4)
        for b in range(2):
            dots = _logical_k(k, pt, 4, b, 11) @ q[b, 0, h]
            np.testing.assert_array_equal(scores[b, 0, :11], np.maximum(dots, 0.0))


def test_scores_linear_in_head_weights_and_scales():
    q, k, w, pt, sl = _small_index_case(3)
    w2 = rng(33).integers(-2, 3, w.shape).astype(np.float32)
    s1, _, _ = oracle.index_scores(bf16(q), w, bf16(k), pt, sl, page_size=4)
    s2, _, _ = oracle.index_scores(bf16(q), w2, bf16(k), pt, sl, page_size=4)
    s12, _, _ = oracle.index_scores(bf16(q), w + w2, bf16(k), pt, sl, page_size=4)
    np.testing.assert_array_equal(s12[..., :11], s1[..., :11] + s2[..., :11])
    # per-token power-of-two key scales and a per-query scale multiply the score exactly
    ks = np.power(2.0, rng(34).integers(-4, 5, k.shape[:2])).astype(np.float32)
    qs = np.array([[0.5], [4.0]], dtype=np.float32)
    k8 = torch.tensor(k).to(torch.float8_e4m3fn)
    q8 = torch.tensor(q).to(torch.float8_e4m3fn)
    sc, _, _ = oracle.index_scores(q8, w, k8, pt, sl, page_size=4, fp8=True, k_scale=ks, q_scale=qs)
    for b in range(2):
        for s in range(11):
            row = pt[b, s // 4] * 4 + s % 4
            assert sc[b, 0, s] == s1[b, 0, s] * ks.reshape(-1)[row] * qs[b, 0]


def test_scores_independent_of_physical_page_placement():
    q, k, w, pt, sl = _small_index_case(4)
    base, _, _ = oracle.index_scores(bf16(q), w, bf16(k), pt, sl, page_size=4)
    # move every page to a new physical slot and rewrite the table to match
    perm = rng(44).permutation(k.shape[0])
    k_moved = np.empty_like(k)
    k_moved[perm] = k
    moved, _, _ = oracle.index_scores(bf16(q), w, bf16(k_moved), perm[pt].astype(np.int32), sl,
                                      page_size=4)
    np.testing.assert_array_equal(base, moved)


def test_fp8_and_bf16_storage_give_identical_scores():
    # integers in [-3,3] are exact in both formats, so the quantised index path must agree
    # with the bf16 baseline exactly (Top-K hit rate 100%)
    q, k, w, pt, sl = _small_index_case(5)
    sb, _, _ = oracle.index_scores(bf16(q), w, bf16(k), pt, sl, page_size=4)
    s8, _, _ = oracle.index_scores(torch.tensor(q).to(torch.float8_e4m3fn), w,
                                   torch.tensor(k).to(torch.float8_e4m3fn), pt, sl, page_size=4,
                                   fp8=True)
    np.testing.assert_array_equal(sb, s8)


def test_causal_visibility_and_query_positions():
    q, k, w, pt, sl = _small_index_case(6, J=2)
    scores, nvis, st = oracle.index_scores(bf16(q), w, bf16(k), pt, sl, page_size=4)
    assert st == 0
    # default positions: seq_len - J + j -> draft at L-2 sees L-1 positions, verify sees L
    assert nvis.tolist() == [[10, 11], [10, 11]]
    assert np.isnan(scores[0, 0, 10]) and not np.isnan(scores[0, 1, 10])
    qp = np.array([[0, 5], [3, 3]], dtype=np.int32)
    scores, nvis, _ = oracle.index_scores(bf16(q), w, bf16(k), pt, sl, page_size=4, q_pos=qp)
    assert nvis.tolist() == [[1, 6], [4, 4]]
    assert np.isnan(scores[0, 0, 1]) and not np.isnan(scores[0, 0, 0])


def test_bad_page_id_is_reported_not_read():
    q, k, w, pt, sl = _small_index_case(7)
    pt = pt.copy()
    pt[1, 1] = k.shape[0] + 5
    _, _, st = oracle.index_scores(bf16(q), w, bf16(k), pt, sl, page_size=4)
    assert st != 0


# ---------------------------------------------------------------- Top-K (step 3)

def _brute_force_topk(scores, k):
    """The unique K-subset that beats every outsider under (score desc, position asc),
    found by enumerating every subset."""
    n = len(scores)
    if n <= k:
        return list(range(n)) + [-1] * (k - n)
    found = []
    for sub in itertools.combinations(range(n), k):
        inside = set(sub)
        if all((scores[i] > scores[j]) or (scores[i] == scores[j] and i < j)
               for i in inside for j in range(n) if j not in inside):
            found.append(list(sub))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("seed", range(12))
def test_topk_matches_brute_force_with_heavy_ties(seed):
    r = rng(100 + seed)
    n = int(r.integers(1, 11))
    k = int(r.integers(1, 6))
    scores = r.integers(-2, 3, n).astype(np.float64)     # few distinct values -> many ties
    got = oracle.topk_row(scores, n, k).tolist()
    assert got == _brute_force_topk(list(scores), k)


def test_topk_invariants_on_large_rows():
    r = rng(200)
    for n, k in [(5000, 2048), (3000, 64), (2048, 2048), (100, 2048)]:
        scores = r.integers(-50, 50, n).astype(np.float64)
        got = oracle.topk_row(scores, n, k)
        sel = got[got >= 0]
        assert len(sel) == min(n, k)
        assert np.all(np.diff(sel) > 0)                    # ascending, no repeats
        if n > k:
            mask = np.zeros(n, bool)
            mask[sel] = True
            thr = scores[mask].min()
            assert scores[~mask].max() <= thr
            # among positions scoring exactly the threshold, the lowest ones are taken
            eq = np.flatnonzero(scores == thr)
            taken = np.flatnonzero(mask & (scores == thr))
            assert taken.tolist() == eq[:len(taken)].tolist()


def test_topk_special_cases():
    assert oracle.topk_row(np.zeros(10), 10, 4).tolist() == [0, 1, 2, 3]
    assert oracle.topk_row(np.array([-0.0, 0.0, -0.0]), 3, 1).tolist() == [0]
    assert oracle.topk_row(np.array([0.0, -0.0, 1.0]), 3, 2).tolist() == [0, 2]
    assert oracle.topk_row(np.array([3.0, 1.0]), 2, 4).tolist() == [0, 1, -1, -1]
    assert oracle.topk_row(np.array([]), 0, 3).tolist() == [-1, -1, -1]


# ---------------------------------------------------------------- attention (steps 4-5)

def _attn_case(seed, B=2, J=2, H=3, DL=8, DR=4, P=4, L=13, K=5):
    r = rng(seed)
    pages = (L + P - 1) // P
    num_pages = B * pages
    pt = r.permutation(num_pages).astype(np.int32).reshape(B, pages)
    q = r.standard_normal((B, J, H, DL + DR)).astype(np.float32)
    kv = r.standard_normal((num_pages, P, DL + DR)).astype(np.float32)
    sl = np.full(B, L, dtype=np.int32)
    topk = np.full((B, J, K), -1, dtype=np.int32)
    for b in range(B):
        for j in range(J):
            p = L - J + j
            sel = np.sort(r.choice(p + 1, size=min(K, p + 1), replace=False))
            topk[b, j, :len(sel)] = sel
    return bf16(q), bf16(kv), pt, sl, topk


def test_attention_hand_worked_example():
    with open(os.path.join(GOLDEN, "worked_attention_example.json")) as f:
        g = json.load(f)
    q = bf16(np.array(g["q"]).reshape(1, 1, 1, 3))
    kv = bf16(np.array(g["rows"] + [[0, 0, 0]]).reshape(1, 4, 3))
    pt = np.array([[0]], dtype=np.int32)
    sl = np.array([3], dtype=np.int32)
    out, lse, st = oracle.sparse_attend(q, kv, pt, sl, np.array([[[0, 2]]], dtype=np.int32),
                                        page_size=4, d_latent=2, scale=1.0)
    assert st == 0
    np.testing.assert_allclose(out[0, 0, 0], [3.0, 2.0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[0, 0, 0], 2.0 + math.log(2.0), rtol=0, atol=1e-15)
    out, lse, _ = oracle.sparse_attend(q, kv, pt, sl, np.array([[[0, 1]]], dtype=np.int32),
                                       page_size=4, d_latent=2, scale=1.0)
    e = math.e
    np.testing.assert_allclose(out[0, 0, 0], [2 * e / (e + 1), (4 * e + 2) / (e + 1)], atol=1e-15)
    np.testing.assert_allclose(lse[0, 0, 0], 2.0 + math.log(1 + 1 / e), atol=1e-15)


def test_sparse_gather_equals_dense_masked_attention():
    q, kv, pt, sl, topk = _attn_case(300)
    Lpad = pt.shape[1] * 4
    allowed = np.zeros((2, 2, Lpad), np.uint8)
    for b in range(2):
        for j in range(2):
            allowed[b, j, topk[b, j][topk[b, j] >= 0]] = 1
    o1, l1, s1 = oracle.sparse_attend(q, kv, pt, sl, topk, page_size=4, d_latent=8, scale=0.3)
    o2, l2, s2 = oracle.dense_masked_attend(q, kv, pt, sl, allowed, page_size=4, d_latent=8,
                                            scale=0.3)
    assert s1 == 0 and s2 == 0
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_topk_covering_the_history_reduces_to_dense_causal_attention():
    q, kv, pt, sl, _ = _attn_case(301, K=16)
    L = 13
    topk = np.full((2, 2, 16), -1, dtype=np.int32)
    for j in range(2):
        n = L - 2 + j + 1
        topk[:, j, :n] = np.arange(n)
    o1, l1, _ = oracle.sparse_attend(q, kv, pt, sl, topk, page_size=4, d_latent=8, scale=0.3)
    # library softmax over the full causal history, rows read through the page table by hand
    qn = q.to(torch.float64).numpy()
    kvn = kv.to(torch.float64).numpy()
    for b in range(2):
        for j in range(2):
            n = L - 2 + j + 1
            rows = np.stack([kvn[pt[b, s // 4], s % 4] for s in range(n)])
            z = 0.3 * rows @ qn[b, j].T                      # [n, H]
            np.testing.assert_allclose(o1[b, j], (softmax(z, axis=0).T @ rows[:, :8]), atol=1e-12)
            np.testing.assert_allclose(l1[b, j], logsumexp(z, axis=0), atol=1e-12)


def test_attention_special_cases():
    q, kv, pt, sl, _ = _attn_case(302, K=4)
    kvn = kv.to(torch.float64).numpy()
    # one selected row: the output is that row's latent part and lse is its logit
    topk = np.full((2, 2, 4), -1, dtype=np.int32)
    topk[:, :, 0] = 7
    o, l, _ = oracle.sparse_attend(q, kv, pt, sl, topk, page_size=4, d_latent=8, scale=0.3)
    for b in range(2):
        row = kvn[pt[b, 1], 3]
        for j in range(2):
            np.testing.assert_array_equal(o[b, j], np.broadcast_to(row[:8], (3, 8)))
            zq = 0.3 * q[b, j].to(torch.float64).numpy() @ row
            np.testing.assert_allclose(l[b, j], zq, atol=1e-12)
    # zero query: uniform weights -> mean of the selected rows, lse = log(count)
    qz = torch.zeros_like(q)
    topk[:, :, :3] = [2, 5, 9]
    o, l, _ = oracle.sparse_attend(qz, kv, pt, sl, topk, page_size=4, d_latent=8, scale=0.3)
    for b in range(2):
        rows = np.stack([kvn[pt[b, s // 4], s % 4] for s in (2, 5, 9)])
        np.testing.assert_allclose(o[b, 0, 0], rows[:, :8].mean(axis=0), atol=1e-12)
    np.testing.assert_allclose(l, math.log(3.0), atol=1e-12)
    # an empty list gives zeros and lse = -inf
    topk[:] = -1
    o, l, _ = oracle.sparse_attend(q, kv, pt, sl, topk, page_size=4, d_latent=8, scale=0.3)
    assert np.all(o == 0) and np.all(np.isneginf(l))


def test_attention_identical_rows_shift_and_list_order():
    q, kv, pt, sl, topk = _attn_case(303)
    DL = 8
    kvn = kv.to(torch.float64).numpy()
    ref_o, ref_l, st = oracle.sparse_attend(q, kv, pt, sl, topk, page_size=4, d_latent=DL, scale=0.3)
    assert st == 0
    # the list is a set: its order does not matter
    perm = topk.copy()
    for b in range(2):
        for j in range(2):
            n = int(np.sum(topk[b, j] >= 0))
            perm[b, j, :n] = topk[b, j, :n][::-1]
    o, l, _ = oracle.sparse_attend(q, kv, pt, sl, perm, page_size=4, d_latent=DL, scale=0.3)
    np.testing.assert_allclose(o, ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, ref_l, rtol=0, atol=1e-12)
    # a constant added to every logit: give every cache row the same first rope value 1 and
    # raise that query component by 1, so each logit grows by exactly the scale; the output
    # (latent part only) is unchanged and the log-sum-exp moves by the scale
    kv1 = kv.clone()
    kv1[:, :, DL] = 1.0
    o0, l0, _ = oracle.sparse_attend(q, kv1, pt, sl, topk, page_size=4, d_latent=DL, scale=0.3)
    q1 = q.clone()
    q1[..., DL] = (q1[..., DL].float() + 1.0).to(torch.bfloat16)
    shifted = (q1[..., DL].double() - q[..., DL].double()).numpy()     # 1, up to bf16 rounding
    o1, l1, _ = oracle.sparse_attend(q1, kv1, pt, sl, topk, page_size=4, d_latent=DL, scale=0.3)
    np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l0 + 0.3 * shifted, rtol=0, atol=1e-12)
    # every selected position holds the same row: the output is that row, lse = z + log(n)
    kv2 = kv.clone()
    kv2[:, :, :] = kv[pt[0, 0], 0]
    o2, l2, _ = oracle.sparse_attend(q, kv2, pt, sl, topk, page_size=4, d_latent=DL, scale=0.3)
    row = kvn[pt[0, 0], 0]
    for b in range(2):
        for j in range(2):
            n = int(np.sum(topk[b, j] >= 0))
            np.testing.assert_allclose(o2[b, j], np.broadcast_to(row[:DL], o2[b, j].shape), rtol=0, atol=1e-12)
            z = 0.3 * q[b, j].to(torch.float64).numpy() @ row
            np.testing.assert_allclose(l2[b, j], z + math.log(n), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- FP8 main cache (NEXT row)

def _fp8_case(seed, B=2, J=1, H=3, DL=512, DR=64, P=4, L=11):
    """e4m3 codes of a random cache, torch's decode of them (float64), the page table."""
    r = rng(seed)
    pages = (L + P - 1) // P
    num_pages = B * pages
    pt = r.permutation(num_pages).astype(np.int32).reshape(B, pages)
    codes = torch.tensor(r.uniform(-3, 3, (num_pages, P, DL + DR)).astype(np.float32)).to(torch.float8_e4m3fn)
    decoded = codes.to(torch.float32).double().numpy()
    q = bf16(r.standard_normal((B, J, H, DL + DR)))
    sl = np.full(B, L, dtype=np.int32)
    return q, codes, decoded, pt, sl


def test_fp8_main_cache_single_row_gives_the_dequantised_row():
    """One selected row: out is that row's latent part, dequantised block by block (scales that
    differ per token and per 128-element block, not powers of two), and lse its logit, whose
    last block is the 64 rope elements."""
    q, codes, decoded, pt, sl = _fp8_case(401)
    DC, DL, P = 576, 512, 4
    nblk = 5
    r = rng(402)
    kv_scale = r.uniform(0.01, 2.0, (codes.shape[0], P, nblk)).astype(np.float32)
    topk = np.full((2, 1, 4), -1, dtype=np.int32)
    topk[:, 0, 0] = [6, 9]
    out, lse, st = oracle.sparse_attend(q, codes, pt, sl, topk, page_size=P, d_latent=DL,
                                        scale=0.05, kv_scale=kv_scale)
    assert st == 0
    blk = np.arange(DC) // 128
    for b, s in enumerate((6, 9)):
        page, off = pt[b, s // P], s % P
        deq = decoded[page, off] * kv_scale[page, off][blk].astype(np.float64)
        for h in range(3):
            np.testing.assert_array_equal(out[b, 0, h], deq[:DL])
            z = 0.05 * float(np.dot(q[b, 0, h].to(torch.float64).numpy(), deq))
            np.testing.assert_allclose(lse[b, 0, h], z, rtol=0, atol=1e-12)


def test_fp8_main_cache_with_power_of_two_scales_equals_the_bf16_cache_of_its_values():
    """Power-of-two block scales keep every dequantised element exact in bf16, so the FP8 path
    must give exactly what the bf16 path gives on a bf16 cache holding those values."""
    q, codes, decoded, pt, sl = _fp8_case(403, J=2, L=13)
    P, DL = 4, 512
    r = rng(404)
    kv_scale = np.power(2.0, r.integers(-3, 4, (codes.shape[0], P, 5))).astype(np.float32)
    deq = decoded * np.repeat(kv_scale.astype(np.float64), 128, axis=2)[:, :, :576]
    kv_bf16 = torch.tensor(deq.astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(kv_bf16.double().numpy(), deq)          # exact in bf16
    topk = np.full((2, 2, 6), -1, dtype=np.int32)
    for b in range(2):
        for j in range(2):
            topk[b, j, :5] = np.sort(r.choice(13 - 2 + j + 1, 5, replace=False))
    o8, l8, s8 = oracle.sparse_attend(q, codes, pt, sl, topk, page_size=P, d_latent=DL,
                                      scale=0.05, kv_scale=kv_scale)
    ob, lb, sb = oracle.sparse_attend(q, kv_bf16, pt, sl, topk, page_size=P, d_latent=DL, scale=0.05)
    assert s8 == 0 and sb == 0
    np.testing.assert_array_equal(o8, ob)
    np.testing.assert_array_equal(l8, lb)


def test_fp8_main_cache_refuses_a_scale_array_of_the_wrong_shape():
    q, codes, _, pt, sl = _fp8_case(405)
    topk = np.zeros((2, 1, 1), dtype=np.int32)
    with pytest.raises(ValueError):
        oracle.sparse_attend(q, codes, pt, sl, topk, page_size=4, d_latent=512, scale=0.05,
                             kv_scale=np.ones((codes.shape[0], 4, 4), np.float32))


# ---------------------------------------------------------------- MXFP8 index path (NEXT row)

def test_e8m0_decode_matches_torch_for_every_code():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).to(torch.float32).double().numpy()
    got = np.array([oracle.e8m0_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert nan.sum() == 1 and np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def _mx_case(seed, B=2, J=2, H=4, D=128, P=4, L=11):
    """Integer-valued e4m3 codes in [-8, 8] and E8M0 scales 2^-4..2^4: every product and sum
    of the score is exact in fp64, so any summation order gives the same value."""
    r = rng(seed)
    pages = (L + P - 1) // P
    num_pages = B * pages
    pt = r.permutation(num_pages).astype(np.int32).reshape(B, pages)
    q = torch.tensor(r.integers(-8, 9, (B, J, H, D)).astype(np.float32)).to(torch.float8_e4m3fn)
    k = torch.tensor(r.integers(-8, 9, (num_pages, P, D)).astype(np.float32)).to(torch.float8_e4m3fn)
    q_mx = r.integers(123, 132, (B, J, H, D // 32)).astype(np.uint8)
    k_mx = r.integers(123, 132, (num_pages, P, D // 32)).astype(np.uint8)
    w = r.integers(-2, 3, (B, J, H)).astype(np.float32)
    sl = np.full(B, L, dtype=np.int32)
    return q, q_mx, w, k, k_mx, pt, sl


def test_mx_scores_with_unit_scales_equal_the_fp8_path():
    q, q_mx, w, k, k_mx, pt, sl = _mx_case(501)
    ones_q, ones_k = np.full_like(q_mx, 127), np.full_like(k_mx, 127)
    mx, nv1, s1 = oracle.index_scores_mx(q, ones_q, w, k, ones_k, pt, sl, page_size=4)
    f8, nv2, s2 = oracle.index_scores(q, w, k, pt, sl, page_size=4, fp8=True)
    assert s1 == 0 and s2 == 0 and np.array_equal(nv1, nv2)
    assert np.array_equal(mx, f8, equal_nan=True)


def test_mx_scores_match_the_closed_form_with_group_scales():
    """I[t,s] = sum_h w ReLU(sum_d (q_d 2^(eq[d/32]-127)) (k_d 2^(ek[d/32]-127))), with the codes
    and scales decoded by torch, against the oracle's own decoding and loop."""
    q, q_mx, w, k, k_mx, pt, sl = _mx_case(502)
    B, J, H, D = q.shape
    got, nv, st = oracle.index_scores_mx(q, q_mx, w, k, k_mx, pt, sl, page_size=4)
    assert st == 0
    e8 = lambda a: torch.tensor(a).view(torch.float8_e8m0fnu).to(torch.float32).double().numpy()
    qd = q.to(torch.float32).double().numpy() * np.repeat(e8(q_mx), 32, axis=-1)
    kd = k.to(torch.float32).double().numpy() * np.repeat(e8(k_mx), 32, axis=-1)
    for b in range(B):
        for j in range(J):
            p = 11 - J + j
            assert nv[b, j] == p + 1
            for s in range(p + 1):
                key = kd[pt[b, s // 4], s % 4]
                want = float(np.sum(w[b, j].astype(np.float64) * np.maximum(qd[b, j] @ key, 0.0)))
                assert got[b, j, s] == want, (b, j, s)
            assert np.all(np.isnan(got[b, j, p + 1:]))


def test_mx_scores_refuse_scale_arrays_of_the_wrong_shape():
    q, q_mx, w, k, k_mx, pt, sl = _mx_case(503)
    with pytest.raises(ValueError):
        oracle.index_scores_mx(q, q_mx[..., :2], w, k, k_mx, pt, sl, page_size=4)


# ---------------------------------------------------------------- generators

def test_workload_generator_is_deterministic_and_shaped():
    wl = workloads.WORKLOADS[1]
    a = workloads.make_inputs(wl)
    b = workloads.make_inputs(wl)
    for key in ("q_idx", "k_cache", "w", "q_attn", "kv_cache", "page_table"):
        assert torch.equal(a[key].view(torch.uint8) if a[key].dtype != torch.float32 else a[key],
                           b[key].view(torch.uint8) if b[key].dtype != torch.float32 else b[key])
    assert a["page_table"].shape == (1, 16)
    assert sorted(a["page_table"].flatten().tolist()) == list(range(16))
    assert a["q_idx"].shape == (1, 1, 4, 32) and a["kv_cache"].shape == (16, 16, 80)
    v = a["q_idx"].float()
    assert v.min() >= -3 and v.max() <= 3 and torch.equal(v, v.round())


# ---------------------------------------------------------------- Zigzag prefill pairing (NEXT row)

def test_zigzag_assignment_matches_the_printed_example():
    from oracle import zigzag
    with open(os.path.join(GOLDEN, "zigzag_example.json")) as f:
        g = json.load(f)
    assert zigzag.assignment(g["cards"]) == g["assignment"]
    assert sorted(s for pair in g["assignment"] for s in pair) == list(range(g["shards"]))


@pytest.mark.parametrize("cards,shard_len", [(1, 5), (2, 3), (4, 16), (8, 7)])
def test_zigzag_balances_causal_load_exactly_when_the_shards_are_equal(cards, shard_len):
    """Shard i covers [iL, (i+1)L): its causal load is L*i*L + L(L+1)/2, so shards i and S-1-i
    together carry L*L*(S-1) + L(L+1) on every card, against a naive split that grows with i."""
    from oracle import zigzag
    T, S = 2 * cards * shard_len, 2 * cards
    loads = [zigzag.causal_load(p) for p in zigzag.card_positions(T, cards)]
    L = shard_len
    assert loads == [L * L * (S - 1) + L * (L + 1)] * cards
    assert sum(loads) == T * (T + 1) // 2
    naive = [zigzag.causal_load(range(i * T // cards, (i + 1) * T // cards)) for i in range(cards)]
    assert cards == 1 or naive[-1] > naive[0]


@pytest.mark.parametrize("tokens,cards", [(0, 2), (5, 2), (17, 4), (64, 8), (1000, 3)])
def test_zigzag_restore_inverts_the_assignment(tokens, cards):
    from oracle import zigzag
    pos = zigzag.card_positions(tokens, cards)
    assert sorted(t for p in pos for t in p) == list(range(tokens))
    per_card = [[("tok", t) for t in p] for p in pos]
    assert zigzag.restore(per_card, tokens, cards) == [("tok", t) for t in range(tokens)]


# ---------------------------------------------------------------- paged cache append (NEXT row)

def _torch_e4m3(x):
    return torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_encode_matches_torch_on_the_grid_on_ties_and_below_overflow():
    grid = [c for c in range(256) if not np.isnan(oracle.e4m3_value(c))]
    for c in grid:                                   # every finite code round-trips
        assert oracle.e4m3_encode(oracle.e4m3_value(c)) == c
    pos = sorted({oracle.e4m3_value(c) for c in grid if oracle.e4m3_value(c) > 0})
    ties = np.array([(a + b) / 2 for a, b in zip([0.0] + pos[:-1], pos)], dtype=np.float32)
    ties = np.concatenate([ties, -ties])             # exact midpoints: ties go to the even code
    r = rng(601)
    rand = np.concatenate([r.uniform(-463, 463, 4000), r.uniform(-0.05, 0.05, 4000)]).astype(np.float32)
    band = np.linspace(448.0, 463.9, 50, dtype=np.float32)   # rounds down to 448 in both
    for x in (ties, rand, band, -band):
        assert np.array_equal(np.array([oracle.e4m3_encode(v) for v in x], np.uint8), _torch_e4m3(x))
    assert oracle.e4m3_encode(1e6) == 0x7E and oracle.e4m3_encode(-500.0) == 0xFE   # saturation


def _append_case(seed, B=3, J=2, D=64, DC=576, P=4, pages_per_seq=3):
    r = rng(seed)
    num_pages = B * pages_per_seq + 2                # two pages no sequence uses
    pt = r.permutation(num_pages)[:B * pages_per_seq].astype(np.int32).reshape(B, pages_per_seq)
    sl = r.integers(J, pages_per_seq * P + 1, B).astype(np.int32)
    new_k = r.standard_normal((B, J, D)).astype(np.float32) * r.uniform(0.01, 100, (B, J, 1)).astype(np.float32)
    new_kv = r.standard_normal((B, J, DC)).astype(np.float32) * r.uniform(0.01, 10, (B, J, 1)).astype(np.float32)
    return pt, sl, new_k, new_kv, num_pages


def _written_rows(pt, sl, J, P):
    return {(b, j): (pt[b, (int(sl[b]) - J + j) // P], (int(sl[b]) - J + j) % P)
            for b in range(pt.shape[0]) for j in range(J)}


def test_cache_append_bf16_writes_exactly_the_new_rows():
    pt, sl, new_k, new_kv, num_pages = _append_case(602)
    B, J, D = new_k.shape
    DC, P = new_kv.shape[2], 4
    nk, nv = bf16(new_k), bf16(new_kv)               # bf16 values, as a bf16 cache holds them
    r = rng(603)
    k_cache = r.integers(0, 65536, (num_pages, P, D)).astype(np.uint16)
    kv_cache = r.integers(0, 65536, (num_pages, P, DC)).astype(np.uint16)
    k0, kv0 = k_cache.copy(), kv_cache.copy()
    assert oracle.cache_append(nk, nv, pt, sl, k_cache, kv_cache, page_size=P) == 0
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    touched = np.zeros((num_pages, P), bool)
    for (b, j), (page, off) in _written_rows(pt, sl, J, P).items():
        assert np.array_equal(k_cache[page, off], bits(nk[b, j]))
        assert np.array_equal(kv_cache[page, off], bits(nv[b, j]))
        touched[page, off] = True
    assert np.array_equal(k_cache[~touched], k0[~touched])
    assert np.array_equal(kv_cache[~touched], kv0[~touched])


def test_cache_append_fp8_scale_rules_and_codes():
    pt, sl, new_k, new_kv, num_pages = _append_case(604)
    B, J, D = new_k.shape
    DC, P = new_kv.shape[2], 4
    new_k[0, 0] = 0.0                                 # an all-zero key: scale 1, codes 0
    k_cache = np.zeros((num_pages, P, D), np.uint8)
    k_scale = np.zeros((num_pages, P), np.float32)
    kv_cache = np.zeros((num_pages, P, DC), np.uint8)
    kv_scale = np.zeros((num_pages, P, 5), np.float32)
    assert oracle.cache_append(new_k, new_kv, pt, sl, k_cache, kv_cache, page_size=P, k_mode="fp8",
                               k_scale=k_scale, kv_scale=kv_scale) == 0
    for (b, j), (page, off) in _written_rows(pt, sl, J, P).items():
        # index key: the smallest power of two s with amax <= 448 s, codes of x / s
        x = new_k[b, j]
        amax = float(np.abs(x).max())
        s = k_scale[page, off]
        if amax == 0.0:
            assert s == 1.0 and not k_cache[page, off].any()
        else:
            e = int(np.log2(s))
            assert s == 2.0 ** e and amax <= 448 * s and amax > 224 * s
            assert np.array_equal(k_cache[page, off], _torch_e4m3(x / np.float32(s)))
        # main cache: per 128-element block, scale = fp32(amax / 448), codes of fp32(x / scale)
        v = new_kv[b, j]
        for g in range(5):
            blk = v[128 * g:128 * g + 128]
            sc = np.float32(np.abs(blk).max()) / np.float32(448.0)
            assert kv_scale[page, off, g] == sc
            assert np.array_equal(kv_cache[page, off, 128 * g:128 * g + 128], _torch_e4m3(blk / sc))
        # dequantised, every element is within half an e4m3 step of its input
        deq = np.array([oracle.e4m3_value(c) for c in kv_cache[page, off]]) * np.repeat(kv_scale[page, off], 128)[:DC]
        step = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(v / np.repeat(kv_scale[page, off], 128)[:DC]), 2.0 ** -6))) - 3), 2.0 ** -9)
        assert np.all(np.abs(deq - v) <= 0.5 * step * np.repeat(kv_scale[page, off], 128)[:DC] * (1 + 1e-6))


def test_cache_append_mx_groups():
    pt, sl, new_k, new_kv, num_pages = _append_case(605, D=128)
    B, J, D = new_k.shape
    P = 4
    k_cache = np.zeros((num_pages, P, D), np.uint8)
    k_mx = np.zeros((num_pages, P, D // 32), np.uint8)
    kv_cache = np.zeros((num_pages, P, new_kv.shape[2]), np.uint16)
    assert oracle.cache_append(bf16(new_k), bf16(new_kv), pt, sl, k_cache, kv_cache, page_size=P,
                               k_mode="mx", k_scale=k_mx) == 0
    xk = bf16(new_k).float().numpy()
    for (b, j), (page, off) in _written_rows(pt, sl, J, P).items():
        for g in range(D // 32):
            x = xk[b, j, 32 * g:32 * g + 32]
            E = int(np.floor(np.log2(np.abs(x).max()))) - 8     # OCP MX shared exponent
            assert k_mx[page, off, g] == E + 127
            y = (x * np.float32(2.0 ** -E)).astype(np.float32)
            want = _torch_e4m3(np.clip(y, -448, 448))           # saturating above 448
            assert np.array_equal(k_cache[page, off, 32 * g:32 * g + 32], want)
