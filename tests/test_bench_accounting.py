"""The roofline numerator of bench.py: the algorithmic bytes of one decode batch, counted here by
hand from the shapes (every visible index-key row once, every selected latent row once, the
queries, weights and page tables in, the outputs out) and compared with what the bench uses."""
import torch

import bench
from indexed_sparse_attention_paged_b200 import workloads


def test_decode_batch_bytes_match_a_hand_count():
    wl = workloads.WORKLOADS[2]
    assert (wl.page_size, wl.idx_heads, wl.idx_dim, wl.top_k, wl.attn_heads, wl.d_latent, wl.d_rope) == \
        (64, 64, 128, 2048, 128, 512, 64)
    inputs = dict(workload=wl, batch=32, n_q=1, seq_lens=torch.full((32,), 8192, dtype=torch.int32))
    ab = bench.algorithmic_bytes(inputs)
    keys = 8192 * 128 * 2                  # every visible index-key row, bf16
    rows = 2048 * (512 + 64) * 2           # the selected latent rows, bf16
    q_attn = 128 * (512 + 64) * 2
    q_idx = 64 * 128 * 2 + 64 * 4          # index query (bf16) and head weights (fp32)
    outs = 128 * 512 * 2 + 128 * 4 + 2048 * 4   # attention out, lse, Top-K list
    tables = 128 * 4 * 2                   # the page-table row, read by each stage
    per_query = keys + rows + q_attn + q_idx + outs + tables
    assert ab["idx_k"] == 32 * keys
    assert ab["kv"] == 32 * rows
    assert ab["total"] == 32 * per_query + 32 * 4      # + the sequence lengths
    assert ab["total"] == 152_363_136


def test_causal_rows_short_of_top_k_count_only_visible_positions():
    wl = workloads.WORKLOADS[2]
    inputs = dict(workload=wl, batch=2, n_q=1, seq_lens=torch.tensor([100, 5000], dtype=torch.int32))
    ab = bench.algorithmic_bytes(inputs)
    assert ab["kv"] == (100 + 2048) * (512 + 64) * 2
    assert ab["idx_k"] == (100 + 5000) * 128 * 2


def test_decode_batch_flops_and_the_roofline_bound():
    wl = workloads.WORKLOADS[2]
    inputs = dict(workload=wl, batch=32, n_q=1, seq_lens=torch.full((32,), 8192, dtype=torch.int32))
    af = bench.algorithmic_flops(inputs)
    # logits over 576 dims and the output over 512, for 128 heads and 2048 rows, 32 queries
    assert af["stage2"] == 32 * 2048 * 128 * 2 * (576 + 512) == 18_253_611_008
    # scoring: 64 heads x 128 dims over every visible position of every query
    assert af["stage1"] == 32 * 8192 * 64 * 128 * 2
    pk = {"hbm_gbs": 6542.4, "bf16_tflops": 1663.5, "bf16_tflops_sustained": 1410.5, "source": "test"}
    ab = bench.algorithmic_bytes(inputs)
    r = bench.roofline_entry("k", ab["stage2"], af["stage2"], 0.05, pk)
    # 84.7 MB at 6542 GB/s (12.9 us) is longer than 18.25 GFLOP at 1663.5 TFLOP/s (11.0 us)
    assert r["bound"] == "hbm" and abs(r["frac"] - r["hbm_frac"]) < 1e-12
    assert abs(r["hbm_frac"] - ab["stage2"] / 50e-6 / 6542.4e9) < 1e-9
    assert abs(r["tensor_frac"] - af["stage2"] / 50e-6 / 1663.5e12) < 1e-9
    rs = bench.roofline_entry("k", ab["stage2"], af["stage2"], 0.05, pk, "bf16_tflops_sustained")
    # against the sustained peak the contraction takes 12.941 us, the bytes 12.947 us: a tie
    assert rs["bound"] == "hbm" and abs(rs["tensor_frac"] / rs["hbm_frac"] - 1.0) < 1e-3


def test_recorded_dram_traffic_is_from_the_current_sources():
    """The `traffic` the bench line carries comes from profiles/traffic.json, and only when that
    capture was taken on the kernel sources as they are now (a hash of csrc/).  Every stage the
    bench reports has such a record, and it is not far from the algorithmic bytes (a capture of
    another workload, or of a kernel that re-reads its inputs, would be)."""
    import json
    import os
    rec = json.load(open(os.path.join(os.path.dirname(bench.__file__), "profiles", "traffic.json")))
    assert set(rec) >= {"index_topk", "sparse_attend"}
    for stage in ("index_topk", "sparse_attend"):
        assert rec[stage]["source_sha"] == bench.source_sha(), stage
        assert rec[stage]["workload"] == "decode_b32_ctx8k"
        assert bench.recorded_traffic(stage) == rec[stage]["dram_bytes_per_launch"]
        assert "ncu" in rec[stage]["command"] and "--clock-control none" in rec[stage]["command"]
    wl = workloads.WORKLOADS[2]
    inputs = dict(workload=wl, batch=32, n_q=1, seq_lens=torch.full((32,), 8192, dtype=torch.int32))
    ab = bench.algorithmic_bytes(inputs)
    # the attention reads the selected rows once; the indexer reads every visible key once
    assert 0.9 * ab["kv"] < rec["sparse_attend"]["dram_bytes_per_launch"] < 1.2 * (ab["total"] - ab["idx_k"])
    assert 0.95 * ab["idx_k"] < rec["index_topk"]["dram_bytes_per_launch"] < 1.1 * ab["idx_k"] + 4e6
