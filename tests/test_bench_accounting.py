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
