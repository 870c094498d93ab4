"""Small, fixed invocations of the library for profiler captures (ncu) and quick timing.

    python -m indexed_sparse_attention_paged_b200.profile_case CASE [--calls N] [--tokens T]

CASE:
  decode          the fused decode of the B=32, context-8192 workload (index + Top-K +
                  attention + merge), N calls on one input set;
  attend          the sparse attention stage alone on the same workload (attention + merge);
  index           stage 1 alone on the same workload (scoring + Top-K);
  prefill-scoring the scoring step alone on a causal prefill chunk of T tokens (default 4096),
                  64 indexer heads x 128 dims bf16;
  decode-fp8kv    the fused decode of the same workload over an FP8 main cache;
  decode-mx       stage 1 on the same workload with MXFP8 index keys and queries.

One untimed call comes first (module loading, first-touch), then N calls, then a device
synchronisation; the process exits 0 when the device status word is clean.  Inputs are the
seeded synthetic workloads of `workloads`.
"""
from __future__ import annotations

import argparse
import sys

import torch

import indexed_sparse_attention_paged_b200 as sia
from indexed_sparse_attention_paged_b200 import workloads


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["decode", "attend", "index", "prefill-scoring", "decode-fp8kv", "decode-mx"])
    ap.add_argument("--calls", type=int, default=3)
    ap.add_argument("--tokens", type=int, default=4096)
    args = ap.parse_args(argv)
    dev = torch.device("cuda:0")
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    if args.case == "prefill-scoring":
        wl = workloads.WORKLOADS[4]
        h = workloads.make_inputs(wl, seq_lens=[args.tokens], n_q=args.tokens)
        d = workloads.to_device(h, dev)
        scores = torch.empty((1, args.tokens, h["max_pages"] * wl.page_size), dtype=torch.float32, device=dev)

        def call():
            sia.index_scores(d["q_idx"], d["w"], d["k_cache"], d["page_table"], d["seq_lens"], scores_out=scores,
                             dev_status=status)
    else:
        wl = workloads.WORKLOADS[2]
        h = workloads.make_inputs(wl)
        if args.case == "decode-fp8kv":
            h = workloads.fp8_main_cache(h)
        if args.case == "decode-mx":
            g = torch.Generator().manual_seed(7)
            B, J, H, D = h["q_idx"].shape
            h["q_idx"] = h["q_idx"].float().to(torch.float8_e4m3fn)
            h["k_cache"] = h["k_cache"].float().to(torch.float8_e4m3fn)
            h["q_mx"] = (127 + torch.randint(-1, 2, (B, J, H, D // 32), generator=g, dtype=torch.int32)).to(torch.uint8)
            pages, P = h["k_cache"].shape[:2]
            h["k_mx"] = (127 + torch.randint(-1, 2, (pages, P, D // 32), generator=g, dtype=torch.int32)).to(torch.uint8)
        d = workloads.to_device(h, dev)
        plan = sia.FusedDecodePlan(d, dev)
        topk = plan.topk

        if args.case in ("decode", "decode-fp8kv"):
            def call():
                plan()
        elif args.case == "attend":
            plan()

            def call():
                sia.sparse_mla_attend(d["q_attn"], d["kv_cache"], d["page_table"], d["seq_lens"], topk,
                                      d_latent=wl.d_latent, softmax_scale=wl.softmax_scale, out=plan.out,
                                      dev_status=status, kv_scale=d.get("kv_scale"))
        else:
            def call():
                sia.sparse_index_topk(d["q_idx"], d["w"], d["k_cache"], d["page_table"], d["seq_lens"],
                                      top_k=wl.top_k, k_scale=d["k_scale"], topk_out=topk, dev_status=status,
                                      q_mx=d.get("q_mx"), k_mx=d.get("k_mx"))
        status = plan.status if args.case in ("decode", "decode-fp8kv") else status

    call()
    torch.cuda.synchronize()
    for _ in range(args.calls):
        call()
    torch.cuda.synchronize()
    st = int(status.item())
    if st != 0:
        sys.stderr.write("device status %#x\n" % st)
        return 1
    print("%s: %d calls ok" % (args.case, args.calls))
    return 0


if __name__ == "__main__":
    sys.exit(main())
