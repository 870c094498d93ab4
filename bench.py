"""Benchmark: fused sparse-attention decode throughput on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload 2]

One step = one fused decode (indexer scoring + Top-K + sparse MLA attention + split merge) over
one batch of the decode workload (batch 32, one query token per sequence, context 8192, page
size 64, shuffled pages; indexer 64 heads x 128 dims bf16; Top-K 2048; 128 attention heads over
512+64 latent dims).  Inputs are seeded synthetic tensors (indexed_sparse_attention_paged_b200.
workloads), resident in HBM before timing.  Several independent input sets whose total is far
larger than L2 are used round-robin, so every step reads its data from HBM; K steps run back to
back between two CUDA events on the launching stream; the reported time is the mean step time,
maximum over ranks.  With N GPUs every rank runs its own independent batch (weak scaling, no
collective on the data path).

Prints one JSON line (rank 0).  The headline is the B=32 decode; the same line carries, under
`workloads`, the FP8-index decode (B=128, ragged contexts), the speculative decode (B=8, J=2,
context 131072) and the causal prefill chunk (T=16384: scoring TFLOP/s against the tensor peak,
and the full index + Top-K + attention path), unless --no-sub-workloads.  `--impl reference`
times the CPU oracle (the only reference implementation: the pages have no code) on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_SUSTAINED = 1400.0
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", type=int, default=2, choices=[2, 3, 4, 5],
                    help="2, 3, 5: fused decode (queries/s); 4: prefill indexer scoring (TFLOP/s)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub-workloads", action="store_true",
                    help="only the headline workload (no configs 3, 4, 5 in the same line)")
    ap.add_argument("--soak-s", type=float, default=1.0,
                    help="seconds of untimed steps right before the timed region, under the clock sampler")
    return ap.parse_args()


def _code_only(text: str) -> str:
    """C/C++/CUDA source with comments removed and whitespace runs collapsed, string and
    character literals kept as they are."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            i = text.find("\n", i)
            i = n if i < 0 else i
        elif text.startswith("/*", i):
            i = text.find("*/", i + 2)
            i = n if i < 0 else i + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def source_sha() -> str:
    """Hash of the CUDA sources' code (comments and layout ignored), to tell whether recorded
    ncu counters are still current."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "indexed_sparse_attention_paged_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(f.encode() + _code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def input_bytes(inputs) -> int:
    return sum(v.numel() * v.element_size() for v in inputs.values() if hasattr(v, "numel"))


def step_bytes(inputs) -> int:
    return algorithmic_bytes(inputs)["total"]


def algorithmic_bytes(inputs) -> dict:
    """Bytes the step must move at minimum: every visible index-K row once per sequence (plus its
    scale), every selected latent row once per query, the queries, weights and page tables in,
    the outputs (attention out, lse, Top-K) out.  Score and split workspaces are not counted."""
    wl = inputs["workload"]
    B, J = inputs["batch"], inputs["n_q"]
    lens = [int(x) for x in inputs["seq_lens"]]
    idx_elem = 1 if wl.idx_fp8 else 2
    idx_k = sum(lens) * wl.idx_dim * idx_elem + (sum(lens) * 4 if wl.idx_fp8 else 0)
    sel = sum(min(wl.top_k, L - J + j + 1) for L in lens for j in range(J))
    kv = sel * (wl.d_latent + wl.d_rope) * 2
    q_idx = B * J * wl.idx_heads * wl.idx_dim * idx_elem + B * J * wl.idx_heads * 4
    q_attn = B * J * wl.attn_heads * (wl.d_latent + wl.d_rope) * 2
    pt = sum((L + wl.page_size - 1) // wl.page_size for L in lens) * 4 * 2 + B * 4
    out = B * J * wl.attn_heads * wl.d_latent * 2 + B * J * wl.attn_heads * 4 + B * J * wl.top_k * 4
    stage1 = idx_k + q_idx + pt // 2 + B * J * wl.top_k * 4
    stage2 = kv + q_attn + pt // 2 + B * J * wl.top_k * 4 + B * J * wl.attn_heads * (wl.d_latent * 2 + 4)
    return dict(total=idx_k + kv + q_idx + q_attn + pt + out, stage1=stage1, stage2=stage2,
                idx_k=idx_k, kv=kv)


def algorithmic_flops(inputs) -> dict:
    """Tensor-core work of one step: the scoring contraction over every visible (query,
    position) pair (2 * H_i * D_i each) and the attention over every selected row of every query
    (2 * H_a * (d_latent + d_rope) for the logits plus 2 * H_a * d_latent for the output)."""
    wl = inputs["workload"]
    J = inputs["n_q"]
    lens = [int(x) for x in inputs["seq_lens"]]
    pairs = sum(L - J + j + 1 for L in lens for j in range(J))
    sel = sum(min(wl.top_k, L - J + j + 1) for L in lens for j in range(J))
    stage1 = 2 * wl.idx_heads * wl.idx_dim * pairs
    stage2 = 2 * wl.attn_heads * sel * ((wl.d_latent + wl.d_rope) + wl.d_latent)
    return dict(stage1=stage1, stage2=stage2, total=stage1 + stage2)


def roofline_entry(kernel, nbytes, flops, ms, pk, tensor_peak_key="bf16_tflops"):
    """Roofline of one timed call: achieved bytes/s and FLOP/s against the measured peaks.  The
    bound is the resource whose roofline time (bytes / bandwidth, FLOPs / tensor peak) is the
    longer; `frac` is achieved / peak for that bound, and both fractions are given."""
    gbs = nbytes / (ms / 1000.0) / 1e9
    tfs = flops / (ms / 1000.0) / 1e12
    t_hbm = nbytes / (pk["hbm_gbs"] * 1e9)
    t_tc = flops / (pk[tensor_peak_key] * 1e12) if flops else 0.0
    hbm = t_hbm >= t_tc
    return {"bound": "hbm" if hbm else "tensor", "kernel": kernel,
            "achieved": gbs if hbm else tfs, "peak": pk["hbm_gbs"] if hbm else pk[tensor_peak_key],
            "unit": "GB/s" if hbm else "TFLOP/s",
            "frac": gbs / pk["hbm_gbs"] if hbm else tfs / pk[tensor_peak_key],
            "hbm_frac": gbs / pk["hbm_gbs"], "tensor_frac": tfs / pk[tensor_peak_key],
            "achieved_gbs": gbs, "achieved_tflops": tfs,
            "roofline_us": max(t_hbm, t_tc) * 1e6,
            "peak_source": "%s (HBM copy; bf16 %s)" % (pk["source"], "burst" if tensor_peak_key == "bf16_tflops" else "sustained"),
            "algorithmic_bytes_per_launch": nbytes, "flops_per_launch": flops, "ms_per_launch": ms}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons every 200 ms while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def peaks() -> dict:
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        burst = float(p["bf16_tflops"])
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": burst,
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", burst)), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": FALLBACK_BF16_SUSTAINED, "source": "fallback"}


# What each stage-level roofline entry times: one C-ABI call, i.e. both kernels of the stage.
STAGE_KERNELS = {
    "sparse_attend": "sparse_attend_kernel + combine_kernel (one sia_sparse_mla_attend call)",
    "index_topk": "index_score_kernel + topk_row_kernel (one sia_sparse_index_topk call)",
}


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this source."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        rec = t.get(kernel)
        if rec and rec.get("source_sha") == source_sha():
            return rec.get("dram_bytes_per_launch")
    except (OSError, ValueError):
        pass
    return None


def cpu_baseline(inputs, rows):
    """The oracle, as it stands, on a bounded sample of query rows: scoring, Top-K, attention."""
    import oracle
    wl = inputs["workload"]
    ks = None if inputs["k_scale"] is None else inputs["k_scale"].numpy()
    pt, sl = inputs["page_table"].numpy(), inputs["seq_lens"].numpy()
    t0 = time.perf_counter()
    topk, _, _ = oracle.index_topk(inputs["q_idx"], inputs["w"].numpy(), inputs["k_cache"], pt, sl,
                                   page_size=wl.page_size, top_k=wl.top_k, fp8=wl.idx_fp8, k_scale=ks,
                                   rows=rows)
    oracle.sparse_attend(inputs["q_attn"], inputs["kv_cache"], pt, sl, topk, page_size=wl.page_size,
                         d_latent=wl.d_latent, scale=wl.softmax_scale, rows=rows)
    dt = time.perf_counter() - t0
    return dict(value=len(rows) / dt, unit="queries/s", cores=oracle.num_threads(), kind="oracle",
                sample="%d of the %d query rows (rows %d..%d), full scoring + Top-K + attention each; %.1f s"
                       % (len(rows), inputs["batch"] * inputs["n_q"], rows[0], rows[-1], dt))


def run_reference(args, rank, world):
    from indexed_sparse_attention_paged_b200 import workloads
    import oracle
    if rank != 0:
        return
    wl = workloads.WORKLOADS[args.workload]
    inputs = workloads.make_inputs(wl)
    n = max(4, min(16, oracle.num_threads()))
    rows = list(range(n))
    for _ in range(args.warmup and 1):
        cpu_baseline(inputs, rows[:1])
    vals = []
    for _ in range(args.steps):
        vals.append(cpu_baseline(inputs, rows))
    v = statistics.mean(x["value"] for x in vals)
    cb = dict(vals[-1])
    cb["value"] = v
    # a step is the whole batch: its time at the sampled rate
    queries = inputs["batch"] * inputs["n_q"]
    line = dict(impl="reference", metric=metric_name(wl), value=v, unit="queries/s", n_gpus=args.gpus,
                steps=args.steps, warmup=args.warmup, ms_per_step=1000.0 * queries / v,
                higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                config=config_of(wl, inputs, "cpu (no L2 flush)"), cpu_baseline=cb,
                e2e={"value": v, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0})
    print(json.dumps(line), flush=True)


def max_over_ranks(values, device):
    """Each value's maximum over the ranks of the job (device times: a job is as slow as its
    slowest rank).  One all-reduce; identity when there is no process group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_rate(world, units_per_rank, ms):
    """Whole-job throughput: every rank processed units_per_rank in (at most) ms."""
    return world * units_per_rank / (ms / 1000.0)


def metric_name(wl):
    return "fused sparse-attn decode queries/s @B=%d ctx=%s; achieved HBM GB/s %% of peak" % (
        wl.batch, "8K" if wl.context == 8192 else str(wl.context or "1k-32k"))


class PackedIO:
    """One step's host<->device traffic as one copy per direction: the per-step inputs packed in
    one pinned host buffer and one device staging buffer (256-byte aligned views), the outputs
    (attention out, lse, Top-K lists) in one device buffer and one pinned host buffer.  A
    fused-decode plan built on the staging views reads its inputs and writes its outputs there;
    the caches stay resident, as a serving KV cache does."""

    IN_KEYS = ("q_idx", "w", "q_attn", "page_table", "seq_lens")

    @staticmethod
    def _layout(specs):
        off, out = 0, []
        for shape, dtype in specs:
            n = 1
            for x in shape:
                n *= x
            nbytes = n * torch_dtype_size(dtype)
            out.append((off, nbytes, shape, dtype))
            off = (off + nbytes + 255) // 256 * 256
        return out, off

    def __init__(self, sia, d, host, dev):
        import torch
        wl = host["workload"]
        B, J = host["batch"], host["n_q"]
        in_specs = [(tuple(host[k].shape), host[k].dtype) for k in self.IN_KEYS]
        self.in_lay, in_bytes = self._layout(in_specs)
        out_specs = [((B, J, wl.attn_heads, wl.d_latent), torch.bfloat16), ((B, J, wl.attn_heads), torch.float32),
                     ((B, J, wl.top_k), torch.int32)]
        self.out_lay, out_bytes = self._layout(out_specs)
        self.h_in = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
        self.d_in = torch.empty(in_bytes, dtype=torch.uint8, device=dev)
        self.d_out = torch.empty(out_bytes, dtype=torch.uint8, device=dev)
        self.h_out = torch.empty(out_bytes, dtype=torch.uint8).pin_memory()
        view = lambda buf, lay: buf[lay[0]:lay[0] + lay[1]].view(lay[3]).view(lay[2])
        for k, lay in zip(self.IN_KEYS, self.in_lay):
            view(self.h_in, lay).copy_(host[k])
        ds = dict(d)
        for k, lay in zip(self.IN_KEYS, self.in_lay):
            ds[k] = view(self.d_in, lay)
        out, lse, topk = (view(self.d_out, lay) for lay in self.out_lay)
        self.plan = sia.FusedDecodePlan(ds, dev, out=out, lse=lse, topk=topk)
        self.h_views = tuple(view(self.h_out, lay) for lay in self.out_lay)
        self.h2d_bytes, self.d2h_bytes = in_bytes, out_bytes

    def step(self, stream_in=None, stream_cmp=None, stream_out=None):
        import torch
        with torch.cuda.stream(stream_in or torch.cuda.current_stream()):
            self.d_in.copy_(self.h_in, non_blocking=True)
        self.plan(stream=stream_cmp)
        with torch.cuda.stream(stream_out or torch.cuda.current_stream()):
            self.h_out.copy_(self.d_out, non_blocking=True)


def torch_dtype_size(dtype) -> int:
    import torch
    return torch.empty((), dtype=dtype).element_size()


def e2e_pipelined(sia, d, host, dev, compute, steps, ref):
    """Mean time per step of the end-to-end loop with copies overlapped across steps.

    Two slots, each a PackedIO (its own staging, plan and pinned host buffers; the caches are
    shared).  Step i uses slot i % 2: the copy-in on `s_in` after the slot's previous call has
    read its inputs, the fused call on `compute` after the copy-in and after the slot's previous
    outputs were copied out, the copy-out on `s_out` after the call.  The outputs are checked
    against the serial loop's (`ref`).
    """
    import torch
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    slots = []
    for _ in range(2):
        io = PackedIO(sia, d, host, dev)
        ev = {k: torch.cuda.Event() for k in ("in", "cmp", "out")}
        slots.append((io, ev))

    def step(i):
        io, ev = slots[i & 1]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev["cmp"])
            io.d_in.copy_(io.h_in, non_blocking=True)
            ev["in"].record(s_in)
        compute.wait_event(ev["in"])
        compute.wait_event(ev["out"])
        io.plan(stream=compute)
        ev["cmp"].record(compute)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["cmp"])
            io.h_out.copy_(io.d_out, non_blocking=True)
            ev["out"].record(s_out)

    torch.cuda.synchronize()
    for i in range(4):
        step(i)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for i in range(steps):
        step(i)
    end.record(s_out)   # after the last copy-out, which follows every earlier operation
    torch.cuda.synchronize()
    for io, ev in slots:
        if int(io.plan.status.item()) != 0 or not all(torch.equal(h, r) for h, r in zip(io.h_views, ref)):
            raise RuntimeError("pipelined outputs differ from the serial loop's")
    return start.elapsed_time(end) / steps


def config_of(wl, inputs, l2):
    return {"workload": wl.name, "batch": inputs["batch"], "n_q": inputs["n_q"],
            "context": wl.context or "uniform[%d,%d]" % (wl.len_lo, wl.len_hi),
            "page_size": wl.page_size, "idx_heads": wl.idx_heads, "idx_dim": wl.idx_dim,
            "idx_dtype": "e4m3" if wl.idx_fp8 else "bf16", "top_k": wl.top_k,
            "attn_heads": wl.attn_heads, "d_latent": wl.d_latent, "d_rope": wl.d_rope,
            "l2": l2, "parallelism": "replicas"}


def prefill_scoring_flops(seq_lens, n_q, heads, dim) -> int:
    """FLOPs of the causal q.k contraction: 2 * D * H per (query, visible position)."""
    total = 0
    for L in seq_lens:
        first = int(L) - n_q                 # query j sits at position L - n_q + j and sees 0..pos
        total += sum(first + j + 1 for j in range(n_q))
    return 2 * heads * dim * total


def measure_prefill(dev, wl, rank, steps, warmup, full_path):
    """Causal prefill chunk (T = 16384): the indexer's scoring step alone (sia_index_scores), in
    TFLOP/s of the causal q.k contraction against the measured bf16 tensor peaks; with
    `full_path`, also the whole path for the chunk (sia_sparse_index_topk over the 1 GiB score
    workspace, then sia_sparse_mla_attend for every query), timed once per step."""
    import torch
    import indexed_sparse_attention_paged_b200 as sia
    from indexed_sparse_attention_paged_b200 import workloads

    host = workloads.make_inputs(wl, seed=1000 + wl.number + 7919 * rank)
    d = workloads.to_device(host, dev)
    B, J = host["batch"], host["n_q"]
    Lpad = host["max_pages"] * wl.page_size
    scores = torch.empty((B, J, Lpad), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        sia.index_scores(d["q_idx"], d["w"], d["k_cache"], d["page_table"], d["seq_lens"],
                         k_scale=d["k_scale"], scores_out=scores, dev_status=status, stream=stream)

    for _ in range(max(3, warmup)):
        step()
    torch.cuda.synchronize()
    n = max(1, min(steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    if int(status.item()) != 0:
        raise RuntimeError("device status %d" % int(status.item()))
    flops = prefill_scoring_flops(host["seq_lens"].tolist(), J, wl.idx_heads, wl.idx_dim)
    out = {"ms_per_step": ms, "steps": n, "flops_per_launch": flops, "launches": n}
    out["_ms"] = ms
    out["_flops"] = flops
    if full_path:
        topk = torch.empty((B, J, wl.top_k), dtype=torch.int32, device=dev)
        att = torch.empty((B, J, wl.attn_heads, wl.d_latent), dtype=torch.bfloat16, device=dev)
        ws1 = torch.empty(max(256, sia.load_library().sia_index_workspace_size(__import__("ctypes").byref(
            sia.index_args(d["q_idx"], d["w"], d["k_cache"], d["page_table"], d["seq_lens"], top_k=wl.top_k,
                           topk_out=topk)))), dtype=torch.uint8, device=dev)

        def full():
            sia.sparse_index_topk(d["q_idx"], d["w"], d["k_cache"], d["page_table"], d["seq_lens"],
                                  top_k=wl.top_k, k_scale=d["k_scale"], topk_out=topk, workspace=ws1,
                                  dev_status=status, stream=stream)
            sia.sparse_mla_attend(d["q_attn"], d["kv_cache"], d["page_table"], d["seq_lens"], topk,
                                  d_latent=wl.d_latent, softmax_scale=wl.softmax_scale, out=att,
                                  dev_status=status, stream=stream)
        full()
        torch.cuda.synchronize()
        nf = 3
        e0.record(stream)
        for _ in range(nf):
            full()
        e1.record(stream)
        torch.cuda.synchronize()
        fms = e0.elapsed_time(e1) / nf
        if int(status.item()) != 0:
            raise RuntimeError("device status %d" % int(status.item()))
        ab = algorithmic_flops(host)
        out["full_path"] = {"ms_per_step": fms, "queries_per_s": B * J / (fms / 1000.0), "steps": nf,
                            "calls": "sia_sparse_index_topk (score workspace %.2f GiB) + sia_sparse_mla_attend"
                                     % (B * J * Lpad * 4 / 2 ** 30),
                            "tensor_flops": ab["total"],
                            "achieved_tflops": ab["total"] / (fms / 1000.0) / 1e12}
        out["launches"] += nf * 4
        del topk, att, ws1
    del scores, d
    torch.cuda.empty_cache()
    return out


def prefill_entry(res, pk, wl):
    ms, flops = res["_ms"], res["_flops"]
    tflops = flops / (ms / 1000.0) / 1e12
    e = {"workload": wl.name, "metric": "prefill indexer scoring TFLOP/s @T=%d causal, %dx%d bf16"
         % (wl.context, wl.idx_heads, wl.idx_dim),
         "value": tflops, "unit": "TFLOP/s", "ms_per_step": ms, "steps": res["steps"],
         "roofline": {"bound": "tensor", "kernel": "index_score_kernel (one sia_index_scores call)",
                      "achieved": tflops, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                      "frac": tflops / pk["bf16_tflops"], "peak_source": pk["source"] + " burst",
                      "frac_of_sustained": tflops / pk["bf16_tflops_sustained"],
                      "traffic": None, "flops_per_launch": flops}}
    if "full_path" in res:
        e["full_path"] = res["full_path"]
    return e


def run_prefill_scoring(args, rank, world, dev, wl):
    """`--workload 4` as the headline: the prefill scoring line."""
    import torch.distributed as dist
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    sampler.start()
    if world > 1:
        dist.barrier()
    res = measure_prefill(dev, wl, rank, args.steps, args.warmup, full_path=False)
    clocks = sampler.stop()
    (ms,) = max_over_ranks([res["_ms"]], dev)
    res["_ms"] = ms
    pk = peaks()
    e = prefill_entry(res, pk, wl)
    if rank == 0:
        line = {"metric": e["metric"], "value": world * e["value"], "unit": "TFLOP/s", "n_gpus": world,
                "steps": res["steps"], "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": wl.name, "tokens": wl.context, "idx_heads": wl.idx_heads,
                           "idx_dim": wl.idx_dim,
                           "l2": "the 16384 x 256 B index keys (4 MB) are L2-resident by design: the "
                                 "contraction reuses each key tile for every query group",
                           "parallelism": "replicas"},
                "roofline": e["roofline"], "gpu_launches": res["launches"], "clocks": clocks}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


class DecodeBench:
    """One decode workload on this rank: input sets (round-robin, larger than L2 together),
    one fused-decode plan per set, and the stage-only calls for the per-stage rooflines."""

    def __init__(self, sia, workloads, wl, rank, dev, min_sets):
        import ctypes
        import torch
        self.wl = wl
        self.host = workloads.make_inputs(wl, seed=1000 + wl.number + 7919 * rank)
        per_step = step_bytes(self.host)
        self.n_sets = max(min_sets, -(-4 * L2_BYTES // max(1, per_step))) if per_step < 4 * L2_BYTES else min_sets
        self.sets = [workloads.to_device(self.host, dev)]
        for i in range(1, self.n_sets):
            self.sets.append(workloads.to_device(
                workloads.make_inputs(wl, seed=1000 + wl.number + 7919 * rank + 104729 * i), dev))
        self.plans = [sia.FusedDecodePlan(d, dev) for d in self.sets]
        self.stream = torch.cuda.current_stream()
        lib = sia.load_library()
        sp = ctypes.c_void_p(self.stream.cuda_stream)
        self.stage1, self.stage2 = [], []
        for pl in self.plans:
            ws1 = torch.empty(max(256, lib.sia_index_workspace_size(ctypes.byref(pl.ia))), dtype=torch.uint8, device=dev)
            ws2 = torch.empty(max(256, lib.sia_attend_workspace_size(ctypes.byref(pl.aa))), dtype=torch.uint8, device=dev)
            st_ptr = ctypes.c_void_p(pl.status.data_ptr())

            def f1(pl=pl, ws1=ws1, st_ptr=st_ptr):
                sia._check(lib.sia_sparse_index_topk(ctypes.byref(pl.ia), ctypes.c_void_p(ws1.data_ptr()), ws1.numel(), st_ptr, sp))

            def f2(pl=pl, ws2=ws2, st_ptr=st_ptr):
                sia._check(lib.sia_sparse_mla_attend(ctypes.byref(pl.aa), ctypes.c_void_p(ws2.data_ptr()), ws2.numel(), st_ptr, sp))
            self.stage1.append(f1)
            self.stage2.append(f2)
        self.kernels_per_step = 3 + (1 if plan_splits(lib, self.plans[0].aa) > 1 else 0)

    def timed(self, fns, steps):
        """Mean device time per call of fns[i % len(fns)], back to back, CUDA events."""
        import torch
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(self.stream)
        for i in range(steps):
            fns[i % len(fns)]()
        e.record(self.stream)
        torch.cuda.synchronize()
        return s.elapsed_time(e) / steps

    def warm(self, n):
        import torch
        for i in range(n):
            self.plans[i % self.n_sets]()
        for f in self.stage1 + self.stage2:
            f()
        torch.cuda.synchronize()

    def soak(self, seconds):
        """Untimed steps back to back for about `seconds` (the clock sampler runs meanwhile)."""
        import torch
        t0 = time.perf_counter()
        i = 0
        while time.perf_counter() - t0 < seconds:
            for _ in range(64):
                self.plans[i % self.n_sets]()
                i += 1
            torch.cuda.synchronize()
        return i

    def check_status(self):
        bad = [int(pl.status.item()) for pl in self.plans if int(pl.status.item()) != 0]
        if bad:
            raise RuntimeError("device status %#x during the benchmark" % bad[0])

    def entry(self, step_ms, s1, s2, pk, steps):
        host = self.host
        queries = host["batch"] * host["n_q"]
        ab = algorithmic_bytes(host)
        af = algorithmic_flops(host)
        r2 = roofline_entry(STAGE_KERNELS["sparse_attend"], ab["stage2"], af["stage2"], s2, pk)
        r1 = roofline_entry(STAGE_KERNELS["index_topk"], ab["stage1"], af["stage1"], s1, pk)
        dominant = "sparse_attend" if s2 >= s1 else "index_topk"
        roof = dict(r2 if dominant == "sparse_attend" else r1)
        roof["traffic"] = recorded_traffic(dominant)
        return {
            "workload": self.wl.name, "metric": metric_name(self.wl), "value": queries / (step_ms / 1000.0),
            "unit": "queries/s", "ms_per_step": step_ms, "steps": steps,
            "config": config_of(self.wl, host, "inputs larger than L2: %d input set(s), %.0f MB of cache bytes "
                                "read per step" % (self.n_sets, ab["total"] / 1e6)),
            "achieved_hbm_gbs": ab["total"] / (step_ms / 1000.0) / 1e9,
            "hbm_frac_of_measured": ab["total"] / (step_ms / 1000.0) / 1e9 / pk["hbm_gbs"],
            "hbm_frac_of_8tbs": ab["total"] / (step_ms / 1000.0) / 1e9 / 8000.0,
            "roofline": roof,
            "stages": {"index_topk_ms": s1, "sparse_attend_ms": s2, "index_topk": r1, "sparse_attend": r2,
                       "step_algorithmic_bytes": ab["total"], "step_tensor_flops": af["total"]},
        }


def bind_to_gpu_cpus(dev_index: int):
    """Restrict this process to the CPUs NVML names as local to the GPU (its NUMA node), so that
    the pinned host buffers of the end-to-end loop are allocated next to the GPU's PCIe root.
    A process setting, not a GPU one; returns (cpus kept, the previous affinity) or None."""
    try:
        import pynvml
        import torch
        before = os.sched_getaffinity(0)
        pr = torch.cuda.get_device_properties(dev_index)
        bus = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
        pynvml.nvmlInit()
        try:
            handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            words = (os.cpu_count() + 63) // 64
            mask = pynvml.nvmlDeviceGetCpuAffinity(handle, words)
        finally:
            pynvml.nvmlShutdown()
        cpus = {64 * w + b for w, m in enumerate(mask) for b in range(64) if (int(m) >> b) & 1} & before
        if not cpus or cpus == before:
            return None
        os.sched_setaffinity(0, cpus)
        return sorted(cpus), before
    except Exception:
        return None


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    import indexed_sparse_attention_paged_b200 as sia
    from indexed_sparse_attention_paged_b200 import build as cuda_build
    from indexed_sparse_attention_paged_b200 import workloads

    cuda_build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    binding = bind_to_gpu_cpus(local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=120))

    wl = workloads.WORKLOADS[args.workload]
    if wl.number == 4:
        return run_prefill_scoring(args, rank, world, dev, wl)
    db = DecodeBench(sia, workloads, wl, rank, dev, min_sets=2)
    host, d, plan = db.host, db.sets[0], db.plans[0]
    db.warm(max(3, args.warmup))

    # ---------------- timed region (the clock sampler runs over a soak of the same steps right
    # before it, so that its median rests on many samples under load, and over the region itself)
    sampler = ClockSampler(local)
    sampler.start()
    db.soak(args.soak_s)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    mean_ms = db.timed(db.plans, args.steps)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    wall = time.perf_counter() - t_wall
    s1 = db.timed(db.stage1, args.steps)
    s2 = db.timed(db.stage2, args.steps)
    clocks = sampler.stop()
    db.check_status()
    mean_ms, s1, s2 = max_over_ranks([mean_ms, s1, s2], dev)

    # ---------------- end-to-end through the C ABI with host buffers: every step copies its
    # inputs in from pinned host memory and its outputs back (one packed copy per direction)
    io = PackedIO(sia, d, host, dev)
    h2d, d2h = io.h2d_bytes, io.d2h_bytes

    n_e2e = max(10, args.steps // 4)
    for _ in range(2):
        io.step()
    torch.cuda.synchronize()
    serial_ms = db.timed([io.step], n_e2e)
    ref = tuple(v.clone() for v in io.h_views)
    # The same calls as a serving loop issues them: two slots of per-step input and output
    # buffers, the host->device copies on one stream, the fused call on another, the
    # device->host copies on a third, so neighbouring steps' copies overlap the compute.
    try:
        pipe_ms = e2e_pipelined(sia, d, host, dev, db.stream, n_e2e, ref)
    except Exception as exc:  # reported below; the serial figure stands
        sys.stderr.write("pipelined end-to-end loop failed: %r\n" % (exc,))
        pipe_ms = float("inf")
    serial_ms, pipe_ms = max_over_ranks([serial_ms, pipe_ms], dev)
    pipelined = pipe_ms < serial_ms
    e2e_ms = pipe_ms if pipelined else serial_ms

    queries = host["batch"] * host["n_q"]
    pk = peaks()
    head = db.entry(mean_ms, s1, s2, pk, args.steps)
    line = {
        "metric": head["metric"], "value": job_rate(world, queries, mean_ms), "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": config_of(wl, host, "inputs larger than L2: %d independent input sets (%.0f MB) used round-robin"
                            % (db.n_sets, db.n_sets * input_bytes(host) / 1e6)),
        "achieved_hbm_gbs": head["achieved_hbm_gbs"],
        "hbm_frac_of_measured": head["hbm_frac_of_measured"],
        "hbm_frac_of_8tbs": head["hbm_frac_of_8tbs"],
        "roofline": head["roofline"],
        "stages": head["stages"],
        "e2e": {"value": job_rate(world, queries, e2e_ms), "unit": "queries/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "loop": ("pipelined: 2 buffer slots, copy-in / compute / copy-out streams" if pipelined
                         else "serial: copy-in, fused call, copy-out on one stream") +
                        "; one packed pinned-host copy per direction per step",
                "serial_ms_per_step": serial_ms,
                "host_cpus": ("%d CPUs local to the GPU (NVML affinity)" % len(binding[0])) if binding
                             else "unrestricted"},
        "gpu_launches": db.kernels_per_step * args.steps,
        "clocks": dict(clocks, window="nvidia-smi every 200 ms over a %.1f s soak of the same steps "
                                      "right before the timed region, the timed region and the "
                                      "stage timings" % args.soak_s),
        "wall_s_timed_region": wall,
    }
    # ---------------- the other configurations, in the same run (not part of the headline)
    if not args.no_sub_workloads:
        del db, d, plan, io
        torch.cuda.empty_cache()
        subs = {}
        for num in (3, 5):
            w2 = workloads.WORKLOADS[num]
            sb = DecodeBench(sia, workloads, w2, rank, dev, min_sets=1)
            sb.warm(3)
            n = max(10, min(args.steps, 200))
            m = sb.timed(sb.plans, n)
            a1 = sb.timed(sb.stage1, n)
            a2 = sb.timed(sb.stage2, n)
            sb.check_status()
            m, a1, a2 = max_over_ranks([m, a1, a2], dev)
            subs[w2.name] = sb.entry(m, a1, a2, pk, n)
            line["gpu_launches"] += sb.kernels_per_step * n
            del sb
            torch.cuda.empty_cache()
        w4 = workloads.WORKLOADS[4]
        res = measure_prefill(dev, w4, rank, min(args.steps, 20), 3, full_path=True)
        (res["_ms"],) = max_over_ranks([res["_ms"]], dev)
        subs[w4.name] = prefill_entry(res, pk, w4)
        line["gpu_launches"] += res["launches"]
        line["workloads"] = subs
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        if binding:
            os.sched_setaffinity(0, binding[1])   # the oracle runs on all of the host's cores again
        n = max(4, min(16, oracle.num_threads()))
        line["cpu_baseline"] = cpu_baseline(host, list(range(n)))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def plan_splits(lib, aa) -> int:
    """Top-K splits the library picks for this attention call (from its workspace size)."""
    import ctypes
    return 2 if lib.sia_attend_workspace_size(ctypes.byref(aa)) > 0 else 1


if __name__ == "__main__":
    main()
