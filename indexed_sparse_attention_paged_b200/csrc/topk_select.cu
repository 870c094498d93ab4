// topk_select.cu -- exact per-query Top-K of the index scores (radix select).
//
// For each query row, picks the K positions with the largest score, ties going to the lower
// position, and writes them in ascending order, padded with -1 when fewer than K positions are
// visible ("Day 0 Inference Adaptation and Performance Optimization for Hybrid Sparse Attention
// LLMs", section "Operator Fusion and Multi-Stream Scheduling", step 3; the fused index
// operator outputs only these indices, "Rapid Adaptation and Inference Optimization",
// section IV.4.1).
//
// Design: keys are the scores mapped to order-preserving uint32 (-0.0 folded onto +0.0).
// Three MSB-first radix passes (11, 11, 10 bits) find the exact K-th largest key T; the
// selection is then every key > T plus the lowest-positioned keys == T, compacted in position
// order with prefix sums, which makes the output ascending without a sort.
//   - Rows of up to 16384 positions (topk_row_kernel): 1024 threads per row (512 and two rows
//     per CTA for rows of up to 8192), 16 consecutive keys per thread in registers,
//     shared-memory histograms with plain atomics, three barriers per pass.
//   - Longer rows (topk_kernel): a thread-block cluster of 2-16 CTAs per row, each keeping a
//     slice of the keys in shared memory; the per-CTA digit histograms are summed across the
//     cluster through distributed shared memory.
#include <cuda_runtime.h>

#include "sia_common.cuh"
#include "sia_internal.h"
#include "sia_ptx.cuh"

namespace sia {
namespace {

constexpr int kBins = 2048;

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;  // -0.0 ranks as +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct TopkShared {
  uint32_t hist[2][kBins];
  int scan[kTopkThreads / 32];
  int scan2[kTopkThreads / 32];
  uint32_t sel_prefix;
  int sel_krem;
  int cta_gt, cta_eq;
};

// Block-wide exclusive prefix sum of (a, b) over threads in thread order; also returns totals.
__device__ __forceinline__ void block_scan2(int a, int b, int& ea, int& eb, int& ta, int& tb,
                                            TopkShared* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int va = __shfl_up_sync(0xffffffffu, ia, o);
    const int vb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) { ia += va; ib += vb; }
  }
  if (lane == 31) { sh->scan[warp] = ia; sh->scan2[warp] = ib; }
  __syncthreads();
  int wa = 0, wb = 0;
  ta = 0; tb = 0;
  for (int w = 0; w < kTopkThreads / 32; ++w) {
    if (w < warp) { wa += sh->scan[w]; wb += sh->scan2[w]; }
    ta += sh->scan[w];
    tb += sh->scan2[w];
  }
  ea = wa + ia - a;
  eb = wb + ib - b;
  __syncthreads();
}

__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(const TopkKernelParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  TopkShared* sh = reinterpret_cast<TopkShared*>(smem);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + sizeof(TopkShared));
  const int tid = threadIdx.x;
  const uint32_t rank = cluster_ctarank();
  const int C = p.cluster;
  const long long row = blockIdx.x / C;
  const int b = (int)(row / p.J), j = (int)(row - (long long)b * p.J);
  int32_t* out = p.topk + row * p.K;

  pdl_wait_primary();  // scores come from the previous kernel on the stream

  bool bad = false;
  const int pos = query_position(p.seq_lens, p.q_pos, p.J, b, j, p.Lpad, &bad);
  if (bad && rank == 0 && tid == 0) report(p.status, SIA_DEV_BAD_POSITION);
  const int n = pos + 1;  // visible positions 0..pos
  if (n <= p.K) {
    // everything visible is selected: 0..n-1 then -1 padding (no scores needed)
    for (int i = rank * kTopkThreads + tid; i < p.K; i += C * kTopkThreads) out[i] = i < n ? i : -1;
    pdl_launch_dependents();
    return;
  }

  // ---- load this CTA's slice of keys
  const int s0 = rank * p.slice;
  const int len = max(0, min(n - s0, p.slice));
  const float* src = p.scores + row * p.Lpad + s0;
  for (int i = tid; i < len; i += kTopkThreads) keys[i] = order_key(src[i]);

  // ---- three radix passes to find the K-th largest key
  uint32_t prefix = 0;
  int krem = p.K;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    uint32_t* h = sh->hist[pass & 1];
    for (int i = tid; i < kBins; i += kTopkThreads) h[i] = 0;
    __syncthreads();
    const int sh_ = shifts[pass];
    const int hi_shift = sh_ + widths[pass];  // bits above this digit must equal the prefix
    const uint32_t dmask = (1u << widths[pass]) - 1u;
    const int rounds = (len + kTopkThreads - 1) / kTopkThreads;
    for (int r = 0; r < rounds; ++r) {
      const int i = r * kTopkThreads + tid;
      if (i < len) {
        // plain shared-memory atomics: on sm_100a they absorb same-bin conflicts far faster
        // than a warp-level __match_any_sync aggregation (measured 1.9k vs 8k-33k cycles per
        // 16k-key pass, growing with the number of distinct bins)
        const uint32_t k = keys[i];
        if (pass == 0 || (k >> hi_shift) == prefix) atomicAdd(&h[(k >> sh_) & dmask], 1u);
      }
    }
    // make every CTA's histogram visible cluster-wide, then sum them
    cluster_sync();
    // each thread owns 4 consecutive bins; count of keys in bins above, found by a suffix scan
    constexpr int per = kBins / kTopkThreads;   // 4 consecutive bins: one 16-byte load per CTA
    static_assert(per == 4, "one v4 load per cluster CTA");
    uint32_t cnt[per] = {0u, 0u, 0u, 0u};
    {
      uint4 v[16];
      const uint32_t local = smem_u32(&h[tid * per]);
#pragma unroll
      for (int r = 0; r < 16; ++r)
        if (r < C) v[r] = ld_cluster_v4(mapa_shared(local, (uint32_t)r));
#pragma unroll
      for (int r = 0; r < 16; ++r)
        if (r < C) {
          cnt[0] += v[r].x;
          cnt[1] += v[r].y;
          cnt[2] += v[r].z;
          cnt[3] += v[r].w;
        }
    }
    const int mine = (int)(cnt[0] + cnt[1] + cnt[2] + cnt[3]);
    // suffix sum over threads in descending bin order: scan with reversed thread index
    int ex_a, ex_b, tot_a, tot_b;
    // thread t's position in descending order is (kTopkThreads-1-t); compute the exclusive
    // prefix over higher threads by scanning the reversed values
    __syncthreads();
    {
      // place values in reversed order through shared scratch
      __shared__ int rev[kTopkThreads];
      rev[kTopkThreads - 1 - tid] = mine;
      __syncthreads();
      const int rv = rev[tid];
      block_scan2(rv, 0, ex_a, ex_b, tot_a, tot_b, sh);
      __syncthreads();
      rev[kTopkThreads - 1 - tid] = ex_a;  // keys in bins of higher threads
      __syncthreads();
      ex_a = rev[tid];
      __syncthreads();
    }
    int above = ex_a;  // keys in bins above this thread's bins
#pragma unroll
    for (int q = per - 1; q >= 0; --q) {
      const int bin = tid * per + q;
      const int c = (int)cnt[q];
      if (above < krem && krem <= above + c) {
        sh->sel_prefix = (prefix << widths[pass]) | (uint32_t)bin;
        sh->sel_krem = krem - above;
      }
      above += c;
    }
    __syncthreads();
    prefix = sh->sel_prefix;
    krem = sh->sel_krem;
    __syncthreads();
  }
  const uint32_t T = prefix;  // the K-th largest key; take every key > T and krem keys == T

  // ---- compaction in position order
  const int chunk = (len + kTopkThreads - 1) / kTopkThreads;
  const int c0 = min(len, tid * chunk), c1 = min(len, c0 + chunk);
  int gt = 0, eq = 0;
  for (int i = c0; i < c1; ++i) {
    gt += keys[i] > T;
    eq += keys[i] == T;
  }
  int ex_gt, ex_eq, tot_gt, tot_eq;
  block_scan2(gt, eq, ex_gt, ex_eq, tot_gt, tot_eq, sh);
  if (tid == 0) { sh->cta_gt = tot_gt; sh->cta_eq = tot_eq; }
  cluster_sync();
  int off_gt = 0, off_eq = 0;
  for (int r = 0; r < (int)rank; ++r) {
    off_gt += (int)ld_cluster_u32(mapa_cluster(&sh->cta_gt, (uint32_t)r));
    off_eq += (int)ld_cluster_u32(mapa_cluster(&sh->cta_eq, (uint32_t)r));
  }
  int gt_before = off_gt + ex_gt, eq_before = off_eq + ex_eq;
  for (int i = c0; i < c1; ++i) {
    const uint32_t k = keys[i];
    if (k > T) {
      out[gt_before + min(eq_before, krem)] = s0 + i;
      ++gt_before;
    } else if (k == T) {
      if (eq_before < krem) out[gt_before + eq_before] = s0 + i;
      ++eq_before;
    }
  }
  pdl_launch_dependents();
  cluster_sync();  // no CTA leaves while a peer may still read its shared memory
}


// ---------------------------------------------------------------------------------------------
// Rows of at most kRowKeys positions: one CTA of 1024 threads holds R rows, a group of 1024 / R
// threads per row, each thread holding 16 consecutive keys in registers (its share is
// contiguous, so thread order is position order).  Two rows per CTA when rows have at most 8192
// positions: the same threads per row, half the SMs (the attention grid launched behind this
// one gets them).  Each group synchronises on its own named barrier.
constexpr int kRowThreads = 1024;
constexpr int kRowPer = 16;
constexpr int kRowKeys = kRowThreads * kRowPer;

struct RowShared {
  uint32_t hist[2][kBins];          // alternate passes use alternate histograms
  int wtot[32];                     // per-warp totals of the bin scan
  int warp_a[32];
  int warp_b[32];
  uint32_t sel_prefix;
  int sel_krem;
};

template <int R>
__device__ __forceinline__ void group_sync(int g) {
  if (R == 1) {
    __syncthreads();
  } else {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "n"(kRowThreads / R) : "memory");
  }
}

// Exclusive prefix sums of (a, b) over the group's threads in thread order, and their totals.
template <int R>
__device__ __forceinline__ void row_scan2(int a, int b, int& ea, int& eb, int& ta, int& tb, RowShared* sh, int g,
                                          int gt) {
  constexpr int kWarps = kRowThreads / R / 32;
  const int lane = gt & 31, warp = gt >> 5;
  int ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int va = __shfl_up_sync(0xffffffffu, ia, o), vb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) { ia += va; ib += vb; }
  }
  if (lane == 31) { sh->warp_a[warp] = ia; sh->warp_b[warp] = ib; }
  group_sync<R>(g);
  if (warp == 0) {
    const int xa = lane < kWarps ? sh->warp_a[lane] : 0, xb = lane < kWarps ? sh->warp_b[lane] : 0;
    int sa = xa, sb_ = xb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int va = __shfl_up_sync(0xffffffffu, sa, o), vb = __shfl_up_sync(0xffffffffu, sb_, o);
      if (lane >= o) { sa += va; sb_ += vb; }
    }
    if (lane < kWarps) {
      sh->warp_a[lane] = sa - xa;   // exclusive warp offsets
      sh->warp_b[lane] = sb_ - xb;
    }
    if (lane == 31) { sh->sel_prefix = (uint32_t)sa; sh->sel_krem = sb_; }   // totals (scratch)
  }
  group_sync<R>(g);
  ea = sh->warp_a[warp] + ia - a;
  eb = sh->warp_b[warp] + ib - b;
  ta = (int)sh->sel_prefix;
  tb = sh->sel_krem;
  group_sync<R>(g);
}

template <int R>
__global__ void __launch_bounds__(kRowThreads, 1) topk_row_kernel(const TopkKernelParams p) {
  constexpr int kGT = kRowThreads / R;     // threads per row
  constexpr int kWarps = kGT / 32;
  constexpr int kBpt = kBins / kGT;        // histogram bins per thread in the bin scan
  __shared__ RowShared shm[R];
  const int g = threadIdx.x / kGT, gt = threadIdx.x - g * kGT;
  RowShared* sh = &shm[g];
  const long long row = (long long)blockIdx.x * R + g;
  const long long nrows = (long long)p.B * p.J;

  pdl_wait_primary();  // scores come from the previous kernel on the stream
  // the next kernel (attention) may be scheduled now: it only reads our output after its own
  // griddepcontrol.wait, which waits for this whole grid to finish
  pdl_launch_dependents();
  if (row >= nrows) return;   // a whole group (the grid's last CTA when the rows are odd)

  const int b = (int)(row / p.J), j = (int)(row - (long long)b * p.J);
  int32_t* out = p.topk + row * p.K;
  bool bad = false;
  const int pos = query_position(p.seq_lens, p.q_pos, p.J, b, j, p.Lpad, &bad);
  if (bad && gt == 0) report(p.status, SIA_DEV_BAD_POSITION);
  const int n = pos + 1;
  if (n <= p.K) {
    for (int i = gt; i < p.K; i += kGT) out[i] = i < n ? i : -1;
    return;
  }
  // this thread's keys: positions [gt*16, gt*16+16) of the visible range
  const int base = gt * kRowPer;
  uint32_t key[kRowPer];
  const float* src = p.scores + row * p.Lpad + base;
  if (base + kRowPer <= n) {
#pragma unroll
    for (int q = 0; q < kRowPer / 4; ++q) {
      const float4 v = reinterpret_cast<const float4*>(src)[q];
      key[4 * q] = order_key(v.x);
      key[4 * q + 1] = order_key(v.y);
      key[4 * q + 2] = order_key(v.z);
      key[4 * q + 3] = order_key(v.w);
    }
  } else {
#pragma unroll
    for (int i = 0; i < kRowPer; ++i) key[i] = base + i < n ? order_key(src[i]) : 0u;
  }
  const int nmine = max(0, min(kRowPer, n - base));

  uint32_t prefix = 0;
  int krem = p.K;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int i = gt; i < kBins; i += kGT) sh->hist[0][i] = 0;
  group_sync<R>(g);
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    uint32_t* hist = sh->hist[pass & 1];
    // the other histogram is cleared for the next pass (nobody reads it in this one)
    for (int i = gt; i < kBins; i += kGT) sh->hist[(pass + 1) & 1][i] = 0;
    const int sh_ = shifts[pass], hi_shift = sh_ + widths[pass];
    const uint32_t dmask = (1u << widths[pass]) - 1u;
#pragma unroll
    for (int i = 0; i < kRowPer; ++i)
      if (i < nmine && (pass == 0 || (key[i] >> hi_shift) == prefix)) atomicAdd(&hist[(key[i] >> sh_) & dmask], 1u);
    group_sync<R>(g);
    // thread gt owns kBpt consecutive bins counted from the top; "above" = keys in higher bins,
    // by a warp scan plus the totals of the warps before (each warp scans those itself)
    const int lane = gt & 31, wid = gt >> 5;
    const int lo_bin = kBins - kBpt * (gt + 1);   // thread 0 owns the top bins
    int cnt[kBpt];
    int mine = 0;
#pragma unroll
    for (int k = 0; k < kBpt; ++k) {
      cnt[k] = (int)hist[lo_bin + kBpt - 1 - k];   // cnt[0] is this thread's highest bin
      mine += cnt[k];
    }
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) sh->wtot[wid] = incl;
    group_sync<R>(g);
    int before;
    {
      const int wt = lane < kWarps ? sh->wtot[lane] : 0;
      int sc = wt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, sc, o);
        if (lane >= o) sc += v;
      }
      before = __shfl_sync(0xffffffffu, sc - wt, wid);
    }
    int ex = before + incl - mine;   // keys in bins above this thread's
#pragma unroll
    for (int k = 0; k < kBpt; ++k) {
      if (ex < krem && krem <= ex + cnt[k]) {
        sh->sel_prefix = (prefix << widths[pass]) | (uint32_t)(lo_bin + kBpt - 1 - k);
        sh->sel_krem = krem - ex;
      }
      ex += cnt[k];
    }
    group_sync<R>(g);
    prefix = sh->sel_prefix;
    krem = sh->sel_krem;
  }
  const uint32_t T = prefix;

  int gtc = 0, eqc = 0;
#pragma unroll
  for (int i = 0; i < kRowPer; ++i) {
    gtc += (i < nmine && key[i] > T);
    eqc += (i < nmine && key[i] == T);
  }
  int ex_gt, ex_eq, tot_gt, tot_eq;
  row_scan2<R>(gtc, eqc, ex_gt, ex_eq, tot_gt, tot_eq, sh, g, gt);
  int gt_before = ex_gt, eq_before = ex_eq;
#pragma unroll
  for (int i = 0; i < kRowPer; ++i) {
    if (i >= nmine) break;
    if (key[i] > T) {
      out[gt_before + min(eq_before, krem)] = base + i;
      ++gt_before;
    } else if (key[i] == T) {
      if (eq_before < krem) out[gt_before + eq_before] = base + i;
      ++eq_before;
    }
  }
}

}  // namespace

long long topk_grid_ctas(const TopkKernelParams& p) {
  const long long rows = (long long)p.B * p.J;
  if (p.Lpad <= kRowKeys) return p.Lpad <= kRowKeys / 2 ? (rows + 3) / 4 * 2 : rows;
  return rows * p.cluster;
}

cudaError_t launch_topk(const TopkKernelParams& p, bool pdl, cudaStream_t stream) {
  if (p.Lpad <= kRowKeys) {
    const long long rows = (long long)p.B * p.J;
    const bool two = p.Lpad <= kRowKeys / 2;   // two rows per CTA
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    // two rows per CTA and CTA pairs launched as 2-CTA clusters: a cluster sits on an SM pair,
    // so the grid blocks as few SM pairs as possible for the 2-CTA clusters of the attention
    // grid launched behind it (a lone CTA on an SM pair leaves its neighbour unusable to them)
    cfg.gridDim = dim3((unsigned)(two ? (rows + 3) / 4 * 2 : rows), 1, 1);
    cfg.blockDim = dim3(kRowThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    int na = 0;
    if (pdl) {
      attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[na].val.programmaticStreamSerializationAllowed = 1;
      ++na;
    }
    if (two) {
      attr[na].id = cudaLaunchAttributeClusterDimension;
      attr[na].val.clusterDim.x = 2;
      attr[na].val.clusterDim.y = 1;
      attr[na].val.clusterDim.z = 1;
      ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return two ? cudaLaunchKernelEx(&cfg, topk_row_kernel<2>, p) : cudaLaunchKernelEx(&cfg, topk_row_kernel<1>, p);
  }
  const size_t smem = sizeof(TopkShared) + (size_t)p.slice * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  if (p.cluster > 8) {
    e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.gridDim = dim3((unsigned)((long long)p.B * p.J * p.cluster), 1, 1);
  cfg.blockDim = dim3(kTopkThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  int na = 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = p.cluster;
  attr[na].val.clusterDim.y = 1;
  attr[na].val.clusterDim.z = 1;
  ++na;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, topk_kernel, p);
}

}  // namespace sia
