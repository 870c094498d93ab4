// sia_api.cu -- the C ABI of libsia (declared in include/sia.h): host-side argument checks,
// workspace layout, TMA descriptor set-up and the launch sequence of each entry point.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "sia.h"
#include "sia_internal.h"

namespace sia {
namespace {

thread_local char g_last_error[512] = "";

sia_status fail(sia_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
  return s;
}

std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};

sia_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SIA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

// ---------------------------------------------------------------- device facts
int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static int cached[64] = {0};
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

// CTA pairs of the attention grid that run at once on the current device: half the SMs, or
// fewer when the GPCs' SM counts leave some SMs that no 2-CTA cluster can use.  A grid with
// more pairs than this would run the extra ones as a second wave.
int attend_pairs(int dl, int dr, bool kv8) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  static std::atomic<int> cached[64][2];   // + 1, so that 0 means "not looked up yet"
  const int half = std::max(1, sm_count() / 2);
  const bool small = dl != 512;
  if (dev < 0 || dev >= 64 || small) {
    const int n = attend_max_clusters(dl, dr, kv8);
    return n > 0 ? std::min(half, n) : half;
  }
  const int c = cached[dev][kv8 ? 1 : 0].load(std::memory_order_relaxed);
  if (c > 0) return c - 1;
  const int n = attend_max_clusters(dl, dr, kv8);
  const int pairs = n > 0 ? std::min(half, n) : half;
  cached[dev][kv8 ? 1 : 0].store(pairs + 1, std::memory_order_relaxed);
  return pairs;
}

int max_smem_optin() {
  int dev = 0, v = 232448;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  return v;
}

// ---------------------------------------------------------------- TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

CUtensorMapSwizzle swizzle_for(int row_bytes) {
  return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : (row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

// 2-D map over a row-major [rows, cols] matrix with a [box_rows, box_cols] box.
sia_status make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
                       uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
                       int row_bytes_in_smem, CUtensorMapL2promotion l2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(SIA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (uint64_t)elem_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle_for(row_bytes_in_smem), l2, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SIA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return SIA_OK;
}

// 3-D map over a [d2, d1, d0] array (d0 innermost) with a [b2, b1, b0] box.
sia_status make_map_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t d0,
                       uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1, uint32_t b2, int row_bytes_in_smem,
                       CUtensorMapL2promotion l2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(SIA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * (uint64_t)elem_bytes, d0 * d1 * (uint64_t)elem_bytes};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle_for(row_bytes_in_smem), l2, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SIA_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed (%d)", (int)r);
  return SIA_OK;
}

// ---------------------------------------------------------------- stage 1 plan
struct IndexPlan {
  IndexKernelParams kp;
  TopkKernelParams tp;
  CUtensorMap kmap;
  CUtensorMap qmap;   // q as [B*J queries, H heads, D]: one box = one query sub-block's K block
  size_t ws_scores;   // workspace bytes for the scores (0 when scores_out is given)
  int grid;
};

sia_status check_index(const sia_index_args* a, bool with_topk) {
  if (!a) return fail(SIA_ERR_INVALID_ARGUMENT, "index args are NULL");
  if (a->batch < 1 || a->n_q < 1 || (with_topk && a->top_k < 1) || a->max_pages_per_seq < 1 || a->num_pages < 1)
    return fail(SIA_ERR_INVALID_ARGUMENT, "batch, n_q, top_k, max_pages_per_seq and num_pages must be >= 1");
  if (!a->q || !a->w || !a->k_cache || !a->page_table || !a->seq_lens || (with_topk && !a->topk_out))
    return fail(SIA_ERR_INVALID_ARGUMENT, "q, w, k_cache, page_table, seq_lens and topk_out must be set");
  if (a->dtype != SIA_BF16 && a->dtype != SIA_FP8_E4M3 && a->dtype != SIA_MXFP8)
    return fail(SIA_ERR_UNSUPPORTED, "unknown dtype %d", (int)a->dtype);
  if (a->n_heads < 1 || a->n_heads > 64) return fail(SIA_ERR_UNSUPPORTED, "n_heads must be 1..64 (got %d)", a->n_heads);
  if (a->dtype == SIA_MXFP8) {
    if (!a->q_mx || !a->k_mx) return fail(SIA_ERR_INVALID_ARGUMENT, "MXFP8 needs q_mx and k_mx");
    if (a->q_scale || a->k_scale) return fail(SIA_ERR_INVALID_ARGUMENT, "MXFP8 takes no q_scale or k_scale");
    if (a->head_dim != 64 && a->head_dim != 128)
      return fail(SIA_ERR_UNSUPPORTED, "MXFP8 head_dim must be 64 or 128 (got %d)", a->head_dim);
  } else if (a->q_mx || a->k_mx) {
    return fail(SIA_ERR_INVALID_ARGUMENT, "q_mx and k_mx are only for SIA_MXFP8");
  }
  const int eb = a->dtype == SIA_BF16 ? 2 : 1;
  const int db = a->head_dim * eb;
  if (a->head_dim < 1 || (db != 64 && db != 128 && db != 256))
    return fail(SIA_ERR_UNSUPPORTED, "head_dim must make a 64-, 128- or 256-byte row (got %d)", a->head_dim);
  if (!pow2(a->page_size) || a->page_size < 8 || a->page_size > 4096)
    return fail(SIA_ERR_UNSUPPORTED, "page_size must be a power of two in [8, 4096] (got %d)", a->page_size);
  if (!aligned(a->q, 16) || !aligned(a->k_cache, 16) || !aligned(a->w, 4) || !aligned(a->topk_out, 4) ||
      (a->scores_out && !aligned(a->scores_out, 16)) || (a->k_scale && !aligned(a->k_scale, 16)) ||
      (a->k_mx && !aligned(a->k_mx, 16)))
    return fail(SIA_ERR_INVALID_ARGUMENT, "q, k_cache, k_scale and scores_out must be 16-byte aligned, other arrays 4-byte aligned");
  const long long lpad = (long long)a->max_pages_per_seq * a->page_size;
  if (lpad > (1ll << 30)) return fail(SIA_ERR_UNSUPPORTED, "max_pages_per_seq * page_size too large");
  if ((long long)a->num_pages * a->page_size > (1ll << 31) - 1)
    return fail(SIA_ERR_UNSUPPORTED, "num_pages * page_size must fit in int32");
  return SIA_OK;
}

sia_status plan_index(const sia_index_args* a, IndexPlan* pl, bool make_maps, bool with_topk = true) {
  sia_status st = check_index(a, with_topk);
  if (st != SIA_OK) return st;
  IndexKernelParams& k = pl->kp;
  memset(&k, 0, sizeof k);
  const int eb = a->dtype == SIA_BF16 ? 2 : 1;
  const bool mx = a->dtype == SIA_MXFP8;
  k.B = a->batch;
  k.J = a->n_q;
  k.H = a->n_heads;
  k.HP = (a->n_heads + 15) / 16 * 16;
  k.P = a->page_size;
  k.max_pages = a->max_pages_per_seq;
  k.num_pages = a->num_pages;
  k.Lpad = (long long)a->max_pages_per_seq * a->page_size;
  k.d_bytes = a->head_dim * eb;
  k.kbw = k.d_bytes >= 128 ? 128 : 64;
  k.n_kblocks = k.d_bytes / k.kbw;
  k.ksteps_per_block = k.kbw / 32;
  k.fp8 = a->dtype != SIA_BF16;
  k.mx = mx ? 1 : 0;
  k.n_groups = mx ? a->head_dim / 32 : 1;
  // queries sharing one A tile: up to 128 accumulator columns per MMA and two MMAs per tile
  // for a prefill chunk, so that two accumulator stages fit in TMEM (the MMA of the next tile
  // overlaps the epilogue of this one)
  // (MXFP8: one query per group; its per-scale-group accumulators take n_groups x the columns)
  k.nq_sub = mx ? 1 : std::max(1, std::min(a->n_q, 128 / k.HP));
  k.n_sub = (!mx && a->n_q > k.nq_sub) ? 2 : 1;
  k.qg = k.nq_sub * k.n_sub;
  k.n_cols = k.nq_sub * k.HP;
  k.acc_cols = k.n_cols * k.n_groups;
  k.groups_per_seq = (a->n_q + k.qg - 1) / k.qg;
  const int cols_per_stage = k.n_sub * k.acc_cols;
  k.acc_stages = (2 * cols_per_stage <= 512) ? 2 : 1;
  uint32_t cols = (uint32_t)(k.acc_stages * cols_per_stage);
  uint32_t alloc = 32;
  while (alloc < cols) alloc <<= 1;
  k.tmem_cols = alloc;
  k.box_rows = std::min(a->page_size, kIndexTileRows);
  // shared memory: K stages | Q | w | info | barriers
  k.k_kblock_bytes = (uint32_t)(kIndexTileRows * k.kbw);
  k.k_stage_bytes = k.k_kblock_bytes * k.n_kblocks;
  k.q_kblock_bytes = (uint32_t)(k.n_cols * k.kbw);
  k.q_sub_bytes = k.q_kblock_bytes * k.n_kblocks;
  const uint32_t q_bytes = k.q_sub_bytes * k.n_sub;
  const uint32_t w_bytes = (uint32_t)round_up((size_t)2 * k.qg * k.HP * 4, 16);  // double-buffered
  const uint32_t info_bytes = 256;
  const uint32_t bar_bytes = 256;
  // per stage: chunk mask + key scales (fp32 per row, or one E8M0 byte per group of each row)
  const uint32_t kinfo_bytes = (uint32_t)round_up(16 + (mx ? k.n_groups : 4) * kIndexTileRows, 16);
  const uint32_t qmx_bytes = mx ? (uint32_t)round_up((size_t)2 * k.HP * k.n_groups * 4, 16) : 0u;
  const uint32_t fixed = q_bytes + w_bytes + info_bytes + qmx_bytes + bar_bytes;
  const int limit = max_smem_optin();
  int stages = (int)((limit - (int)fixed) / (int)(k.k_stage_bytes + kinfo_bytes));
  stages = std::min(stages, 8);
  if (stages < 2) return fail(SIA_ERR_UNSUPPORTED, "indexer tile does not fit in shared memory");
  k.k_stages = stages;
  k.off_k = 0;
  k.off_q = k.k_stage_bytes * stages;
  k.off_w = k.off_q + q_bytes;
  k.off_info = k.off_w + w_bytes;
  k.off_kinfo = k.off_info + info_bytes;
  k.kinfo_bytes = kinfo_bytes;
  k.off_qmx = k.off_kinfo + kinfo_bytes * stages;
  k.off_bar = k.off_qmx + qmx_bytes;
  k.smem_bytes = k.off_bar + bar_bytes;
  k.q = static_cast<const uint8_t*>(a->q);
  k.q_scale = a->q_scale;
  k.w = a->w;
  k.k_scale = a->k_scale;
  k.q_mx = a->q_mx;
  k.k_mx = a->k_mx;
  k.page_table = a->page_table;
  k.seq_lens = a->seq_lens;
  k.q_pos = a->q_pos;
  k.scores = a->scores_out;
  pl->ws_scores = a->scores_out ? 0 : round_up((size_t)a->batch * a->n_q * (size_t)k.Lpad * 4, 256);
  pl->grid = sm_count();

  TopkKernelParams& t = pl->tp;
  memset(&t, 0, sizeof t);
  t.B = a->batch;
  t.J = a->n_q;
  t.K = a->top_k;
  t.Lpad = k.Lpad;
  int cs = 1;
  while ((k.Lpad + cs - 1) / cs > kTopkSliceMax) cs <<= 1;
  if (with_topk && cs > 16)
    return fail(SIA_ERR_UNSUPPORTED, "context too long for the Top-K kernel (max %d)", 16 * kTopkSliceMax);
  const long long rows = (long long)a->batch * a->n_q;
  // rows of up to 16384 positions take one CTA each (no cluster); longer rows split across a
  // cluster, widened while that still leaves SMs idle
  if (cs > 1)
    while (cs < 8 && rows * cs * 2 <= 2ll * pl->grid) cs <<= 1;
  t.cluster = cs;
  t.slice = (int)round_up((size_t)((k.Lpad + cs - 1) / cs), 32);
  if (with_topk && rows * cs > 0x7fffffffll) return fail(SIA_ERR_UNSUPPORTED, "too many query rows");
  t.seq_lens = a->seq_lens;
  t.q_pos = a->q_pos;
  t.topk = a->topk_out;

  if (make_maps) {
    st = make_map_2d(&pl->kmap, a->k_cache, k.fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                     eb, (uint64_t)a->num_pages * a->page_size, (uint64_t)a->head_dim, (uint32_t)k.box_rows,
                     (uint32_t)(k.kbw / eb), k.kbw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
    if (st != SIA_OK) return st;
    st = make_map_3d(&pl->qmap, a->q, k.fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, eb,
                     (uint64_t)a->head_dim, (uint64_t)a->n_heads, (uint64_t)a->batch * a->n_q,
                     (uint32_t)(k.kbw / eb), (uint32_t)k.HP, (uint32_t)k.nq_sub, k.kbw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
    if (st != SIA_OK) return st;
  }
  return SIA_OK;
}

sia_status run_index(IndexPlan* pl, void* ws, size_t ws_bytes, int32_t* dev_status, cudaStream_t stream, bool pdl_first) {
  if (pl->ws_scores) {
    if (!ws) return fail(SIA_ERR_WORKSPACE, "a workspace of %zu bytes is needed", pl->ws_scores);
    if (ws_bytes < pl->ws_scores) return fail(SIA_ERR_WORKSPACE, "workspace too small: %zu < %zu", ws_bytes, pl->ws_scores);
    if (!aligned(ws, 256)) return fail(SIA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    pl->kp.scores = static_cast<float*>(ws);
  }
  pl->kp.status = dev_status;
  pl->kp.wait_ns = wait_limit_ns();
  pl->tp.scores = pl->kp.scores;
  pl->tp.status = dev_status;
  cudaError_t e = launch_index_score(pl->kp, pl->kmap, pl->qmap, pl->grid, pdl_first, stream);
  if (e != cudaSuccess) return cuda_fail(e, "index scoring launch");
  e = launch_topk(pl->tp, true, stream);
  if (e != cudaSuccess) return cuda_fail(e, "top-k launch");
  return SIA_OK;
}

// ---------------------------------------------------------------- stage 2 plan
struct AttendPlan {
  AttnKernelParams ap;
  CombineKernelParams cp;
  CUtensorMap q_rope;   // the query rows' rope slices (the only TMA load of the attention)
  size_t ws_part;
  long long records;  // partial-result records in the workspace (two per pair)
  bool merge;         // some query straddles a pair boundary: launch the merge
  int n_clusters;
};

sia_status check_attend(const sia_attend_args* a) {
  if (!a) return fail(SIA_ERR_INVALID_ARGUMENT, "attend args are NULL");
  if (a->batch < 1 || a->n_q < 1 || a->top_k < 1 || a->max_pages_per_seq < 1 || a->num_pages < 1 || a->page_size < 1)
    return fail(SIA_ERR_INVALID_ARGUMENT, "batch, n_q, top_k, page_size, max_pages_per_seq and num_pages must be >= 1");
  if (!a->q || !a->kv_cache || !a->page_table || !a->seq_lens || !a->topk || !a->out)
    return fail(SIA_ERR_INVALID_ARGUMENT, "q, kv_cache, page_table, seq_lens, topk and out must be set");
  if (!((a->d_latent == 512 && a->d_rope == 64) || (a->d_latent == 64 && a->d_rope == 16)))
    return fail(SIA_ERR_UNSUPPORTED, "(d_latent, d_rope) must be (512, 64) or (64, 16) (got %d, %d)", a->d_latent, a->d_rope);
  if (a->n_heads < 1 || a->n_heads > 128) return fail(SIA_ERR_UNSUPPORTED, "n_heads must be 1..128 (got %d)", a->n_heads);
  if (a->top_k > kAttnMaxSplitRows)
    return fail(SIA_ERR_UNSUPPORTED, "top_k must be <= %d (got %d)", kAttnMaxSplitRows, a->top_k);
  if (!std::isfinite(a->softmax_scale)) return fail(SIA_ERR_INVALID_ARGUMENT, "softmax_scale must be finite");
  if (!aligned(a->q, 16) || !aligned(a->kv_cache, 16) || !aligned(a->out, 16) || !aligned(a->topk, 4) ||
      (a->lse && !aligned(a->lse, 4)) || (a->kv_scale && !aligned(a->kv_scale, 4)))
    return fail(SIA_ERR_INVALID_ARGUMENT, "q, kv_cache and out must be 16-byte aligned");
  if ((long long)a->num_pages * a->page_size > (1ll << 31) - 1)
    return fail(SIA_ERR_UNSUPPORTED, "num_pages * page_size must fit in int32");
  if ((long long)a->batch * a->n_q * a->n_heads > (1ll << 31) - 1)
    return fail(SIA_ERR_UNSUPPORTED, "batch * n_q * n_heads must fit in int32");
  return SIA_OK;
}

// busy_sms: SMs that the preceding grid on the stream holds while this one is launched (the
// Top-K grid in the fused call); the pairs that can only start once it leaves get less work.
sia_status plan_attend(const sia_attend_args* a, AttendPlan* pl, bool make_maps, int busy_sms = 0) {
  sia_status st = check_attend(a);
  if (st != SIA_OK) return st;
  AttnKernelParams& k = pl->ap;
  memset(&k, 0, sizeof k);
  k.B = a->batch;
  k.J = a->n_q;
  k.H = a->n_heads;
  k.DL = a->d_latent;
  k.DR = a->d_rope;
  k.P = a->page_size;
  k.max_pages = a->max_pages_per_seq;
  k.num_pages = a->num_pages;
  k.K = a->top_k;
  k.scale_log2 = a->softmax_scale * 1.4426950408889634f;
  const long long bj = (long long)a->batch * a->n_q;
  const int pairs = attend_pairs(a->d_latent, a->d_rope, a->kv_scale != nullptr);
  // the flat (query, 64-row tile) list split evenly over the CTA pairs (see attn_next_unit)
  const long long TQ = (a->top_k + kAttnTileRows - 1) / kAttnTileRows;
  const long long G = bj * TQ;
  if (G > 0x7fffffffll) return fail(SIA_ERR_UNSUPPORTED, "batch * n_q * ceil(top_k / 64) must fit in int32");
  // With at most as many queries as pairs, every query gets the same number s of pairs and the
  // even split then puts each pair inside one query (pair c's range starts at c TQ / s): a pair
  // that moves on to a second query pays that query's start (its query rows, its first gathers)
  // and the first one's output on its critical path, which costs more than the few tiles an
  // uneven count saves.  With more queries than pairs, the flat list is split evenly.
  const bool per_query = bj <= pairs;
  const int C = per_query ? (int)(std::min<long long>(pairs / bj, TQ) * bj)
                          : (int)std::min<long long>(std::min(pairs, kAttnMaxPairs), G);
  k.tiles_per_q = (int)TQ;
  k.split.G = G;
  k.split.C = C;
  k.split.n_early = C;
  k.split.w_early = 1;
  k.split.w_late = 1;
  if (busy_sms > 0 && !per_query) {
    // the late pairs start about when the preceding grid ends, a few microseconds into a stage
    // of some tens: 7/8 of the work of an early pair
    k.split.n_early = std::max(0, std::min(C, (sm_count() - busy_sms) / 2));
    k.split.w_early = 8;
    k.split.w_late = 7;
  }
  // pieces (and their merge) only when some pair boundary falls inside a query; the workspace
  // holds the two records of every pair whenever there is more than one pair, so that its size
  // does not depend on how the pairs are weighted
  const long long records = C > 1 ? 2ll * C : 0;
  pl->merge = false;
  for (int c = 1; c < C; ++c)
    if (attn_pair_start(k.split, c) % TQ != 0) {
      pl->merge = true;
      break;
    }
  k.q = a->q;
  k.kv = a->kv_cache;
  k.kv_scale = a->kv_scale;
  k.kv_fp8 = a->kv_scale ? 1 : 0;
  k.nblk = (a->d_latent + a->d_rope + 127) / 128;
  k.page_table = a->page_table;
  k.seq_lens = a->seq_lens;
  k.topk = a->topk;
  k.out = static_cast<uint16_t*>(a->out);
  k.lse = a->lse;
  pl->n_clusters = C;
  pl->records = records;
  pl->ws_part = 0;
  if (records > 0) {
    const size_t o = round_up((size_t)records * a->n_heads * a->d_latent * 4, 256);
    const size_t l = round_up((size_t)records * 2 * a->n_heads * 4, 256);
    pl->ws_part = o + l;
  }
  CombineKernelParams& c = pl->cp;
  c.BJ = (int)bj;
  c.H = a->n_heads;
  c.DL = a->d_latent;
  c.tiles_per_q = k.tiles_per_q;
  c.split = k.split;
  c.out = k.out;
  c.lse = a->lse;

  if (make_maps) {
    const int dc = a->d_latent + a->d_rope;
    const int rope_kbw = a->d_latent == 512 ? 64 : 32;
    const uint64_t q_rows = (uint64_t)bj * a->n_heads;
    st = make_map_2d(&pl->q_rope, a->q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q_rows, dc, 128, rope_kbw / 2, rope_kbw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
    if (st != SIA_OK) return st;
  }
  return SIA_OK;
}

sia_status run_attend(AttendPlan* pl, void* ws, size_t ws_bytes, int32_t* dev_status, cudaStream_t stream, bool pdl_first) {
  if (pl->ws_part) {
    if (!ws) return fail(SIA_ERR_WORKSPACE, "a workspace of %zu bytes is needed", pl->ws_part);
    if (ws_bytes < pl->ws_part) return fail(SIA_ERR_WORKSPACE, "workspace too small: %zu < %zu", ws_bytes, pl->ws_part);
    if (!aligned(ws, 256)) return fail(SIA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    float* o = static_cast<float*>(ws);
    const size_t ob = round_up((size_t)pl->records * pl->ap.H * pl->ap.DL * 4, 256);
    pl->ap.part_o = o;
    pl->ap.part_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + ob);
    pl->cp.part_o = pl->ap.part_o;
    pl->cp.part_lse = pl->ap.part_lse;
  }
  pl->ap.status = dev_status;
  pl->ap.wait_ns = wait_limit_ns();
  cudaError_t e = launch_sparse_attend(pl->ap, pl->q_rope, pl->n_clusters, pdl_first, stream);
  if (e != cudaSuccess) return cuda_fail(e, "sparse attention launch");
  if (pl->merge) {
    e = launch_combine(pl->cp, true, stream);
    if (e != cudaSuccess) return cuda_fail(e, "split combine launch");
  }
  return SIA_OK;
}

}  // namespace

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

sia_status set_last_error(sia_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
  return s;
}

}  // namespace sia

using namespace sia;

extern "C" {

size_t sia_index_workspace_size(const sia_index_args* a) {
  IndexPlan pl;
  if (!a || plan_index(a, &pl, false) != SIA_OK) return 0;
  return pl.ws_scores;
}

size_t sia_attend_workspace_size(const sia_attend_args* a) {
  AttendPlan pl;
  if (!a || plan_attend(a, &pl, false) != SIA_OK) return 0;
  return pl.ws_part;
}

size_t sia_workspace_size(const sia_index_args* ia, const sia_attend_args* aa) {
  return round_up(sia_index_workspace_size(ia), 256) + round_up(sia_attend_workspace_size(aa), 256);
}

sia_status sia_sparse_index_topk(const sia_index_args* a, void* workspace, size_t ws_bytes, int32_t* dev_status,
                                 void* stream) {
  g_last_error[0] = 0;
  IndexPlan pl;
  sia_status st = plan_index(a, &pl, true);
  if (st != SIA_OK) return st;
  return run_index(&pl, workspace, ws_bytes, dev_status, static_cast<cudaStream_t>(stream), true);
}

sia_status sia_index_scores(const sia_index_args* a, int32_t* dev_status, void* stream) {
  g_last_error[0] = 0;
  if (a && !a->scores_out) return fail(SIA_ERR_INVALID_ARGUMENT, "scores_out is required");
  IndexPlan pl;
  sia_status st = plan_index(a, &pl, true, false);
  if (st != SIA_OK) return st;
  pl.kp.scores = a->scores_out;
  pl.kp.status = dev_status;
  pl.kp.wait_ns = wait_limit_ns();
  cudaError_t e = launch_index_score(pl.kp, pl.kmap, pl.qmap, pl.grid, true, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "index scoring launch");
  return SIA_OK;
}

sia_status sia_sparse_mla_attend(const sia_attend_args* a, void* workspace, size_t ws_bytes, int32_t* dev_status,
                                 void* stream) {
  g_last_error[0] = 0;
  AttendPlan pl;
  sia_status st = plan_attend(a, &pl, true);
  if (st != SIA_OK) return st;
  return run_attend(&pl, workspace, ws_bytes, dev_status, static_cast<cudaStream_t>(stream), false);
}

sia_status sia_fused_decode(const sia_index_args* ia, const sia_attend_args* aa, void* workspace, size_t ws_bytes,
                            int32_t* dev_status, void* stream) {
  g_last_error[0] = 0;
  if (!ia || !aa) return fail(SIA_ERR_INVALID_ARGUMENT, "both argument sets are required");
  if (ia->batch != aa->batch || ia->n_q != aa->n_q || ia->page_size != aa->page_size ||
      ia->max_pages_per_seq != aa->max_pages_per_seq || ia->top_k != aa->top_k || ia->page_table != aa->page_table ||
      ia->seq_lens != aa->seq_lens || ia->topk_out != aa->topk)
    return fail(SIA_ERR_INVALID_ARGUMENT,
                "index and attention arguments must describe the same sequences and share the Top-K buffer");
  IndexPlan ip;
  AttendPlan ap;
  sia_status st = plan_index(ia, &ip, true);
  if (st != SIA_OK) return st;
  // the Top-K grid holds one SM per CTA while the attention grid is launched
  const long long topk_ctas = topk_grid_ctas(ip.tp);
  st = plan_attend(aa, &ap, true, (int)std::min<long long>(topk_ctas, sm_count()));
  if (st != SIA_OK) return st;
  const size_t need = round_up(ip.ws_scores, 256) + round_up(ap.ws_part, 256);
  if (need && (!workspace || ws_bytes < need || !aligned(workspace, 256)))
    return fail(SIA_ERR_WORKSPACE, "the fused call needs a 256-byte aligned workspace of %zu bytes", need);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = run_index(&ip, workspace, ip.ws_scores, dev_status, s, true);
  if (st != SIA_OK) return st;
  void* ws2 = ap.ws_part ? static_cast<uint8_t*>(workspace) + round_up(ip.ws_scores, 256) : nullptr;
  return run_attend(&ap, ws2, ap.ws_part, dev_status, s, true);
}

sia_status sia_cache_append(const sia_append_args* a, int32_t* dev_status, void* stream) {
  g_last_error[0] = 0;
  if (!a) return fail(SIA_ERR_INVALID_ARGUMENT, "append args are NULL");
  if (a->batch < 1 || a->n_q < 1 || a->page_size < 1 || a->max_pages_per_seq < 1 || a->num_pages < 1)
    return fail(SIA_ERR_INVALID_ARGUMENT, "batch, n_q, page_size, max_pages_per_seq and num_pages must be >= 1");
  if (!a->new_k || !a->new_kv || !a->page_table || !a->seq_lens || !a->k_cache || !a->kv_cache)
    return fail(SIA_ERR_INVALID_ARGUMENT, "new_k, new_kv, page_table, seq_lens, k_cache and kv_cache must be set");
  if (a->key_format != SIA_KEY_BF16 && a->key_format != SIA_KEY_FP8_POW2 && a->key_format != SIA_KEY_MXFP8)
    return fail(SIA_ERR_UNSUPPORTED, "unknown key format %d", (int)a->key_format);
  if (a->kv_format != SIA_KV_BF16 && a->kv_format != SIA_KV_FP8_BLOCK128)
    return fail(SIA_ERR_UNSUPPORTED, "unknown kv format %d", (int)a->kv_format);
  if (a->head_dim < 32 || a->head_dim > 256 || a->head_dim % 32)
    return fail(SIA_ERR_UNSUPPORTED, "head_dim must be a multiple of 32 in [32, 256] (got %d)", a->head_dim);
  if (a->d_kv < 16 || a->d_kv > 1024 || a->d_kv % 2)
    return fail(SIA_ERR_UNSUPPORTED, "d_kv must be even and in [16, 1024] (got %d)", a->d_kv);
  if ((a->key_format != SIA_KEY_BF16) != (a->k_scale != nullptr))
    return fail(SIA_ERR_INVALID_ARGUMENT, "k_scale must be set exactly when the key format is quantised");
  if ((a->kv_format != SIA_KV_BF16) != (a->kv_scale != nullptr))
    return fail(SIA_ERR_INVALID_ARGUMENT, "kv_scale must be set exactly when the kv format is FP8");
  if (!aligned(a->new_k, 2) || !aligned(a->new_kv, 2) || !aligned(a->k_cache, 2) || !aligned(a->kv_cache, 2) ||
      (a->k_scale && a->key_format == SIA_KEY_FP8_POW2 && !aligned(a->k_scale, 4)) ||
      (a->kv_scale && !aligned(a->kv_scale, 4)) || !aligned(a->page_table, 4) || !aligned(a->seq_lens, 4))
    return fail(SIA_ERR_INVALID_ARGUMENT, "misaligned pointer");
  if ((long long)a->num_pages * a->page_size > (1ll << 31) - 1)
    return fail(SIA_ERR_UNSUPPORTED, "num_pages * page_size must fit in int32");
  if ((long long)a->batch * a->n_q > 0x7fffffffll) return fail(SIA_ERR_UNSUPPORTED, "too many tokens");
  AppendKernelParams k;
  memset(&k, 0, sizeof k);
  k.B = a->batch;
  k.J = a->n_q;
  k.D = a->head_dim;
  k.DC = a->d_kv;
  k.P = a->page_size;
  k.max_pages = a->max_pages_per_seq;
  k.num_pages = a->num_pages;
  k.key_format = (int)a->key_format;
  k.kv_format = (int)a->kv_format;
  k.new_k = a->new_k;
  k.new_kv = a->new_kv;
  k.page_table = a->page_table;
  k.seq_lens = a->seq_lens;
  k.k_cache = a->k_cache;
  k.k_scale = a->k_scale;
  k.kv_cache = a->kv_cache;
  k.kv_scale = a->kv_scale;
  k.status = dev_status;
  cudaError_t e = launch_cache_append(k, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cache append launch");
  return SIA_OK;
}

const char* sia_status_string(sia_status s) {
  switch (s) {
    case SIA_OK: return "SIA_OK";
    case SIA_ERR_INVALID_ARGUMENT: return "SIA_ERR_INVALID_ARGUMENT";
    case SIA_ERR_UNSUPPORTED: return "SIA_ERR_UNSUPPORTED";
    case SIA_ERR_CUDA: return "SIA_ERR_CUDA";
    case SIA_ERR_WORKSPACE: return "SIA_ERR_WORKSPACE";
  }
  return "SIA_ERR_UNKNOWN";
}

const char* sia_last_error(void) { return g_last_error; }

uint64_t sia_set_wait_limit_ns(uint64_t ns) {
  return g_wait_limit_ns.exchange(ns ? ns : 2000000000ull);
}

int32_t sia_version(void) { return 100; }

}  // extern "C"
