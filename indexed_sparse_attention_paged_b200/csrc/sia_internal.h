// sia_internal.h -- launch parameters shared between the C-ABI layer (sia_api.cu) and the
// kernels of libsia.  Host and device code; no torch types.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "sia.h"

namespace sia {

// Rows (positions) per indexer tile: the M of every tcgen05 MMA of the indexer.
constexpr int kIndexTileRows = 128;
// Latent rows per attention tile, and the most Top-K entries one attention unit (a split of a
// query's list) may hold.
constexpr int kAttnTileRows = 64;
constexpr int kAttnMaxSplitRows = 2048;
// Most CTA pairs one attention launch uses (148 SMs / 2 on a B200; the merge kernel keeps the
// pairs' first tiles in shared memory).
constexpr int kAttnMaxPairs = 128;
// Largest Top-K slice one CTA keeps in shared memory (keys, 4 bytes each).
constexpr int kTopkSliceMax = 16384;
constexpr int kTopkThreads = 512;

// -------------------------------------------------------------------------- indexer scoring
struct IndexKernelParams {
  int B, J, H, HP;            // batch, queries per sequence, heads, heads padded to 16
  int P, max_pages, num_pages;
  long long Lpad;             // score row length = max_pages * P
  int d_bytes;                // bytes of one q / k row
  int kbw;                    // bytes per K block row (128 or 64)
  int n_kblocks;              // d_bytes / kbw
  int ksteps_per_block;       // kbw / 32
  int fp8;                    // e4m3 codes (per-token scales, or MXFP8 when mx)
  int mx;                     // MXFP8: one E8M0 scale per 32 elements of q and of each key
  int n_groups;               // MX scale groups per row (head_dim / 32)
  int nq_sub;                 // queries per accumulator sub-block
  int n_sub;                  // accumulator sub-blocks per A tile (1 or 2)
  int qg;                     // queries per group = nq_sub * n_sub
  int n_cols;                 // N of one MMA = nq_sub * HP
  int acc_cols;               // TMEM columns of one accumulator: n_cols, or n_groups * n_cols (MX)
  int groups_per_seq;         // ceil(J / qg)
  int acc_stages;             // accumulator stages in TMEM
  int k_stages;               // K-tile stages in shared memory
  int box_rows;               // rows per TMA box = min(P, 128)
  uint32_t tmem_cols;
  // shared-memory layout, byte offsets from the 1024-aligned base
  uint32_t off_k, k_stage_bytes, k_kblock_bytes;
  uint32_t off_q, q_sub_bytes, q_kblock_bytes;
  uint32_t off_w, off_info, off_kinfo, off_qmx, off_bar, smem_bytes;
  uint32_t kinfo_bytes;       // per K stage: chunk mask + the rows' key scales
  const uint8_t* q;
  const float* q_scale;
  const float* w;
  const float* k_scale;
  const uint8_t* q_mx;        // MX: E8M0 [B, J, H, n_groups]
  const uint8_t* k_mx;        // MX: E8M0 [num_pages * P, n_groups]
  const int32_t* page_table;
  const int32_t* seq_lens;
  const int32_t* q_pos;
  float* scores;
  int32_t* status;
  uint64_t wait_ns;           // limit of every bounded in-kernel wait
};

// -------------------------------------------------------------------------- Top-K
struct TopkKernelParams {
  int B, J, K;
  long long Lpad;
  int cluster;                // CTAs per query row
  int slice;                  // keys per CTA (multiple of 32, <= kTopkSliceMax)
  const float* scores;
  const int32_t* seq_lens;
  const int32_t* q_pos;
  int32_t* topk;
  int32_t* status;
};

// -------------------------------------------------------------------------- attention
// How the flat (query, 64-row tile) list is divided between the CTA pairs of an attention
// launch: pair c takes tiles [start(c), start(c + 1)) with start(c) = G W(c) / W(C), where the
// first n_early pairs weigh w_early and the others w_late.  In the fused call the pairs launched
// last can only become resident when the Top-K grid's CTAs leave their SMs, so they get less.
struct AttnSplit {
  long long G;                // total tiles
  int C;                      // pairs
  int n_early, w_early, w_late;
};

__host__ __device__ inline long long attn_weight_before(const AttnSplit& s, int c) {
  const int e = c < s.n_early ? c : s.n_early;
  return (long long)s.w_early * e + (long long)s.w_late * (c - e);
}

__host__ __device__ inline long long attn_pair_start(const AttnSplit& s, int c) {
  return s.G * attn_weight_before(s, c) / attn_weight_before(s, s.C);
}

struct AttnKernelParams {
  int B, J, H, DL, DR, P, max_pages, num_pages, K;
  float scale_log2;           // softmax_scale * log2(e)
  int tiles_per_q;            // ceil(K / kAttnTileRows) <= 32
  AttnSplit split;            // the pairs' ranges of the flat tile list
  const void* q;              // bf16 [B*J, H, DL + DR]
  const void* kv;             // bf16 [num_pages * P, DL + DR], or e4m3 codes when kv_fp8
  const float* kv_scale;      // kv_fp8: fp32 [num_pages * P, nblk], one per 128-element block
  int kv_fp8;
  int nblk;                   // ceil((DL + DR) / 128)
  const int32_t* page_table;
  const int32_t* seq_lens;
  const int32_t* topk;
  uint16_t* out;              // bf16 bits
  float* lse;
  float* part_o;              // [2 * n_pairs][H][DL] fp32, normalised pieces
  float* part_lse;            // [2 * n_pairs][2 (CTA of the pair)][H]
  int32_t* status;
  uint64_t wait_ns;           // limit of every bounded in-kernel wait
};

struct CombineKernelParams {
  int BJ, H, DL;
  int tiles_per_q;
  AttnSplit split;
  const float* part_o;
  const float* part_lse;
  uint16_t* out;
  float* lse;
};

// -------------------------------------------------------------------------- paged cache append
struct AppendKernelParams {
  int B, J, D, DC, P, max_pages, num_pages;
  int key_format;             // sia_key_format
  int kv_format;              // sia_kv_format
  const void* new_k;          // bf16 [B*J, D]
  const void* new_kv;         // bf16 [B*J, DC]
  const int32_t* page_table;
  const int32_t* seq_lens;
  void* k_cache;
  void* k_scale;
  void* kv_cache;
  float* kv_scale;
  int32_t* status;
};

// Launchers (each returns cudaSuccess or the launch error).  `pdl` asks for programmatic
// dependent launch on the previous kernel of the stream.
cudaError_t launch_index_score(const IndexKernelParams& p, const CUtensorMap& kmap, const CUtensorMap& qmap, int grid,
                               bool pdl, cudaStream_t stream);
// CTAs of the Top-K grid launch_topk starts for these parameters.
long long topk_grid_ctas(const TopkKernelParams& p);
cudaError_t launch_topk(const TopkKernelParams& p, bool pdl, cudaStream_t stream);
// q_rope: 2-D map over the query rows [B*J*H, DL+DR] whose box is one CTA's rope slice of 128 heads
cudaError_t launch_sparse_attend(const AttnKernelParams& p, const CUtensorMap& q_rope,
                                 int n_clusters, bool pdl, cudaStream_t stream);
cudaError_t launch_combine(const CombineKernelParams& p, bool pdl, cudaStream_t stream);
cudaError_t launch_cache_append(const AppendKernelParams& p, cudaStream_t stream);

// Shared memory the attention kernel needs for (d_latent, d_rope).
size_t attend_smem_bytes(int dl, int dr);
// 2-CTA clusters of the attention kernel the current device holds at once; 0 if unknown.
int attend_max_clusters(int dl, int dr, bool kv8);

// Limit of every bounded in-kernel wait, in nanoseconds (set by sia_set_wait_limit_ns).
uint64_t wait_limit_ns();

// Records the detail message that sia_last_error() returns on this host thread; returns s.
sia_status set_last_error(sia_status s, const char* fmt, ...);

}  // namespace sia
