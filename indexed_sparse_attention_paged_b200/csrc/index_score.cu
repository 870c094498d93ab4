// index_score.cu -- the indexer's scoring stage on the sm_100a tensor cores.
//
// Computes, for every query (b, j) and every causal position s <= p(b, j),
//     I[s] = q_scale[b,j] * k_scale[s] * sum_h w[b,j,h] * ReLU(q[b,j,h] . k[s])
// reading k[s] straight out of the paged index-K cache ("Rapid Adaptation and Inference
// Optimization: Key Engineering Practices for Day0 LLM Support", section IV.4.1; the score form
// is the spec's fixed reading of the "score, then weight and sum the heads" steps in "Day 0
// Inference Adaptation and Performance Optimization for Hybrid Sparse Attention LLMs", section
// "Operator Fusion and Multi-Stream Scheduling").  Prefill and decode share this one kernel, as
// the pages ask of the fused indexer.
//
// Design (B200): one tcgen05 MMA per (128-position tile, query sub-block):
//   A = K tile   [128 positions x D]   (TMA from the paged cache, K-major, swizzled; M = 128)
//   B = Q group  [nq_sub*HP rows x D]  (one 3-D TMA box per K block, K-major, swizzled;
//                                       N = queries x heads)
//   D = TMEM     [128 lanes x N fp32 columns], two accumulator stages
// so that in the epilogue each thread owns one position and reduces sum_h w*ReLU(d) over its
// own registers, without shuffles.  The grid is persistent (one CTA per SM); the flat list of
// (query group, tile) work is split between CTAs by a weight of tiles plus a per-group set-up
// cost, which balances ragged context lengths and the causal "light at the start, heavy at the
// end" prefill load.  The kernel is a programmatic dependent of the previous kernel on the
// stream: it touches no global memory before that grid has completed.
//
// Exactness: for integer-valued q, k, w (the tests' inputs) every product and every partial
// sum is an integer below 2^24, so the fp32 result equals the exact score whatever order the
// tensor core and the epilogue add in.
#include <cuda.h>
#include <cuda_runtime.h>

#include "sia_common.cuh"
#include "sia_internal.h"
#include "sia_ptx.cuh"

namespace sia {
namespace {

// Per K stage (p.kinfo_bytes): 16 bytes of chunk mask, then the tile rows' key scales (one fp32
// per row, or with MXFP8 keys one E8M0 byte per 32-element group of each row).

struct IndexBarriers {
  uint64_t k_full[8];
  uint64_t k_empty[8];
  uint64_t acc_full[2][2];
  uint64_t acc_empty[2][2];
  uint64_t q_full;    // every epilogue thread staged the group's w and positions
  uint64_t q_tma;     // the group's q boxes landed (TMA bytes only)
  uint64_t q_empty;
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  int start_item, start_tile, count;
};
// the host reserves 256 bytes for the barrier block (bar_bytes in the stage-1 plan)
static_assert(sizeof(IndexBarriers) <= 256, "barrier block outgrew its shared-memory slot");

struct GroupInfo {
  int b, g;         // sequence, query group
  int max_pos;      // largest visible position among the group's queries (-1: none)
  int n_tiles;
};

__device__ __forceinline__ GroupInfo group_info(const IndexKernelParams& p, int item) {
  GroupInfo gi;
  gi.b = item / p.groups_per_seq;
  gi.g = item - gi.b * p.groups_per_seq;
  int mp = -1;
  const int j0 = gi.g * p.qg;
  const int j1 = min(p.J, j0 + p.qg);
  if (p.q_pos == nullptr) {
    mp = query_position(p.seq_lens, nullptr, p.J, gi.b, j1 - 1, p.Lpad);
  } else {
    for (int j = j0; j < j1; ++j) mp = max(mp, query_position(p.seq_lens, p.q_pos, p.J, gi.b, j, p.Lpad));
  }
  gi.max_pos = mp;
  gi.n_tiles = mp < 0 ? 0 : mp / kIndexTileRows + 1;
  return gi;
}

// Work per (query group, tile) list entry, in tile units: a group also costs about two tiles of
// set-up (its q and w staged, the pipeline drained and refilled), which matters for the short
// groups at the start of a causal prefill chunk.
constexpr long long kGroupCost = 2;

// Warp 0 finds this CTA's share of the flat tile list: the weighted work (tiles + kGroupCost per
// group) is split evenly between CTAs; the share is returned as (first group, first tile, tile
// count).
__device__ void locate_start(const IndexKernelParams& p, IndexBarriers* sb) {
  const int lane = threadIdx.x & 31;
  const int items = p.B * p.groups_per_seq;
  long long total = 0;
  for (int base = 0; base < items; base += 32) {
    const int it = base + lane;
    const int nt = it < items ? group_info(p, it).n_tiles : 0;
    long long t = nt > 0 ? nt + kGroupCost : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    total += t;
  }
  // (item, tile) and tiles-before of a weighted position: inside a group the set-up comes first
  auto find = [&](long long pos, int& item_out, int& tile_out, long long& tiles_before) {
    long long wbefore = 0, tbefore = 0;
    item_out = items;
    tile_out = 0;
    tiles_before = 0;
    for (int base = 0; base < items; base += 32) {
      const int it = base + lane;
      const int nt = it < items ? group_info(p, it).n_tiles : 0;
      const long long w = nt > 0 ? nt + kGroupCost : 0;
      long long wi = w, ti = nt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long vw = __shfl_up_sync(0xffffffffu, wi, o);
        const long long vt = __shfl_up_sync(0xffffffffu, ti, o);
        if (lane >= o) { wi += vw; ti += vt; }
      }
      const long long wex = wbefore + wi - w, tex = tbefore + ti - nt;
      const bool here = w > 0 && pos >= wex && pos < wex + w;
      const unsigned m = __ballot_sync(0xffffffffu, here);
      if (m) {
        const int src = __ffs(m) - 1;
        item_out = __shfl_sync(0xffffffffu, it, src);
        const long long off = pos - __shfl_sync(0xffffffffu, wex, src);
        tile_out = (int)(off > kGroupCost ? off - kGroupCost : 0);
        tiles_before = __shfl_sync(0xffffffffu, tex, src) + tile_out;
        return;
      }
      wbefore += __shfl_sync(0xffffffffu, wi, 31);
      tbefore += __shfl_sync(0xffffffffu, ti, 31);
    }
    tiles_before = tbefore;   // past the end: every tile is before
  };
  const long long begin = total * blockIdx.x / gridDim.x;
  const long long end = total * (blockIdx.x + 1) / gridDim.x;
  int start_item, start_tile, end_item, end_tile;
  long long tb_begin, tb_end;
  find(begin, start_item, start_tile, tb_begin);
  find(end, end_item, end_tile, tb_end);
  if (lane == 0) {
    sb->start_item = start_item;
    sb->start_tile = start_tile;
    sb->count = (int)(tb_end - tb_begin);
  }
}

// KBW (64 or 128 bytes per K-block row), NKB (K blocks per row) and KIND (0 bf16, 1 FP8 E4M3,
// 2 MXFP8) are compile-time so that the MMA issue loop is fully unrolled with constant
// descriptors: with runtime trip counts each tcgen05.mma took about three times longer to issue.
//
// MXFP8 (one E8M0 scale per 32 elements of q and of each key, "Rapid Adaptation and Inference
// Optimization", tiered quantisation table, and "Day 0 Inference Adaptation ... for Hybrid
// Sparse Attention LLMs", section 5.1): one kind::f8f6f4 MMA step covers K = 32 elements, which
// is exactly one scale group, so every group's partial dot products go to an accumulator of their
// own, and the epilogue forms d = sum_g D_g * 2^(eq[h,g] + ek[s,g]) before the ReLU.  For
// integer-valued codes and moderate exponents every term and partial sum is exact in fp32.
template <int NSUB, int KBW, int NKB, int KIND>
__global__ void __launch_bounds__(64 + 128 * NSUB, 1)
    index_score_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                       const IndexKernelParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  IndexBarriers* sb = reinterpret_cast<IndexBarriers*>(smem + p.off_bar);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int kEpiThreads = 128 * NSUB;
  constexpr bool FP8 = KIND != 0;
  constexpr bool MX = KIND == 2;
  constexpr int kGroups = NKB * KBW / 32;   // MX scale groups per row (one MMA K step each)
  static_assert(!MX || NSUB == 1, "MXFP8 uses one query per group and one sub-block");

  if ((smem_u32(smem) & 1023u) != 0) {  // the swizzled layouts need a 1024-byte aligned base
    pdl_wait_primary();
    if (threadIdx.x == 0) report(p.status, SIA_DEV_INTERNAL);
    return;
  }
  // The next kernel on the stream may be scheduled as soon as every CTA of this grid runs: it
  // waits for this grid's completion itself, so only its launch and set-up overlap this grid.
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.k_stages; ++s) {
      mbar_init(&sb->k_full[s], 1);
      mbar_init(&sb->k_empty[s], 1 + 4 * NSUB);  // MMA commit + every epilogue warp
    }
    for (int a = 0; a < p.acc_stages; ++a)
      for (int s = 0; s < NSUB; ++s) {
        mbar_init(&sb->acc_full[a][s], 1);
        mbar_init(&sb->acc_empty[a][s], 128);
      }
    mbar_init(&sb->q_full, kEpiThreads);
    mbar_init(&sb->q_tma, 1);
    mbar_init(&sb->q_empty, 1);
    mbar_init(&sb->mma_done, 1);
    sb->abort = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&qmap);
  }
  // Launched as a programmatic dependent of the previous kernel on the stream: nothing in global
  // memory (inputs, workspace, status) is touched before that grid has completed.
  pdl_wait_primary();
  if (warp == 0) locate_start(p, sb);
  if (warp == 1) {
    tmem_alloc(&sb->tmem_base, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sb->tmem_base;
  volatile int* abort = &sb->abort;
  const WaitCtl wc{abort, p.status, p.wait_ns};
  const int start_item = sb->start_item;
  const int start_tile = sb->start_tile;
  const int my_count = sb->count;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    int it = 0;
    int item = start_item, t0 = start_tile, remaining = my_count;
    bool ok = true;
    const uint64_t stream_policy = l2_evict_first_policy();   // keys are read once per call
    while (remaining > 0 && ok) {
      const GroupInfo gi = group_info(p, item);
      const int t1 = min(gi.n_tiles, t0 + remaining);
      const int32_t* pt_row = p.page_table + (long long)gi.b * p.max_pages;
      int cached_base = -(1 << 30), cached_page = -1;  // nothing cached yet
      for (int t = t0; t < t1 && ok; ++t, ++it) {
        const int stage = it % p.k_stages;
        const uint32_t phase = (uint32_t)(it / p.k_stages) & 1u;
        int go = 1;
        if (lane == 0) go = mbar_wait(&sb->k_empty[stage], phase ^ 1u, wc);
        go = __shfl_sync(0xffffffffu, go, 0);
        if (!go) { ok = false; break; }
        uint8_t* kst = smem + p.off_k + stage * p.k_stage_bytes;
        const int chunks = kIndexTileRows / p.box_rows;   // 1..16 boxes of whole-page rows
        // lane c < chunks resolves chunk c's page id through the warp's window of 32 cached
        // page-table entries (registers only: one shuffle per lane)
        const int tile_pos0 = t * kIndexTileRows;
        const int lp_first = tile_pos0 / p.P;
        const int lp_last = (tile_pos0 + (chunks - 1) * p.box_rows) / p.P;
        if (lp_first < cached_base || lp_last >= cached_base + 32) {   // warp-uniform
          cached_base = lp_first;
          cached_page = (lp_first + lane < p.max_pages) ? pt_row[lp_first + lane] : -1;
        }
        const int my_pos = tile_pos0 + lane * p.box_rows;
        const int my_lp = lane < chunks ? my_pos / p.P : lp_first;
        const int my_page = __shfl_sync(0xffffffffu, cached_page, my_lp - cached_base);
        const bool in_range = lane < chunks && my_pos <= gi.max_pos;
        const bool page_ok = my_page >= 0 && my_page < p.num_pages;
        if (in_range && !page_ok) report(p.status, SIA_DEV_BAD_PAGE);
        const uint32_t valid_mask = __ballot_sync(0xffffffffu, in_range && page_ok);
        uint8_t* info = smem + p.off_kinfo + stage * p.kinfo_bytes;
        const uint32_t row_scale_bytes = MX ? (uint32_t)kGroups : 4u;
        const void* kscale_src = MX ? static_cast<const void*>(p.k_mx) : static_cast<const void*>(p.k_scale);
        const uint32_t scale_bytes = kscale_src ? (uint32_t)p.box_rows * row_scale_bytes : 0u;
        if (lane == 0) {
          // per-stage info read by the epilogue: which chunks hold real pages, and (FP8) the
          // per-token key scales of the tile, copied next to the K tile
          *reinterpret_cast<uint32_t*>(info) = valid_mask;
          const uint32_t bytes =
              (uint32_t)__popc(valid_mask) * (NKB * p.box_rows * KBW + scale_bytes);
          mbar_arrive_expect_tx(&sb->k_full[stage], bytes);
        }
        __syncwarp();
        // lane c issues chunk c's boxes: a TMA instruction blocks its issuing thread for a few
        // hundred cycles, so several issuing lanes move a tile's bytes sooner than one
        if (valid_mask >> lane & 1u) {
          const int y = my_page * p.P + (my_pos % p.P);
#pragma unroll
          for (int kb = 0; kb < NKB; ++kb)
            tma_load_2d_hint(kst + kb * p.k_kblock_bytes + lane * p.box_rows * KBW, &kmap,
                             &sb->k_full[stage], kb * KBW / (FP8 ? 1 : 2), y, stream_policy);
          if (kscale_src)
            bulk_load(info + 16 + lane * p.box_rows * row_scale_bytes,
                      static_cast<const uint8_t*>(kscale_src) + (long long)y * row_scale_bytes, scale_bytes,
                      &sb->k_full[stage]);
        }
        __syncwarp();
      }
      remaining -= (t1 - t0);
      ++item;
      t0 = 0;
    }
    // do not leave while loads into our shared memory may still be landing: the last k_stages
    // tiles issued (earlier ones were consumed before their stage was refilled) are drained
    // whether or not the CTA is aborting
    if (lane == 0 && it > 0) {
      const int first = it > p.k_stages ? it - p.k_stages : 0;
      for (int i = first; i < it; ++i)
        mbar_drain(&sb->k_full[i % p.k_stages], (uint32_t)(i / p.k_stages) & 1u, p.status);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = FP8 ? umma_idesc(0, 0, false, false, p.n_cols, 128)
                                 : umma_idesc(1, 1, false, false, p.n_cols, 128);
      constexpr uint32_t layout = umma_layout_type(KBW);
      constexpr uint32_t sbo = 8 * KBW;
      constexpr uint32_t a_kblock = kIndexTileRows * KBW;
      int it = 0, acc_it = 0, seg = 0;
      int item = start_item, t0 = start_tile, remaining = my_count;
      bool ok = true;
      while (remaining > 0 && ok) {
        const GroupInfo gi = group_info(p, item);
        const int t1 = min(gi.n_tiles, t0 + remaining);
        if (t1 > t0) {
          if (!mbar_wait(&sb->q_full, (uint32_t)seg & 1u, wc)) { ok = false; break; }
          if (!mbar_wait(&sb->q_tma, (uint32_t)seg & 1u, wc)) { ok = false; break; }
          tc_fence_after();
          for (int t = t0; t < t1; ++t, ++it, ++acc_it) {
            const int stage = it % p.k_stages;
            if (!mbar_wait(&sb->k_full[stage], (uint32_t)(it / p.k_stages) & 1u, wc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const int as = acc_it % p.acc_stages;
            const uint32_t aph = (uint32_t)(acc_it / p.acc_stages) & 1u;
            const uint32_t a_base = smem_u32(smem + p.off_k + stage * p.k_stage_bytes);
            for (int sub = 0; sub < NSUB; ++sub) {
              if (!mbar_wait(&sb->acc_empty[as][sub], aph ^ 1u, wc)) { ok = false; break; }
              tc_fence_after();
              const uint32_t d_tmem = tmem_base + (uint32_t)((as * NSUB + sub) * p.acc_cols);
              const uint32_t b_base = smem_u32(smem + p.off_q + sub * p.q_sub_bytes);
              const uint32_t q_kblock = p.q_kblock_bytes;
#pragma unroll
              for (int kb = 0; kb < NKB; ++kb)
#pragma unroll
                for (int ks = 0; ks < KBW / 32; ++ks) {
                  const uint64_t ad = umma_smem_desc(a_base + kb * a_kblock + ks * 32, 16, sbo, layout);
                  const uint64_t bd = umma_smem_desc(b_base + kb * q_kblock + ks * 32, 16, sbo, layout);
                  if (MX) umma_f8(d_tmem + (uint32_t)((kb * (KBW / 32) + ks) * p.n_cols), ad, bd, idesc, false);
                  else if (FP8) umma_f8(d_tmem, ad, bd, idesc, (kb | ks) != 0);
                  else umma_f16(d_tmem, ad, bd, idesc, (kb | ks) != 0);
                }
              umma_commit(&sb->acc_full[as][sub]);
            }
            if (!ok) break;
            umma_commit(&sb->k_empty[stage]);
          }
          umma_commit(&sb->q_empty);
          ++seg;
        }
        remaining -= (t1 - t0);
        ++item;
        t0 = 0;
      }
      umma_commit(&sb->mma_done);
      mbar_drain(&sb->mma_done, 0, p.status);   // every MMA (reading shared memory, writing TMEM) done
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue warps
    const int et = threadIdx.x - 64;          // 0 .. kEpiThreads-1
    const int sub = (warp - 2) >> 2;          // accumulator sub-block of this warp
    const int quad = warp & 3;                // TMEM lane quarter this warp may access
    const int row = quad * 32 + lane;         // position inside the tile
    // w and per-query info are double-buffered by segment parity: a warp may start staging
    // the next group while another still reads the current one (it cannot get two groups ahead,
    // since every epilogue thread must stage a group before its MMAs can run)
    const int w_words = p.qg * p.HP;
    int acc_it = 0, seg = 0, q_issued = 0;
    int item = start_item, t0 = start_tile, remaining = my_count;
    bool ok = true;
    while (remaining > 0 && ok) {
      const GroupInfo gi = group_info(p, item);
      const int t1 = min(gi.n_tiles, t0 + remaining);
      if (t1 > t0) {
        // -- stage this group's q (swizzled, zero-padded) and head weights
        if (seg > 0 && !mbar_wait_warp(&sb->q_empty, (uint32_t)(seg - 1) & 1u, wc)) { ok = false; break; }
        float* w_s = reinterpret_cast<float*>(smem + p.off_w) + (seg & 1) * w_words;
        int* info_pos = reinterpret_cast<int*>(smem + p.off_info) + (seg & 1) * 16;
        float* info_qs = reinterpret_cast<float*>(smem + p.off_info + 128) + (seg & 1) * 16;
        // MXFP8: the query's group scales 2^(e - 127) as fp32, [head][group]
        float* qmx_s = reinterpret_cast<float*>(smem + p.off_qmx) + (seg & 1) * (p.HP * kGroups);
        if (et == 0) {
          // q of the group: one 3-D TMA box (nq_sub queries x HP heads x one K block, heads
          // past H and queries past the batch zero-filled) per (sub-block, K block)
          mbar_arrive_expect_tx(&sb->q_tma, (uint32_t)(NSUB * NKB) * p.q_kblock_bytes);
#pragma unroll
          for (int sb_ = 0; sb_ < NSUB; ++sb_)
#pragma unroll
            for (int kb = 0; kb < NKB; ++kb)
              tma_load_3d(smem + p.off_q + sb_ * p.q_sub_bytes + kb * p.q_kblock_bytes, &qmap, &sb->q_tma,
                          kb * KBW / (FP8 ? 1 : 2), 0, gi.b * p.J + gi.g * p.qg + sb_ * p.nq_sub);
          ++q_issued;
        }
        for (int i = et; i < p.qg * p.HP; i += kEpiThreads) {
          const int ql = i / p.HP, h = i - ql * p.HP;
          const int j = gi.g * p.qg + ql;
          w_s[i] = (j < p.J && h < p.H) ? p.w[((long long)gi.b * p.J + j) * p.H + h] : 0.0f;
        }
        if (MX) {
          const int j = gi.g;   // one query per group
          for (int i = et; i < p.HP * kGroups; i += kEpiThreads) {
            const int h = i / kGroups;
            const uint32_t code = h < p.H ? p.q_mx[(((long long)gi.b * p.J + j) * p.H + h) * kGroups + i % kGroups] : 127u;
            // E8M0: 2^(code - 127); code 0 is 2^-127 (a subnormal fp32), 0xFF NaN
            qmx_s[i] = code == 0xFFu ? __int_as_float(0x7fc00000) : ldexpf(1.0f, (int)code - 127);
          }
        }
        if (et < p.qg) {
          const int j = gi.g * p.qg + et;
          info_pos[et] = j < p.J ? query_position(p.seq_lens, p.q_pos, p.J, gi.b, j, p.Lpad) : -1;
          info_qs[et] = (j < p.J && p.q_scale) ? p.q_scale[(long long)gi.b * p.J + j] : 1.0f;
        }
        mbar_arrive(&sb->q_full);
        // every epilogue thread has staged its share (w_s / info are visible after this)
        if (!mbar_wait_warp(&sb->q_full, (uint32_t)seg & 1u, wc)) { ok = false; break; }
        const long long out_row0 = (long long)gi.b * p.J;
        for (int t = t0; t < t1; ++t, ++acc_it) {
          const int as = acc_it % p.acc_stages;
          const uint32_t aph = (uint32_t)(acc_it / p.acc_stages) & 1u;
          const int kstage = acc_it % p.k_stages;
          const int s = t * kIndexTileRows + row;
          if (!mbar_wait_warp(&sb->acc_full[as][sub], aph, wc)) { ok = false; break; }
          // the K stage of this tile is still held (k_empty also waits for us): its loads have
          // landed, and waiting on k_full makes the scales and the chunk mask visible here
          if (!mbar_wait_warp(&sb->k_full[kstage], (uint32_t)(acc_it / p.k_stages) & 1u, wc)) { ok = false; break; }
          tc_fence_after();
          const uint8_t* info = smem + p.off_kinfo + kstage * p.kinfo_bytes;
          // a position whose page id is outside the pool is ranked last (-inf)
          float ks = 1.0f;
          const bool page_ok = (*reinterpret_cast<const uint32_t*>(info) >> (row / p.box_rows)) & 1u;
          if (!page_ok)
            ks = __int_as_float(0xff800000);
          else if (!MX && p.k_scale)
            ks = reinterpret_cast<const float*>(info + 16)[row];
          const uint32_t col0 = (uint32_t)((as * NSUB + sub) * p.acc_cols);
          if constexpr (MX) {
            // this position's key group scales, then per 16-head chunk all groups' partial dot
            // products in one TMEM wait: d_h = sum_g D_g[h] * sq[h][g] * sk[g]
            float sk[kGroups];
#pragma unroll
            for (int g = 0; g < kGroups; ++g) {
              const uint32_t code = page_ok ? info[16 + row * kGroups + g] : 127u;
              sk[g] = code == 0xFFu ? __int_as_float(0x7fc00000) : ldexpf(1.0f, (int)code - 127);
            }
            const float* wq = w_s;
            float a4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            for (int hc = 0; hc < 4; ++hc) {
              if (hc * 16 >= p.H) break;   // warp-uniform
              uint32_t v[kGroups][16];
#pragma unroll
              for (int g = 0; g < kGroups; ++g)
                tmem_ld16(tmem_addr(tmem_base, quad * 32, col0 + g * p.n_cols + hc * 16), v[g]);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int h = hc * 16 + i;
                const float* sq = qmx_s + h * kGroups;
                float d = 0.0f;
#pragma unroll
                for (int g = 0; g < kGroups; ++g) d = fmaf(__uint_as_float(v[g][i]), sq[g] * sk[g], d);
                a4[i & 3] = fmaf(wq[h], fmaxf(d, 0.0f), a4[i & 3]);
              }
            }
            const float acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
            const int pos = info_pos[0];
            if (s <= pos) p.scores[(out_row0 + gi.g) * p.Lpad + s] = isinf(ks) ? ks : acc;
          } else {
          // QB queries' columns (up to QB x 64 heads) per TMEM wait: the loads of a batch are in
          // flight together, so each tile pays the TMEM latency once per batch (QB = 1 with two
          // sub-blocks, to stay within the registers of 320 threads)
          constexpr int QB = NSUB == 1 ? 2 : 1;
          for (int q0 = 0; q0 < p.nq_sub; q0 += QB) {
            uint32_t v[QB][4][16];
#pragma unroll
            for (int qq = 0; qq < QB; ++qq)
#pragma unroll
              for (int hc = 0; hc < 4; ++hc)
                if (q0 + qq < p.nq_sub && hc * 16 < p.H)   // warp-uniform
                  tmem_ld16(tmem_addr(tmem_base, quad * 32, col0 + (q0 + qq) * p.HP + hc * 16), v[qq][hc]);
            tmem_wait_ld();
#pragma unroll
            for (int qq = 0; qq < QB; ++qq) {
              if (q0 + qq >= p.nq_sub) break;
              const int qloc = sub * p.nq_sub + q0 + qq;
              const float4* wq = reinterpret_cast<const float4*>(w_s + qloc * p.HP);
              // four independent partial sums over the heads (w from shared memory, 4 per load),
              // updated two at a time by packed fp32 FMAs (each lane rounds as fmaf does)
              float a4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
              for (int hc = 0; hc < 4; ++hc) {
                if (hc * 16 >= p.H) break;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const float4 wv = wq[hc * 4 + i];
                  fma_f32x2(a4[0], a4[1], wv.x, wv.y, fmaxf(__uint_as_float(v[qq][hc][4 * i]), 0.0f),
                            fmaxf(__uint_as_float(v[qq][hc][4 * i + 1]), 0.0f));
                  fma_f32x2(a4[2], a4[3], wv.z, wv.w, fmaxf(__uint_as_float(v[qq][hc][4 * i + 2]), 0.0f),
                            fmaxf(__uint_as_float(v[qq][hc][4 * i + 3]), 0.0f));
                }
              }
              const float acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
              const int pos = info_pos[qloc];
              if (s <= pos) {
                const int j = gi.g * p.qg + qloc;
                const float val = isinf(ks) ? ks : acc * ks * info_qs[qloc];
                p.scores[(out_row0 + j) * p.Lpad + s] = val;
              }
            }
          }
          }
          tc_fence_before();
          mbar_arrive(&sb->acc_empty[as][sub]);
          __syncwarp();
          if (lane == 0) mbar_arrive(&sb->k_empty[kstage]);
        }
        ++seg;
      }
      remaining -= (t1 - t0);
      ++item;
      t0 = 0;
    }
    // the q boxes of the last group this thread issued land before the CTA may leave (one group
    // at a time: the next group's boxes are only issued once the MMAs have read this one's)
    if (et == 0 && q_issued > 0) mbar_drain(&sb->q_tma, (uint32_t)(q_issued - 1) & 1u, p.status);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

}  // namespace

cudaError_t launch_index_score(const IndexKernelParams& p, const CUtensorMap& kmap, const CUtensorMap& qmap, int grid,
                               bool pdl, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(64 + 128 * p.n_sub, 1, 1);
  cfg.dynamicSmemBytes = p.smem_bytes;
  cfg.stream = stream;
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  auto go = [&](auto kernel) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem_bytes);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, kernel, kmap, qmap, p);
  };
  // (K-block width, K blocks) from the row size: 64 B -> (64, 1), 128 B -> (128, 1), 256 B -> (128, 2)
  const int shape = p.kbw == 64 ? 0 : (p.n_kblocks == 1 ? 1 : 2);
#define SIA_INDEX_CASE(NS, SH, KB, NK)                                                            \
  if (p.n_sub == NS && shape == SH) return p.fp8 ? go(index_score_kernel<NS, KB, NK, 1>)         \
                                                 : go(index_score_kernel<NS, KB, NK, 0>);
  if (p.mx) {
    if (p.n_sub != 1) return cudaErrorInvalidValue;
    if (shape == 0) return go(index_score_kernel<1, 64, 1, 2>);
    if (shape == 1) return go(index_score_kernel<1, 128, 1, 2>);
    return cudaErrorInvalidValue;   // at most four groups (128 elements) per row
  }
  SIA_INDEX_CASE(1, 0, 64, 1)
  SIA_INDEX_CASE(1, 1, 128, 1)
  SIA_INDEX_CASE(1, 2, 128, 2)
  SIA_INDEX_CASE(2, 0, 64, 1)
  SIA_INDEX_CASE(2, 1, 128, 1)
  SIA_INDEX_CASE(2, 2, 128, 2)
#undef SIA_INDEX_CASE
  return cudaErrorInvalidValue;
}

}  // namespace sia
