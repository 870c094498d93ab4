// sparse_attend.cu -- MLA-style sparse attention over the Top-K latent rows, on tcgen05.
//
// For each query (b, j) and head h:
//     z_s = scale * q[h] . c[s]  (all d_latent + d_rope dims),  out[h] = sum_s softmax(z)_s c[s][:DL]
// over the positions s of the query's Top-K list, where c[s] is read straight out of the paged
// main latent KV cache through the page table ("Rapid Adaptation and Inference Optimization:
// Key Engineering Practices for Day0 LLM Support", section IV.4.2; steps 4-5 of the decode chain
// in "Day 0 Inference Adaptation and Performance Optimization for Hybrid Sparse Attention LLMs",
// section "Operator Fusion and Multi-Stream Scheduling"; MLA absorbed form: the value is the
// latent part of the same row).
//
// Design (B200).  All 128 heads of a query form the M = 128 side of every MMA.  The output
// accumulator O [128 heads x 512 dims] fp32 would fill the whole 256 KB of TMEM, so a CLUSTER
// OF TWO CTAs shares one (query, Top-K split):
//   - CTA r owns output dims [r*DL/2, (r+1)*DL/2) and gathers only its half of each latent row
//     (plus half of the rope dims), so together the pair reads each 1152-byte row once;
//   - each CTA computes a partial S = Q_r . C_r^T over its own dims, the two partials are
//     exchanged through distributed shared memory and summed (fp32 addition is commutative,
//     so both CTAs hold bit-identical S and take identical softmax decisions);
//   - each CTA runs the online softmax and accumulates O_r += P . C_r[:, its dims] in TMEM.
// Rows are gathered by TMA tile::gather4 (4 rows per instruction) into 128B/64B/32B-swizzled
// K-major tiles; the same tile serves as the K-major B operand of Q.C^T and as the MN-major B
// operand of P.C.  Rescaling of O is lazy: only when a head's running max grows by more than
// 2^8.  Splits of the Top-K list (to fill the GPU at small batch) write fp32 partials that
// combine_kernel merges by log-sum-exp.
#include <cuda.h>
#include <cuda_runtime.h>

#include "sia_internal.h"
#include "sia_ptx.cuh"

namespace sia {
namespace {

constexpr int kAttnThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 softmax / epilogue
constexpr int kStages = 2;         // latent-row tiles in flight per CTA
constexpr int kRows = kAttnTileRows;

template <int DL, int DR>
struct AttnLayout;

template <>
struct AttnLayout<512, 64> {
  static constexpr int kLatBlocks = 4;    // 4 x 64 latent dims per CTA
  static constexpr int kLatKbw = 128;
  static constexpr int kRopeKbw = 64;     // 32 rope dims per CTA
  static constexpr int kPvN = 256;
  static constexpr uint32_t kTmemCols = 512;
  __device__ static int lat_x(int r, int i) { return 256 * r + 64 * i; }
  __device__ static bool has_rope(int) { return true; }
  __device__ static int rope_x(int r) { return 512 + 32 * r; }
};

template <>
struct AttnLayout<64, 16> {
  static constexpr int kLatBlocks = 1;    // 32 latent dims per CTA
  static constexpr int kLatKbw = 64;
  static constexpr int kRopeKbw = 32;     // all 16 rope dims on CTA 0
  static constexpr int kPvN = 32;
  static constexpr uint32_t kTmemCols = 256;
  __device__ static int lat_x(int r, int) { return 32 * r; }
  __device__ static bool has_rope(int r) { return r == 0; }
  __device__ static int rope_x(int) { return 64; }
};

struct AttnMaps {
  CUtensorMap q_lat, q_rope, kv_lat, kv_rope;
};

template <class Lay>
struct AttnSmem {
  static constexpr uint32_t kQLatBytes = 128 * Lay::kLatKbw;
  static constexpr uint32_t kQRopeBytes = 128 * Lay::kRopeKbw;
  static constexpr uint32_t kCLatBytes = kRows * Lay::kLatKbw;
  static constexpr uint32_t kCRopeBytes = kRows * Lay::kRopeKbw;
  static constexpr uint32_t kCStageBytes = Lay::kLatBlocks * kCLatBytes + kCRopeBytes;
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffC = kOffQ + Lay::kLatBlocks * kQLatBytes + kQRopeBytes;
  static constexpr uint32_t kOffP = kOffC + kStages * kCStageBytes;
  static constexpr uint32_t kOffSx = kOffP + 128 * 128;                 // P: 128 x 64 bf16
  static constexpr uint32_t kOffBar = kOffSx + kRows * 128 * 4;         // Sx: 64 x 128 fp32
  static constexpr uint32_t kBytes = kOffBar + 256;
};

struct AttnBarriers {
  uint64_t c_full[kStages], c_empty[kStages];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full, p_empty;
  uint64_t q_full, q_empty;
  uint64_t o_full, o_empty;
  uint64_t sx_ready, sx_free;
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Does tile t of unit (bj, split) exist?  A tile exists when its first Top-K entry is a
// position (valid entries come first in a Top-K row, -1 padding after them).
__device__ __forceinline__ bool tile_exists(const AttnKernelParams& p, long long row_base,
                                            int row0, int row_end, int t) {
  const int r = row0 + t * kRows;
  return r < row_end && p.topk[row_base + r] >= 0;
}

// Physical cache row of Top-K entry idx of sequence b, or -1 when the entry is padding or
// points outside the context / page pool.
__device__ __forceinline__ int phys_row(const AttnKernelParams& p, int b, int idx, int L,
                                        bool report_bad) {
  if (idx < 0) return -1;
  if (idx >= L) {
    if (report_bad) report(p.status, SIA_DEV_BAD_POSITION);
    return -1;
  }
  const int page = p.page_table[(long long)b * p.max_pages + idx / p.P];
  if (page < 0 || page >= p.num_pages) {
    if (report_bad) report(p.status, SIA_DEV_BAD_PAGE);
    return -1;
  }
  return page * p.P + idx % p.P;
}

template <int DL, int DR>
__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attend_kernel(const __grid_constant__ AttnMaps maps, const AttnKernelParams p) {
  using Lay = AttnLayout<DL, DR>;
  using Sm = AttnSmem<Lay>;
  extern __shared__ __align__(1024) uint8_t smem[];
  AttnBarriers* sb = reinterpret_cast<AttnBarriers*>(smem + Sm::kOffBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int cluster_id = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;
  const bool rope = Lay::has_rope((int)rank);

  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) report(p.status, SIA_DEV_TIMEOUT);
    return;  // both CTAs of the pair see the same base alignment and leave together
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sb->c_full[s], 1);
      mbar_init(&sb->c_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sb->s_full[s], 1);
      mbar_init(&sb->s_empty[s], 128);
    }
    mbar_init(&sb->p_full, 128);
    mbar_init(&sb->p_empty, 1);
    mbar_init(&sb->q_full, 1);
    mbar_init(&sb->q_empty, 1);
    mbar_init(&sb->o_full, 1);
    mbar_init(&sb->o_empty, 128);
    mbar_init(&sb->sx_ready, 128);   // arrived by the peer's 128 softmax threads
    mbar_init(&sb->sx_free, 128);
    mbar_init(&sb->mma_done, 1);
    sb->abort = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&maps.q_lat);
    tma_prefetch_desc(&maps.q_rope);
    tma_prefetch_desc(&maps.kv_lat);
    tma_prefetch_desc(&maps.kv_rope);
  }
  if (warp == 1) {
    tmem_alloc(&sb->tmem_base, Lay::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = sb->tmem_base;
  volatile int* abort = &sb->abort;
  const uint32_t o_col = 0, s_col = Lay::kPvN;

  pdl_wait_primary();  // the Top-K lists come from the previous kernel on the stream

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    int it = 0, u_it = 0;
    bool ok = true;
    for (int u = cluster_id; u < p.units && ok; u += n_clusters, ++u_it) {
      const int bj = u / p.splits, split = u - bj * p.splits;
      const int b = bj / p.J;
      const int L = p.seq_lens[b];
      const long long row_base = (long long)bj * p.K;
      const int row0 = split * p.rows_per_split;
      const int row_end = min(p.K, row0 + p.rows_per_split);
      // query rows of all heads
      int go = 1;
      if (lane == 0) go = mbar_wait(&sb->q_empty, ((uint32_t)u_it & 1u) ^ 1u, abort, p.status);
      if (!__shfl_sync(0xffffffffu, go, 0)) { ok = false; break; }
      if (lane == 0) {
        const uint32_t qbytes = Lay::kLatBlocks * Sm::kQLatBytes + (rope ? Sm::kQRopeBytes : 0);
        mbar_arrive_expect_tx(&sb->q_full, qbytes);
        const int y = bj * p.H;
        for (int i = 0; i < Lay::kLatBlocks; ++i)
          tma_load_2d(smem + Sm::kOffQ + i * Sm::kQLatBytes, &maps.q_lat, &sb->q_full,
                      Lay::lat_x((int)rank, i), y);
        if (rope)
          tma_load_2d(smem + Sm::kOffQ + Lay::kLatBlocks * Sm::kQLatBytes, &maps.q_rope,
                      &sb->q_full, Lay::rope_x((int)rank), y);
      }
      for (int t = 0; tile_exists(p, row_base, row0, row_end, t); ++t, ++it) {
        const int stage = it % kStages;
        if (lane == 0) go = mbar_wait(&sb->c_empty[stage], ((uint32_t)(it / kStages) & 1u) ^ 1u, abort, p.status);
        if (!__shfl_sync(0xffffffffu, go, 0)) { ok = false; break; }
        // lanes 0..15 each gather one group of 4 rows
        int y[4] = {0, 0, 0, 0};
        if (lane < 16) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = row0 + t * kRows + lane * 4 + i;
            const int idx = r < row_end ? p.topk[row_base + r] : -1;
            const int pr = phys_row(p, b, idx, L, rank == 0);
            y[i] = pr < 0 ? 0 : pr;   // absent rows read row 0 (finite data) and are masked
          }
        }
        if (lane == 0)
          mbar_arrive_expect_tx(&sb->c_full[stage], Lay::kLatBlocks * Sm::kCLatBytes + (rope ? Sm::kCRopeBytes : 0));
        __syncwarp();
        if (lane < 16) {
          uint8_t* cst = smem + Sm::kOffC + stage * Sm::kCStageBytes;
#pragma unroll
          for (int i = 0; i < Lay::kLatBlocks; ++i)
            tma_gather4(cst + i * Sm::kCLatBytes + lane * 4 * Lay::kLatKbw, &maps.kv_lat,
                        &sb->c_full[stage], Lay::lat_x((int)rank, i), y[0], y[1], y[2], y[3]);
          if (rope)
            tma_gather4(cst + Lay::kLatBlocks * Sm::kCLatBytes + lane * 4 * Lay::kRopeKbw,
                        &maps.kv_rope, &sb->c_full[stage], Lay::rope_x((int)rank), y[0], y[1],
                        y[2], y[3]);
        }
        __syncwarp();
      }
    }
    if (lane == 0) {  // let in-flight gathers land before the CTA may leave
      const int first = it > kStages ? it - kStages : 0;
      for (int i = first; i < it; ++i)
        mbar_wait(&sb->c_full[i % kStages], (uint32_t)(i / kStages) & 1u, abort, p.status);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = umma_idesc(1, 1, false, false, kRows, 128);
      const uint32_t idesc_pv = umma_idesc(1, 1, false, true, Lay::kPvN, 128);
      const uint32_t q_base = smem_u32(smem + Sm::kOffQ);
      const uint32_t p_base = smem_u32(smem + Sm::kOffP);
      int it = 0, s_it = 0, pv_it = 0, u_it = 0;
      bool ok = true;
      for (int u = cluster_id; u < p.units && ok; u += n_clusters, ++u_it) {
        const int bj = u / p.splits, split = u - bj * p.splits;
        const long long row_base = (long long)bj * p.K;
        const int row0 = split * p.rows_per_split;
        const int row_end = min(p.K, row0 + p.rows_per_split);
        if (!mbar_wait(&sb->q_full, (uint32_t)u_it & 1u, abort, p.status)) { ok = false; break; }
        tc_fence_after();
        bool o_claimed = false, q_released = false;
        int prev_stage = -1;
        for (int t = 0;; ++t) {
          const bool exists = tile_exists(p, row_base, row0, row_end, t);
          if (exists) {
            const int stage = it % kStages;
            const int sbuf = s_it & 1;
            if (!mbar_wait(&sb->c_full[stage], (uint32_t)(it / kStages) & 1u, abort, p.status)) { ok = false; break; }
            if (!mbar_wait(&sb->s_empty[sbuf], ((uint32_t)(s_it >> 1) & 1u) ^ 1u, abort, p.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t c_base = smem_u32(smem + Sm::kOffC + stage * Sm::kCStageBytes);
            const uint32_t d = tmem_base + s_col + (uint32_t)(sbuf * kRows);
            bool acc = false;
#pragma unroll
            for (int i = 0; i < Lay::kLatBlocks; ++i)
#pragma unroll
              for (int ks = 0; ks < Lay::kLatKbw / 32; ++ks) {
                const uint64_t ad = umma_smem_desc(q_base + i * Sm::kQLatBytes + ks * 32, 16,
                                                   8 * Lay::kLatKbw, umma_layout_type(Lay::kLatKbw));
                const uint64_t bd = umma_smem_desc(c_base + i * Sm::kCLatBytes + ks * 32, 16,
                                                   8 * Lay::kLatKbw, umma_layout_type(Lay::kLatKbw));
                umma_f16(d, ad, bd, idesc_qk, acc);
                acc = true;
              }
            if (rope) {
#pragma unroll
              for (int ks = 0; ks < Lay::kRopeKbw / 32; ++ks) {
                const uint64_t ad = umma_smem_desc(q_base + Lay::kLatBlocks * Sm::kQLatBytes + ks * 32, 16,
                                                   8 * Lay::kRopeKbw, umma_layout_type(Lay::kRopeKbw));
                const uint64_t bd = umma_smem_desc(c_base + Lay::kLatBlocks * Sm::kCLatBytes + ks * 32, 16,
                                                   8 * Lay::kRopeKbw, umma_layout_type(Lay::kRopeKbw));
                umma_f16(d, ad, bd, idesc_qk, true);
              }
            }
            umma_commit(&sb->s_full[sbuf]);
            if (!tile_exists(p, row_base, row0, row_end, t + 1)) {
              umma_commit(&sb->q_empty);  // Q may be reloaded once these MMAs are done
              q_released = true;
            }
          }
          if (t > 0) {
            // P . C for the previous tile
            if (!mbar_wait(&sb->p_full, (uint32_t)pv_it & 1u, abort, p.status)) { ok = false; break; }
            if (!o_claimed) {
              if (!mbar_wait(&sb->o_empty, ((uint32_t)u_it & 1u) ^ 1u, abort, p.status)) { ok = false; break; }
              o_claimed = true;
            }
            tc_fence_after();
            const uint32_t c_base = smem_u32(smem + Sm::kOffC + prev_stage * Sm::kCStageBytes);
#pragma unroll
            for (int ks = 0; ks < kRows / 16; ++ks) {
              const uint64_t ad = umma_smem_desc(p_base + ks * 32, 16, 1024, umma_layout_type(128));
              const uint64_t bd = umma_smem_desc(c_base + ks * 16 * Lay::kLatKbw, Sm::kCLatBytes,
                                                 8 * Lay::kLatKbw, umma_layout_type(Lay::kLatKbw));
              umma_f16(tmem_base + o_col, ad, bd, idesc_pv, (t > 1) || ks > 0);
            }
            umma_commit(&sb->c_empty[prev_stage]);
            umma_commit(&sb->p_empty);
            ++pv_it;
          }
          if (!exists) break;
          prev_stage = it % kStages;
          ++it;
          ++s_it;
        }
        if (!ok) break;
        if (!q_released) umma_commit(&sb->q_empty);
        if (!o_claimed) {
          if (!mbar_wait(&sb->o_empty, ((uint32_t)u_it & 1u) ^ 1u, abort, p.status)) { ok = false; break; }
        }
        umma_commit(&sb->o_full);
      }
      umma_commit(&sb->mma_done);
      mbar_wait(&sb->mma_done, 0, abort, p.status);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int quad = warp & 3;
    const int h = quad * 32 + lane;   // head = TMEM lane
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quad * 32) << 16);
    float* sx = reinterpret_cast<float*>(smem + Sm::kOffSx);
    const uint32_t sx_peer = mapa_cluster(sx, peer);
    const uint32_t p_row = smem_u32(smem + Sm::kOffP);
    int s_it = 0, pv_it = 0, u_it = 0;
    bool ok = true;
    for (int u = cluster_id; u < p.units && ok; u += n_clusters, ++u_it) {
      const int bj = u / p.splits, split = u - bj * p.splits;
      const int b = bj / p.J;
      const int L = p.seq_lens[b];
      const long long row_base = (long long)bj * p.K;
      const int row0 = split * p.rows_per_split;
      const int row_end = min(p.K, row0 + p.rows_per_split);
      float m = -INFINITY, l = 0.0f;
      int t = 0;
      for (; tile_exists(p, row_base, row0, row_end, t); ++t, ++s_it, ++pv_it) {
        // which of the tile's 64 rows are real positions
        const int r_lo = row0 + t * kRows + lane, r_hi = r_lo + 32;
        const int i_lo = r_lo < row_end ? p.topk[row_base + r_lo] : -1;
        const int i_hi = r_hi < row_end ? p.topk[row_base + r_hi] : -1;
        const uint32_t v_lo = __ballot_sync(0xffffffffu, phys_row(p, b, i_lo, L, false) >= 0);
        const uint32_t v_hi = __ballot_sync(0xffffffffu, phys_row(p, b, i_hi, L, false) >= 0);
        const uint64_t valid = ((uint64_t)v_hi << 32) | v_lo;

        const int sbuf = s_it & 1;
        if (!mbar_wait(&sb->s_full[sbuf], (uint32_t)(s_it >> 1) & 1u, abort, p.status)) { ok = false; break; }
        tc_fence_after();
        float s[kRows];
        {
          uint32_t r[4][16];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld16(lane_addr + s_col + sbuf * kRows + c * 16, r[c]);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 16; ++i) s[c * 16 + i] = __uint_as_float(r[c][i]);
        }
        tc_fence_before();
        mbar_arrive(&sb->s_empty[sbuf]);

        // exchange partial scores with the peer CTA: Sx[row/4][head][row%4]
        if (!mbar_wait<true>(&sb->sx_free, ((uint32_t)s_it & 1u) ^ 1u, abort, p.status)) { ok = false; break; }
#pragma unroll
        for (int g = 0; g < kRows / 4; ++g)
          st_cluster_v4(sx_peer + (uint32_t)((g * 128 + h) * 16), s[4 * g], s[4 * g + 1], s[4 * g + 2], s[4 * g + 3]);
        mbar_arrive_cluster(&sb->sx_ready, peer);
        if (!mbar_wait<true>(&sb->sx_ready, (uint32_t)s_it & 1u, abort, p.status)) { ok = false; break; }
#pragma unroll
        for (int g = 0; g < kRows / 4; ++g) {
          const float4 v = *reinterpret_cast<const float4*>(sx + (g * 128 + h) * 4);
          s[4 * g] += v.x;
          s[4 * g + 1] += v.y;
          s[4 * g + 2] += v.z;
          s[4 * g + 3] += v.w;
        }
        mbar_arrive_cluster(&sb->sx_free, peer);

        // online softmax (base 2), lazy rescale
        float mt = -INFINITY;
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
          s[i] = (valid >> i & 1ull) ? s[i] * p.scale_log2 : -INFINITY;
          mt = fmaxf(mt, s[i]);
        }
        float alpha = 1.0f;
        const bool need = mt > m + 8.0f;
        if (need) {
          alpha = fast_exp2(m - mt);   // 0 when m is -inf
          m = mt;
        }
        float psum = 0.0f;
        uint32_t pk[kRows / 2];
#pragma unroll
        for (int i = 0; i < kRows; i += 2) {
          const float p0 = (valid >> i & 1ull) ? fast_exp2(s[i] - m) : 0.0f;
          const float p1 = (valid >> (i + 1) & 1ull) ? fast_exp2(s[i + 1] - m) : 0.0f;
          psum += p0 + p1;
          pk[i / 2] = pack_bf16x2(p0, p1);
        }
        l = l * alpha + psum;

        // P . C of the previous tile must be done before O is rescaled or P overwritten
        if (!mbar_wait(&sb->p_empty, ((uint32_t)pv_it & 1u) ^ 1u, abort, p.status)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, need && t > 0)) {
#pragma unroll 1
          for (int c = 0; c < Lay::kPvN; c += 16) {
            uint32_t r[16];
            tmem_ld16(lane_addr + o_col + c, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st16(lane_addr + o_col + c, r);
          }
          tmem_wait_st();
        }
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(p_row + swizzled_offset((uint32_t)h, (uint32_t)(c * 16), 128), pk[4 * c],
                       pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sb->p_full);
      }
      if (!ok) break;
      // ---- unit epilogue: normalise O and write it out
      if (!mbar_wait(&sb->o_full, (uint32_t)u_it & 1u, abort, p.status)) { ok = false; break; }
      tc_fence_after();
      const bool any = t > 0 && l > 0.0f;
      const float inv = any ? 1.0f / l : 0.0f;
      const float lse = any ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
      const bool real_head = h < p.H;
      if (p.splits == 1) {
        uint16_t* orow = p.out + ((long long)bj * p.H + h) * p.DL + rank * Lay::kPvN;
#pragma unroll 1
        for (int c = 0; c < Lay::kPvN; c += 16) {
          uint32_t r[16];
          if (t > 0) {
            tmem_ld16(lane_addr + o_col + c, r);
            tmem_wait_ld();
          }
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            w[i] = t > 0 ? pack_bf16x2(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv) : 0u;
          if (real_head) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c);
            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
          }
        }
        if (real_head && rank == 0 && p.lse) p.lse[(long long)bj * p.H + h] = lse;
      } else {
        float* orow = p.part_o + (((long long)split * p.B * p.J + bj) * p.H + h) * p.DL + rank * Lay::kPvN;
#pragma unroll 1
        for (int c = 0; c < Lay::kPvN; c += 16) {
          uint32_t r[16];
          if (t > 0) {
            tmem_ld16(lane_addr + o_col + c, r);
            tmem_wait_ld();
          }
          if (real_head) {
            float4* dst = reinterpret_cast<float4*>(orow + c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = t > 0 ? make_float4(__uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
                                           __uint_as_float(r[4 * i + 2]) * inv, __uint_as_float(r[4 * i + 3]) * inv)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        if (real_head && rank == 0) p.part_lse[((long long)split * p.B * p.J + bj) * p.H + h] = lse;
      }
      tc_fence_before();
      mbar_arrive(&sb->o_empty);
    }
  }
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer no longer writes into our shared memory or arrives on our barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Lay::kTmemCols);
  }
}

// Log-sum-exp merge of the per-split partial results of one query row.
__global__ void __launch_bounds__(256) combine_kernel(const CombineKernelParams p) {
  pdl_wait_primary();
  const int bj = blockIdx.x;
  const int per_head = p.DL / 4;
  for (int i = threadIdx.x; i < p.H * per_head; i += blockDim.x) {
    const int h = i / per_head, d4 = (i - h * per_head) * 4;
    float mx = -INFINITY;
    for (int s = 0; s < p.splits; ++s)
      mx = fmaxf(mx, p.part_lse[((long long)s * p.BJ + bj) * p.H + h]);
    float wsum = 0.0f, o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
    if (mx != -INFINITY) {
      for (int s = 0; s < p.splits; ++s) {
        const float ls = p.part_lse[((long long)s * p.BJ + bj) * p.H + h];
        const float wgt = ls == -INFINITY ? 0.0f : expf(ls - mx);
        const float4 v = *reinterpret_cast<const float4*>(p.part_o + (((long long)s * p.BJ + bj) * p.H + h) * p.DL + d4);
        o0 += wgt * v.x;
        o1 += wgt * v.y;
        o2 += wgt * v.z;
        o3 += wgt * v.w;
        wsum += wgt;
      }
    }
    const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
    uint16_t* dst = p.out + ((long long)bj * p.H + h) * p.DL + d4;
    const uint32_t a = pack_bf16x2(o0 * inv, o1 * inv), c = pack_bf16x2(o2 * inv, o3 * inv);
    *reinterpret_cast<uint2*>(dst) = make_uint2(a, c);
    if (d4 == 0 && p.lse) p.lse[(long long)bj * p.H + h] = wsum > 0.0f ? mx + logf(wsum) : -INFINITY;
  }
  pdl_launch_dependents();
}

template <int DL, int DR>
cudaError_t launch_attend_impl(const AttnKernelParams& p, const CUtensorMap* maps, int n_clusters,
                               bool pdl, cudaStream_t stream) {
  using Sm = AttnSmem<AttnLayout<DL, DR>>;
  // at most two CTAs per SM may share the 512 TMEM columns (kTmemCols each <= 256 when two fit)
  const size_t smem = Sm::kBytes < 100 * 1024 ? 100 * 1024 : Sm::kBytes;
  cudaError_t e = cudaFuncSetAttribute(sparse_attend_kernel<DL, DR>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  AttnMaps m;
  m.q_lat = maps[0];
  m.q_rope = maps[1];
  m.kv_lat = maps[2];
  m.kv_rope = maps[3];
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.gridDim = dim3(2 * n_clusters, 1, 1);
  cfg.blockDim = dim3(kAttnThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  int na = 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = 2;
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
  return cudaLaunchKernelEx(&cfg, sparse_attend_kernel<DL, DR>, m, p);
}

}  // namespace

size_t attend_smem_bytes(int dl, int dr) {
  if (dl == 512 && dr == 64) return AttnSmem<AttnLayout<512, 64>>::kBytes;
  if (dl == 64 && dr == 16) return AttnSmem<AttnLayout<64, 16>>::kBytes;
  return 0;
}

cudaError_t launch_sparse_attend(const AttnKernelParams& p, const CUtensorMap* maps,
                                 int n_clusters, bool pdl, cudaStream_t stream) {
  if (p.DL == 512 && p.DR == 64) return launch_attend_impl<512, 64>(p, maps, n_clusters, pdl, stream);
  if (p.DL == 64 && p.DR == 16) return launch_attend_impl<64, 16>(p, maps, n_clusters, pdl, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_combine(const CombineKernelParams& p, bool pdl, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3((unsigned)p.BJ, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, combine_kernel, p);
}

}  // namespace sia
