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
#include <cuda_fp16.h>

#include <type_traits>
#include <cuda_runtime.h>

#include "sia_internal.h"
#include "sia_ptx.cuh"

namespace sia {
namespace {

constexpr int kProducerWarps = 8;   // cp.async gather (+ TMA for q)
constexpr int kFirstExchangeWarp = 4;
constexpr int kFirstProducerWarp = 8;
constexpr int kMmaWarp = 16;
// warps 0-3 softmax + epilogue, 4-7 partial-logit exchange, 8-15 gather, 16 MMA
constexpr int kAttnThreads = 544;
// Registers per thread after the split.  The block is launched with kLaunchRegs x 544
// registers (ptxas' allocation for 544 threads); the softmax warpgroup takes 168 (a tile of
// fp32 logits), the two gather warpgroups give back down to 56, the exchange warpgroup and the
// MMA warp keep the launch value, so setmaxnreg.inc never waits for registers that are not there.
constexpr int kLaunchRegs = 96;
constexpr int kSoftmaxRegs = 168;
constexpr int kGatherRegs = 56;
static_assert(128 * kSoftmaxRegs + 256 * kGatherRegs + 128 * kLaunchRegs + 32 * kLaunchRegs <=
                  kAttnThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr int kStages = 3;          // latent-row tiles in flight per CTA
constexpr int kRows = kAttnTileRows;

template <int DL, int DR>
struct AttnLayout;

// Per-CTA share of each latent row: CTA r gathers latent dims [DL/2 r, DL/2 (r+1)) (used by both
// Q.C^T and P.C) and a share of the rope dims (used by Q.C^T only).
template <>
struct AttnLayout<512, 64> {
  static constexpr int kLatBlocks = 4;    // 4 x 64 latent dims per CTA, 128-byte swizzled rows
  static constexpr int kLatKbw = 128;
  static constexpr int kRopeKbw = 64;     // 32 rope dims per CTA, 64-byte swizzled rows
  static constexpr int kPvN = 256;
  static constexpr uint32_t kTmemCols = 512;
  __device__ static bool has_rope(int) { return true; }
  __device__ static int lat_x(int r, int i) { return 256 * r + 64 * i; }   // q columns (elements)
  __device__ static int rope_x(int r) { return 512 + 32 * r; }
  static constexpr int kChunks0 = 36, kChunks1 = 36;                      // 16-byte pieces per row
  __device__ static int chunk_src(int r, int k) { return k < 32 ? 512 * r + 16 * k : 1024 + 64 * r + 16 * (k - 32); }
  __device__ static uint32_t chunk_dst(int row, int k) {
    return k < 32 ? (uint32_t)(k >> 3) * (kAttnTileRows * 128) + swizzled_offset(row, (k & 7) * 16, 128)
                  : 4u * (kAttnTileRows * 128) + swizzled_offset(row, (k - 32) * 16, 64);
  }
};

template <>
struct AttnLayout<64, 16> {
  static constexpr int kLatBlocks = 1;    // 32 latent dims per CTA, 64-byte swizzled rows
  static constexpr int kLatKbw = 64;
  static constexpr int kRopeKbw = 32;     // all 16 rope dims on CTA 0, 32-byte swizzled rows
  static constexpr int kPvN = 32;
  static constexpr uint32_t kTmemCols = 256;
  __device__ static bool has_rope(int r) { return r == 0; }
  __device__ static int lat_x(int r, int) { return 32 * r; }
  __device__ static int rope_x(int) { return 64; }
  static constexpr int kChunks0 = 6, kChunks1 = 4;
  __device__ static int chunk_src(int r, int k) { return k < 4 ? 64 * r + 16 * k : 128 + 16 * (k - 4); }
  __device__ static uint32_t chunk_dst(int row, int k) {
    return k < 4 ? swizzled_offset(row, k * 16, 64) : (uint32_t)(kAttnTileRows * 64) + swizzled_offset(row, (k - 4) * 16, 32);
  }
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
  static constexpr uint32_t kOffSx = kOffC + kStages * kCStageBytes;   // peer logits, fp16
  static constexpr uint32_t kOffRows = kOffSx + kRows * 128 * 2;
  // per unit (double-buffered): physical cache row of each Top-K entry, validity bits, and
  // each gather warp's lowest position of a -1 entry
  static constexpr uint32_t kOffMask = kOffRows + 2 * kAttnMaxSplitRows * 4;
  static constexpr uint32_t kOffFirstNeg = kOffMask + 2 * (kAttnMaxSplitRows / 8);
  static constexpr uint32_t kOffBar = kOffFirstNeg + 2 * kProducerWarps * 4;
  static constexpr uint32_t kBytes = kOffBar + 256;
};

struct AttnBarriers {
  uint64_t c_full[kStages], c_empty[kStages];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2], p_empty[2];
  uint64_t q_full, q_empty;
  uint64_t o_full, o_empty;
  uint64_t sx_ready, sx_free;
  uint64_t tab_full[2], tab_free[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float2 unpack_f16x2(uint32_t v) {
  __half2 h = *reinterpret_cast<__half2*>(&v);
  return __half22float2(h);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

template <int DL, int DR>
__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attend_kernel(const __grid_constant__ AttnMaps maps, const AttnKernelParams p) {
  static_assert(kAttnThreads == 544, "role layout assumes 17 warps");
  using Lay = AttnLayout<DL, DR>;
  using Sm = AttnSmem<Lay>;
  extern __shared__ __align__(1024) uint8_t smem[];
  AttnBarriers* sb = reinterpret_cast<AttnBarriers*>(smem + Sm::kOffBar);
  int32_t* rows_tab = reinterpret_cast<int32_t*>(smem + Sm::kOffRows);        // [2][max rows]
  uint32_t* mask_tab = reinterpret_cast<uint32_t*>(smem + Sm::kOffMask);      // [2][max rows/32]
  int32_t* fneg_tab = reinterpret_cast<int32_t*>(smem + Sm::kOffFirstNeg);    // [2][gather warps]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int cluster_id = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;
  const bool rope = Lay::has_rope((int)rank);
  const int DC = p.DL + p.DR;

  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) report(p.status, SIA_DEV_TIMEOUT);
    return;  // both CTAs of the pair see the same base alignment and leave together
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sb->c_full[s], kProducerWarps * 32);  // one cp.async completion per gather thread
      mbar_init(&sb->c_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sb->s_full[s], 1);
      mbar_init(&sb->s_empty[s], 128);
      mbar_init(&sb->p_full[s], 128);
      mbar_init(&sb->p_empty[s], 1);
      mbar_init(&sb->tab_full[s], kProducerWarps * 32);
      mbar_init(&sb->tab_free[s], 128);
    }
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
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sb->tmem_base, Lay::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = sb->tmem_base;
  volatile int* abort = &sb->abort;
  const uint32_t o_col = 0, s_col = Lay::kPvN, p_col = Lay::kPvN + 2 * kRows;

  pdl_wait_primary();  // the Top-K lists come from the previous kernel on the stream

  if (warp >= kFirstProducerWarp && warp < kFirstProducerWarp + kProducerWarps) {
    // ---------------------------------------------------------------- gather (4 warps)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kGatherRegs));
    const int ptid = threadIdx.x - kFirstProducerWarp * 32;   // 0..255
    const int pwarp = warp - kFirstProducerWarp;
    const uint8_t* kv = static_cast<const uint8_t*>(p.kv);
    // one tile of gathers: consecutive threads take consecutive 16-byte pieces of a row, so a
    // warp reads whole 512-byte runs of a latent row at a time
    auto gather_tile = [&](auto nch_c, uint32_t cst, const int32_t* rows) {
      constexpr int NCH = decltype(nch_c)::value;
#pragma unroll 4
      for (int i = ptid; i < kRows * NCH; i += kProducerWarps * 32) {
        const int row = i / NCH, k = i - row * NCH;
        cp_async16(cst + Lay::chunk_dst(row, k), kv + (size_t)(uint32_t)rows[row] * (DC * 2) + Lay::chunk_src((int)rank, k));
      }
    };
    int it = 0, u_it = 0;
    bool ok = true;
    for (int u = cluster_id; u < p.units && ok; u += n_clusters, ++u_it) {
      const int bj = u / p.splits, split = u - bj * p.splits;
      const int b = bj / p.J;
      const int L = p.seq_lens[b];
      const long long row_base = (long long)bj * p.K;
      const int row0 = split * p.rows_per_split;
      const int nrows = min(p.K, row0 + p.rows_per_split) - row0;
      const int nrows_pad = (nrows + kRows - 1) / kRows * kRows;
      const int buf = u_it & 1;
      // query rows of all heads (TMA; independent of the Top-K list)
      if (ptid == 0) {
        if (mbar_wait(&sb->q_empty, ((uint32_t)u_it & 1u) ^ 1u, abort, p.status)) {
          const uint32_t qbytes = Lay::kLatBlocks * Sm::kQLatBytes + (rope ? Sm::kQRopeBytes : 0);
          mbar_arrive_expect_tx(&sb->q_full, qbytes);
          const int y = bj * p.H;
          for (int i = 0; i < Lay::kLatBlocks; ++i)
            tma_load_2d(smem + Sm::kOffQ + i * Sm::kQLatBytes, &maps.q_lat, &sb->q_full, Lay::lat_x((int)rank, i), y);
          if (rope)
            tma_load_2d(smem + Sm::kOffQ + Lay::kLatBlocks * Sm::kQLatBytes, &maps.q_rope, &sb->q_full,
                        Lay::rope_x((int)rank), y);
        }
      }
      // resolve this unit's Top-K entries to physical cache rows: 16 entries per thread, all
      // loads of a thread in flight at once
      if (!mbar_wait(&sb->tab_free[buf], ((uint32_t)(u_it >> 1) & 1u) ^ 1u, abort, p.status)) { ok = false; break; }
      int32_t* rt = rows_tab + buf * kAttnMaxSplitRows;
      uint32_t* mt = mask_tab + buf * (kAttnMaxSplitRows / 32);
      const int32_t* tk = p.topk + row_base + row0;
      const int32_t* pt_row = p.page_table + (long long)b * p.max_pages;
      constexpr int kPer = kAttnMaxSplitRows / (kProducerWarps * 32);
      int idx[kPer], pg[kPer];
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int r = ptid + k * kProducerWarps * 32;
        idx[k] = r < nrows ? tk[r] : -1;
      }
#pragma unroll
      for (int k = 0; k < kPer; ++k) pg[k] = (idx[k] >= 0 && idx[k] < L) ? pt_row[idx[k] / p.P] : -1;
      int fneg = nrows;
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int r = ptid + k * kProducerWarps * 32;
        if (k * kProducerWarps * 32 < nrows_pad) {     // warp-uniform (nrows_pad is a multiple of 64)
          if (r < nrows && idx[k] < 0) fneg = min(fneg, r);
          const bool pos_ok = idx[k] >= 0 && idx[k] < L;
          const bool page_ok = pg[k] >= 0 && pg[k] < p.num_pages;
          if (rank == 0 && idx[k] >= 0) {
            if (idx[k] >= L) report(p.status, SIA_DEV_BAD_POSITION);
            else if (!page_ok) report(p.status, SIA_DEV_BAD_PAGE);
          }
          const bool v = pos_ok && page_ok;
          rt[r] = v ? pg[k] * p.P + idx[k] % p.P : 0;   // absent rows read row 0 (finite data)
          const unsigned bits = __ballot_sync(0xffffffffu, v);
          if (lane == 0) mt[(r - lane) / 32] = bits;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) fneg = min(fneg, __shfl_xor_sync(0xffffffffu, fneg, o));
      if (lane == 0) fneg_tab[buf * kProducerWarps + pwarp] = fneg;
      mbar_arrive(&sb->tab_full[buf]);
      if (!mbar_wait(&sb->tab_full[buf], (uint32_t)(u_it >> 1) & 1u, abort, p.status)) { ok = false; break; }
      int first_neg = nrows;
#pragma unroll
      for (int w = 0; w < kProducerWarps; ++w) first_neg = min(first_neg, fneg_tab[buf * kProducerWarps + w]);
      const int ntiles = (first_neg + kRows - 1) / kRows;
      for (int t = 0; t < ntiles; ++t, ++it) {
        const int stage = it % kStages;
        if (!mbar_wait(&sb->c_empty[stage], ((uint32_t)(it / kStages) & 1u) ^ 1u, abort, p.status)) { ok = false; break; }
        const uint32_t cst = smem_u32(smem + Sm::kOffC + stage * Sm::kCStageBytes);
        const int32_t* rows = rt + t * kRows;
        if (rank == 0) gather_tile(std::integral_constant<int, Lay::kChunks0>{}, cst, rows);
        else gather_tile(std::integral_constant<int, Lay::kChunks1>{}, cst, rows);
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&sb->c_full[stage])) : "memory");
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // our copies have landed before we may leave
    if (ptid == 0 && u_it > 0) mbar_wait(&sb->q_full, (uint32_t)(u_it - 1) & 1u, abort, p.status);
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = umma_idesc(1, 1, false, false, kRows, 128);
      const uint32_t idesc_pv = umma_idesc(1, 1, false, true, Lay::kPvN, 128);
      const uint32_t q_base = smem_u32(smem + Sm::kOffQ);
      int it = 0, s_it = 0, pv_it = 0, u_it = 0;
      bool ok = true;
      for (int u = cluster_id; u < p.units && ok; u += n_clusters, ++u_it) {
        const int buf = u_it & 1;
        if (!mbar_wait(&sb->tab_full[buf], (uint32_t)(u_it >> 1) & 1u, abort, p.status)) { ok = false; break; }
        int first_neg = 1 << 30;
        for (int w = 0; w < kProducerWarps; ++w) first_neg = min(first_neg, fneg_tab[buf * kProducerWarps + w]);
        const int ntiles = (first_neg + kRows - 1) / kRows;
        if (!mbar_wait(&sb->q_full, (uint32_t)u_it & 1u, abort, p.status)) { ok = false; break; }
        tc_fence_after();
        bool o_claimed = false;
        int prev_stage = -1;
        for (int t = 0; t <= ntiles; ++t) {
          if (t < ntiles) {
            const int stage = it % kStages;
            const int sbuf = s_it & 1;
            if (!mbar_wait(&sb->c_full[stage], (uint32_t)(it / kStages) & 1u, abort, p.status)) { ok = false; break; }
            if (!mbar_wait(&sb->s_empty[sbuf], ((uint32_t)(s_it >> 1) & 1u) ^ 1u, abort, p.status)) { ok = false; break; }
            fence_proxy_async_smem();   // the gathered rows were written by cp.async
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
            if (t + 1 == ntiles) umma_commit(&sb->q_empty);  // Q reusable once these are done
          }
          if (t > 0) {
            // O += P . C for the previous tile, with P (bf16) read straight from TMEM
            const int pb = pv_it & 1;
            if (!mbar_wait(&sb->p_full[pb], (uint32_t)(pv_it >> 1) & 1u, abort, p.status)) { ok = false; break; }
            if (!o_claimed) {
              if (!mbar_wait(&sb->o_empty, ((uint32_t)u_it & 1u) ^ 1u, abort, p.status)) { ok = false; break; }
              o_claimed = true;
            }
            tc_fence_after();
            const uint32_t c_base = smem_u32(smem + Sm::kOffC + prev_stage * Sm::kCStageBytes);
#pragma unroll
            for (int ks = 0; ks < kRows / 16; ++ks) {
              const uint64_t bd = umma_smem_desc(c_base + ks * 16 * Lay::kLatKbw, Sm::kCLatBytes,
                                                 8 * Lay::kLatKbw, umma_layout_type(Lay::kLatKbw));
              umma_f16_ts(tmem_base + o_col, tmem_base + p_col + (uint32_t)(pb * (kRows / 2) + ks * 8), bd,
                          idesc_pv, (t > 1) || ks > 0);
            }
            umma_commit(&sb->c_empty[prev_stage]);
            umma_commit(&sb->p_empty[pb]);
            ++pv_it;
          }
          if (t < ntiles) {
            prev_stage = it % kStages;
            ++it;
            ++s_it;
          }
        }
        if (!ok) break;
        if (ntiles == 0) umma_commit(&sb->q_empty);
        if (!o_claimed) {
          if (!mbar_wait(&sb->o_empty, ((uint32_t)u_it & 1u) ^ 1u, abort, p.status)) { ok = false; break; }
        }
        umma_commit(&sb->o_full);
      }
      umma_commit(&sb->mma_done);
      mbar_wait(&sb->mma_done, 0, abort, p.status);
    }
    __syncwarp();
  } else if (warp >= kFirstExchangeWarp && warp < kFirstExchangeWarp + 4) {
    // ---------------------------------------------------------------- partial-logit exchange
    // Reads this CTA's partial logits of a tile from TMEM, rounds them to fp16 (scaled to base
    // 2) and pushes them into the peer CTA's exchange buffer; the peer's softmax warps add them
    // to their own partials.  Both CTAs add the same two fp16 values, so their softmax inputs
    // agree bit for bit.
    const int quad = warp & 3;
    const int h = quad * 32 + lane;
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quad * 32) << 16);
    const uint32_t sx_peer = mapa_shared(smem_u32(smem + Sm::kOffSx), peer);
    int s_it = 0, u_it = 0;
    bool ok = true;
    for (int u = cluster_id; u < p.units && ok; u += n_clusters, ++u_it) {
      const int buf = u_it & 1;
      if (!mbar_wait(&sb->tab_full[buf], (uint32_t)(u_it >> 1) & 1u, abort, p.status)) { ok = false; break; }
      int first_neg = 1 << 30;
      for (int w = 0; w < kProducerWarps; ++w) first_neg = min(first_neg, fneg_tab[buf * kProducerWarps + w]);
      const int ntiles = (first_neg + kRows - 1) / kRows;
      for (int t = 0; t < ntiles; ++t, ++s_it) {
        const int sbuf = s_it & 1;
        const uint32_t scol = lane_addr + s_col + sbuf * kRows;
        if (!mbar_wait(&sb->s_full[sbuf], (uint32_t)(s_it >> 1) & 1u, abort, p.status)) { ok = false; break; }
        tc_fence_after();
        uint32_t own[kRows / 2];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t r[2][16];
          tmem_ld16(scol + half * 32, r[0]);
          tmem_ld16(scol + half * 32 + 16, r[1]);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int i = 0; i < 8; ++i)
              own[half * 16 + c * 8 + i] = pack_f16x2(__uint_as_float(r[c][2 * i]) * p.scale_log2,
                                                      __uint_as_float(r[c][2 * i + 1]) * p.scale_log2);
        }
        if (!mbar_wait<true>(&sb->sx_free, ((uint32_t)s_it & 1u) ^ 1u, abort, p.status)) { ok = false; break; }
#pragma unroll
        for (int g = 0; g < kRows / 8; ++g)
          asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sx_peer + (uint32_t)((g * 128 + h) * 16)),
                       "r"(own[4 * g]), "r"(own[4 * g + 1]), "r"(own[4 * g + 2]), "r"(own[4 * g + 3])
                       : "memory");
        mbar_arrive_cluster(&sb->sx_ready, peer);
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    const int quad = warp & 3;
    const int h = quad * 32 + lane;   // head = TMEM lane
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quad * 32) << 16);
    int s_it = 0, pv_it = 0, u_it = 0;
    bool ok = true;

    for (int u = cluster_id; u < p.units && ok; u += n_clusters, ++u_it) {
      const int bj = u / p.splits, split = u - bj * p.splits;
      const int buf = u_it & 1;
      if (!mbar_wait(&sb->tab_full[buf], (uint32_t)(u_it >> 1) & 1u, abort, p.status)) { ok = false; break; }
      int first_neg = 1 << 30;
      for (int w = 0; w < kProducerWarps; ++w) first_neg = min(first_neg, fneg_tab[buf * kProducerWarps + w]);
      const int ntiles = (first_neg + kRows - 1) / kRows;
      const uint32_t* mt = mask_tab + buf * (kAttnMaxSplitRows / 32);
      float m = -INFINITY, l = 0.0f;
      float s[kRows];
      for (int t = 0; t < ntiles; ++t, ++pv_it) {
        // logits of tile t (base 2) = own partial (TMEM) + the peer's partial (exchange buffer),
        // each rounded to fp16 exactly as the exchange warps of both CTAs round them
        const int sbuf = s_it & 1;
        if (!mbar_wait(&sb->s_full[sbuf], (uint32_t)(s_it >> 1) & 1u, abort, p.status)) { ok = false; break; }
        if (!mbar_wait<true>(&sb->sx_ready, (uint32_t)s_it & 1u, abort, p.status)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t r[2][16];
          tmem_ld16(lane_addr + s_col + sbuf * kRows + half * 32, r[0]);
          tmem_ld16(lane_addr + s_col + sbuf * kRows + half * 32 + 16, r[1]);
          tmem_wait_ld();
#pragma unroll
          for (int g2 = 0; g2 < 4; ++g2) {
            const int g = half * 4 + g2;
            const uint4 v = *reinterpret_cast<const uint4*>(smem + Sm::kOffSx + (g * 128 + h) * 16);
            const uint32_t pv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int col = g2 * 8 + 2 * i;
              const float2 a = unpack_f16x2(pack_f16x2(__uint_as_float(r[col >> 4][col & 15]) * p.scale_log2,
                                                       __uint_as_float(r[col >> 4][(col & 15) + 1]) * p.scale_log2));
              const float2 c = unpack_f16x2(pv[i]);
              s[8 * g + 2 * i] = a.x + c.x;
              s[8 * g + 2 * i + 1] = a.y + c.y;
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&sb->s_empty[sbuf]);
        mbar_arrive_cluster(&sb->sx_free, peer);
        ++s_it;
        uint64_t valid = ((uint64_t)mt[2 * t + 1] << 32) | mt[2 * t];
        const int live = first_neg - t * kRows;            // rows past the first -1 are padding
        if (live < kRows) valid &= (1ull << live) - 1ull;

        // online softmax (base 2), lazy rescale
        float mt_ = -INFINITY;
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
          s[i] = (valid >> i & 1ull) ? s[i] : -INFINITY;
          mt_ = fmaxf(mt_, s[i]);
        }
        float alpha = 1.0f;
        const bool need = mt_ > m + 8.0f;
        if (need) {
          alpha = fast_exp2(m - mt_);   // 0 when m is -inf
          m = mt_;
        }
        float psum = 0.0f;
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
          s[i] = (valid >> i & 1ull) ? fast_exp2(s[i] - m) : 0.0f;
          psum += s[i];
        }
        l = l * alpha + psum;

        const int pb = pv_it & 1;
        if (__any_sync(0xffffffffu, need && t > 0)) {
          // O holds tiles < t of this unit once P . C of tile t-1 is done: rescale it
          const int prev = pv_it - 1;
          if (!mbar_wait(&sb->p_empty[prev & 1], (uint32_t)(prev >> 1) & 1u, abort, p.status)) { ok = false; break; }
          tc_fence_after();
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
        // the P buffer of tile t-2 must have been consumed by its P . C
        if (!mbar_wait(&sb->p_empty[pb], ((uint32_t)(pv_it >> 1) & 1u) ^ 1u, abort, p.status)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(s[32 * half + 2 * i], s[32 * half + 2 * i + 1]);
          tmem_st16(lane_addr + p_col + pb * (kRows / 2) + 16 * half, w);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sb->p_full[pb]);
      }
      if (!ok) break;
      mbar_arrive(&sb->tab_free[buf]);
      // ---- unit epilogue: normalise O and write it out
      if (!mbar_wait(&sb->o_full, (uint32_t)u_it & 1u, abort, p.status)) { ok = false; break; }
      tc_fence_after();
      const bool any = ntiles > 0 && l > 0.0f;
      const float inv = any ? 1.0f / l : 0.0f;
      const float lse = any ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
      const bool real_head = h < p.H;
      if (p.splits == 1) {
        uint16_t* orow = p.out + ((long long)bj * p.H + h) * p.DL + rank * Lay::kPvN;
#pragma unroll 1
        for (int c = 0; c < Lay::kPvN; c += 16) {
          uint32_t r[16];
          if (ntiles > 0) {
            tmem_ld16(lane_addr + o_col + c, r);
            tmem_wait_ld();
          }
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            w[i] = ntiles > 0 ? pack_bf16x2(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv) : 0u;
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
          if (ntiles > 0) {
            tmem_ld16(lane_addr + o_col + c, r);
            tmem_wait_ld();
          }
          if (real_head) {
            float4* dst = reinterpret_cast<float4*>(orow + c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = ntiles > 0 ? make_float4(__uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
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
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Lay::kTmemCols);
  }
}

// Log-sum-exp merge of the per-split partial results: one CTA per (query row, head), each
// thread 4 output dims.
__global__ void __launch_bounds__(128) combine_kernel(const CombineKernelParams p) {
  pdl_wait_primary();
  const long long bjh = blockIdx.x;            // = bj * H + h
  const int d4 = threadIdx.x * 4;
  if (d4 < p.DL) {
    const long long stride_lse = (long long)p.BJ * p.H;
    float mx = -INFINITY;
    for (int s = 0; s < p.splits; ++s) mx = fmaxf(mx, p.part_lse[s * stride_lse + bjh]);
    float wsum = 0.0f, o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
    if (mx != -INFINITY) {
      for (int s = 0; s < p.splits; ++s) {
        const float ls = p.part_lse[s * stride_lse + bjh];
        const float wgt = ls == -INFINITY ? 0.0f : expf(ls - mx);
        const float4 v = *reinterpret_cast<const float4*>(p.part_o + (s * stride_lse + bjh) * p.DL + d4);
        o0 += wgt * v.x;
        o1 += wgt * v.y;
        o2 += wgt * v.z;
        o3 += wgt * v.w;
        wsum += wgt;
      }
    }
    const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
    uint16_t* dst = p.out + bjh * p.DL + d4;
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(o0 * inv, o1 * inv), pack_bf16x2(o2 * inv, o3 * inv));
    if (d4 == 0 && p.lse) p.lse[bjh] = wsum > 0.0f ? mx + logf(wsum) : -INFINITY;
  }
  pdl_launch_dependents();
}

template <int DL, int DR>
cudaError_t launch_attend_impl(const AttnKernelParams& p, const CUtensorMap* maps, int n_clusters,
                               bool pdl, cudaStream_t stream) {
  using Sm = AttnSmem<AttnLayout<DL, DR>>;
  {
    // the warpgroup register split assumes the launch allocation kLaunchRegs per thread
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, sparse_attend_kernel<DL, DR>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  }
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
  cfg.gridDim = dim3((unsigned)((long long)p.BJ * p.H), 1, 1);
  cfg.blockDim = dim3(128, 1, 1);
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
