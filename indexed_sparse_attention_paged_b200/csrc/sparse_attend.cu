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
// OF TWO CTAs shares each piece of work:
//   - CTA r owns output dims [r*DL/2, (r+1)*DL/2) and gathers only its half of each latent row
//     (plus half of the rope dims), so together the pair reads each 1152-byte row once;
//   - each CTA computes a partial S = Q_r . C_r^T over its own dims, with its latent half of Q
//     held in TMEM (the A operand of the MMA) and only the rope part of Q in shared memory;
//   - the partials cross to the peer through distributed shared memory as int16 with one
//     power-of-two scale per head and half tile, and each CTA adds the peer's decoded partial
//     to its own exact fp32 one (read straight from TMEM);
//   - P (bf16) is written to a 128B-swizzled shared buffer and is the A operand of
//     O_r += P . C_r.
// Warp roles (576 threads): two softmax warpgroups (warps 0-3 and 4-7; each owns 32 of a tile's
// 64 rows for all heads, and does that half's logit exchange, its part of the q load into TMEM
// and half of the output columns), the row gather (8-15), the S = Q C^T issuer (16) and the
// P . C issuer (17); setmaxnreg splits the registers between them.  Rows are gathered with
// 16-byte cp.async from a per-unit table of physical cache rows into swizzled K-major tiles (four
// latent stages, a separate two-slot rope ring); the same tile serves as the K-major B operand
// of Q.C^T and as the MN-major B operand of P.C.  Rescaling of O is lazy: only when a head's
// running max grows by more than 2^8.  The (query, 64-row tile) work is split evenly over all CTA
// pairs; queries that straddle a pair boundary are computed in pieces (normalised bf16 partials
// and log-sum-exps) that combine_kernel merges.  Every pipeline wait is an mbarrier wait with a
// bounded spin.
#include <cuda.h>
#include <cuda_fp16.h>

#include <type_traits>
#include <cuda_runtime.h>

#include "sia_internal.h"
#include "sia_ptx.cuh"

namespace sia {
namespace {

constexpr int kProducerWarps = 8;   // cp.async gather (+ TMA for the rope part of q)
constexpr int kFirstProducerWarp = 8;
constexpr int kMmaWarp = 16;    // S = Q . C^T issuer (and TMEM owner)
constexpr int kPvWarp = 17;     // O += P . C issuer
// warps 0-3 softmax, 4-7 partial-logit exchange (both also load q and write the output), 8-15
// gather, 16 S = Q . C^T issuer, 17 O += P . C issuer
constexpr int kAttnThreads = 576;
// Registers per thread after the split.  The block is launched with kLaunchRegs x 576
// registers (ptxas' allocation for 576 threads); the softmax warpgroup takes kSoftmaxRegs (a
// tile's 64 fp32 logits per thread plus the rescale of O), the exchange warpgroup kExchangeRegs
// (a tile's 64 partials per thread), the two gather warpgroups give back down to kGatherRegs and
// the two MMA warps keep the launch value.  The sum stays within the launch allocation, so
// setmaxnreg.inc never waits for registers that are not there.
constexpr int kLaunchRegs = 96;
constexpr int kSoftmaxRegs = 152;
constexpr int kExchangeRegs = 104;
constexpr int kGatherRegs = 64;
static_assert(128 * kSoftmaxRegs + 128 * kExchangeRegs + 256 * kGatherRegs + 64 * kLaunchRegs <=
                  kAttnThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
// setmaxnreg.inc may only raise a warp's count and setmaxnreg.dec only lower it
static_assert(kSoftmaxRegs >= kLaunchRegs && kExchangeRegs >= kLaunchRegs && kGatherRegs <= kLaunchRegs,
              "the softmax and exchange warpgroups grow, the gather warpgroups shrink");
constexpr int kStages = 3;          // latent-row tiles in flight per CTA
constexpr int kRopeSlots = 2;       // their rope parts (read by S = Q . C^T only) in flight
constexpr int kRows = kAttnTileRows;

template <int DL, int DR>
struct AttnLayout;

// Per-CTA share of each latent row: CTA r gathers latent dims [DL/2 r, DL/2 (r+1)) (used by both
// Q.C^T and P.C) and a share of the rope dims (used by Q.C^T only).
template <>
struct AttnLayout<512, 64> {
  static constexpr int kLatDims = 256;    // latent dims per CTA (q part held in TMEM)
  static constexpr int kLatBlocks = 4;    // 4 x 64 latent dims per CTA, 128-byte swizzled rows
  static constexpr int kLatKbw = 128;
  static constexpr int kRopeKbw = 64;     // 32 rope dims per CTA, 64-byte swizzled rows
  static constexpr int kPvN = 256;
  static constexpr uint32_t kTmemCols = 512;
  __device__ static bool has_rope(int) { return true; }
  __device__ static int rope_x(int r) { return 512 + 32 * r; }
  static constexpr int kChunks0 = 36, kChunks1 = 36;                      // 16-byte pieces per row
  static constexpr int kLatChunks = 32;                                   // the first 32 are latent
  __device__ static int chunk_src(int r, int k) { return k < 32 ? 512 * r + 16 * k : 1024 + 64 * r + 16 * (k - 32); }
  // offset inside the latent stage (k < kLatChunks) or inside the rope slot
  __device__ static uint32_t chunk_dst(int row, int k) {
    return k < 32 ? (uint32_t)(k >> 3) * (kAttnTileRows * 128) + swizzled_offset(row, (k & 7) * 16, 128)
                  : swizzled_offset(row, (k - 32) * 16, 64);
  }
  // FP8 main cache (one byte per element, one fp32 scale per 128-element block of the row):
  // CTA r's 16-element code pieces are 16 latent ones from element 256 r and 2 rope ones from
  // element 512 + 32 r (a piece's scale is that of block element / 128 of the row)
  static constexpr int kLatPieces8 = 16, kMaxRopePieces8 = 2, kRopeCodeBytes = 32;
  __device__ static int rope_pieces8(int) { return 2; }
  __device__ static int piece_src8(int r, int k) { return k < 16 ? 256 * r + 16 * k : 512 + 32 * r + 16 * (k - 16); }
};

template <>
struct AttnLayout<64, 16> {
  static constexpr int kLatDims = 32;
  static constexpr int kLatBlocks = 1;    // 32 latent dims per CTA, 64-byte swizzled rows
  static constexpr int kLatKbw = 64;
  static constexpr int kRopeKbw = 32;     // all 16 rope dims on CTA 0, 32-byte swizzled rows
  static constexpr int kPvN = 32;
  static constexpr uint32_t kTmemCols = 256;
  __device__ static bool has_rope(int r) { return r == 0; }
  __device__ static int rope_x(int) { return 64; }
  static constexpr int kChunks0 = 6, kChunks1 = 4;
  static constexpr int kLatChunks = 4;
  __device__ static int chunk_src(int r, int k) { return k < 4 ? 64 * r + 16 * k : 128 + 16 * (k - 4); }
  __device__ static uint32_t chunk_dst(int row, int k) {
    return k < 4 ? swizzled_offset(row, k * 16, 64) : swizzled_offset(row, (k - 4) * 16, 32);
  }
  // FP8 main cache: 2 latent code pieces from element 32 r, and CTA 0's one rope piece (element
  // 64); the 80-element row is one scale block
  static constexpr int kLatPieces8 = 2, kMaxRopePieces8 = 1, kRopeCodeBytes = 16;
  __device__ static int rope_pieces8(int r) { return r == 0 ? 1 : 0; }
  __device__ static int piece_src8(int r, int k) { return k < 2 ? 32 * r + 16 * k : 64; }
};

// TMEM columns: O [0, kPvN), two logit buffers of kRows fp32 columns, then the CTA's latent
// half of q as bf16 pairs (the A operand of Q . C^T).
template <class Lay>
struct AttnTmem {
  static constexpr uint32_t kO = 0;
  static constexpr uint32_t kS = Lay::kPvN;
  static constexpr uint32_t kQ = kS + 2 * kRows;
  static_assert(kQ + Lay::kLatDims / 2 <= Lay::kTmemCols, "TMEM columns overflow");
};

struct AttnMaps {
  CUtensorMap q_rope;
};

template <class Lay>
struct AttnSmem {
  static constexpr uint32_t kQRopeBytes = 128 * Lay::kRopeKbw;
  static constexpr uint32_t kCLatBytes = kRows * Lay::kLatKbw;       // one latent block of a tile
  static constexpr uint32_t kCStageBytes = Lay::kLatBlocks * kCLatBytes;
  static constexpr uint32_t kCRopeBytes = kRows * Lay::kRopeKbw;     // one rope slot
  static constexpr uint32_t kOffQ = 0;                                  // rope part of q only
  static constexpr uint32_t kOffC = (kOffQ + kQRopeBytes + 1023u) & ~1023u;
  static constexpr uint32_t kOffR = kOffC + kStages * kCStageBytes;

  // Partial-logit exchange, one block per tile: 64 rows x 128 heads of int16 codes ([row / 8]
  // [head] in 16-byte groups of 8 rows), then the 128 heads' power-of-two scale exponents
  // (int32).  Sx holds the blocks the peer copies in and the stash this CTA's own blocks, two
  // tiles each (by tile parity); a stash block is read by this CTA's softmax and is the source of
  // the copy to the peer.
  static constexpr uint32_t kSxCodes = kRows * 128 * 2;
  static constexpr uint32_t kSxBlock = kSxCodes + 128 * 4;
  // P (bf16, 128 heads x kRows, 128B-swizzled K-major): the A operand of P . C
  static constexpr uint32_t kOffP = (kOffR + kRopeSlots * kCRopeBytes + 1023u) & ~1023u;
  static constexpr uint32_t kOffSx = kOffP + 128 * kRows * 2;
  static constexpr uint32_t kOffStash = kOffSx + 2 * kSxBlock;
  // each head's sum and max of the softmax (read by the other warpgroup at a unit's end)
  static constexpr uint32_t kOffL = kOffStash + 2 * kSxBlock;
  // the physical cache row of each Top-K entry of the unit being gathered (read by the gather
  // threads only, which rebuild it between units), then per unit (double-buffered) the validity
  // bits and each gather warp's lowest position of a -1 entry
  static constexpr uint32_t kOffRows = kOffL + 2 * 128 * 4;
  static constexpr uint32_t kOffMask = kOffRows + kAttnMaxSplitRows * 4;
  static constexpr uint32_t kOffFirstNeg = kOffMask + 2 * (kAttnMaxSplitRows / 8);
  static constexpr uint32_t kOffBar = kOffFirstNeg + 2 * kProducerWarps * 4;
  static constexpr uint32_t kBarBytes = 512;
  static constexpr uint32_t kBytes = kOffBar + kBarBytes;
  static_assert(kOffP % 1024 == 0, "P must sit on a 1024-byte swizzle atom");
  static_assert(kSxBlock % 16 == 0 && kOffSx % 16 == 0 && kOffStash % 16 == 0, "bulk copies move 16-byte units");
  static_assert(kSxBlock >= 4 * 4096, "an exchange block also stages one warpgroup's output slices");
  static_assert(kBytes <= 232448, "shared memory over the 227 KB a CTA may opt into");
};

struct AttnBarriers {
  uint64_t c_full[kStages], c_empty[kStages];   // a tile's rows landed / latent stage free
  uint64_t r_empty[kRopeSlots];                 // rope slot free (its S = Q . C^T done)
  uint64_t s_full[2], s_empty[2];   // partial logits in TMEM / read by the exchange warps
  uint64_t stash_full[2], own_free[2];  // own block stashed / decoded by the softmax and copied
  uint64_t p_full;                  // all softmax threads wrote P (waited by the P . C issuer)
  uint64_t p_empty;                 // P . C of the previous tile done (P buffer and O free)
  uint64_t epi_sync;                // all softmax threads are past the unit's last tile
  uint64_t q_full, q_empty;       // q in TMEM written by the 128 loader threads / q reusable
  uint64_t q_tma;                 // the rope part of q landed (TMA bytes only)
  uint64_t o_full;
  uint64_t sx_ready[2], sx_free[2];  // [tile parity]: the peer's block landed / was decoded
  uint64_t g_sync;                          // every gather thread issued the unit's tiles
  uint64_t tab_full[2], tab_free[2];
  uint64_t mma_done, pv_done;
  uint64_t g_loaded[2];             // FP8 cache: every gather thread read its staged codes
  uint32_t tmem_base;
  int abort;
};

static_assert(sizeof(AttnBarriers) <= 512, "barrier block outgrew its shared-memory slot");

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The partial logits cross to the peer CTA as 16-bit integers with one power-of-two scale per
// head and tile: x = round(v 2^e), |x| < 2^14.  fma(v, 2^e, kMagic) puts x + 2^15 in the low 16
// bits of an fp32 in [2^23, 2^24) (where the spacing is 1, so the rounding is to the nearest
// integer), and the receiver rebuilds 2^23 + x + 2^15 from those bits and removes kMagic exactly.
constexpr float kMagic = 8421376.0f;   // 2^23 + 2^15

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ void cp_async16_hint(uint32_t dst, const void* src, uint64_t policy) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "l"(policy)
               : "memory");
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// The work of a call is the flat list of (query, 64-row tile) pairs, query-major with
// tiles_per_q <= 32 tiles per query, divided between the CTA pairs (AttnSplit): pair c takes
// global tiles [start(c), start(c + 1)).  A unit is the part of that range inside one query.  A query
// covered by one unit gets its output written directly; a query that straddles a pair
// boundary is computed in pieces, each written as a partial result (normalised O and the
// log-sum-exp of each CTA of the pair) into a record of the workspace, and combine_kernel
// merges them.  Only a pair's first and last unit can be pieces, so pair c owns records 2c
// (its first unit) and 2c + 1 (its last unit, when that is another unit).

struct AttnUnit {
  int bj;        // query row (b * J + j)
  int row0;      // first Top-K entry of the unit
  int nrows;     // entries in the unit (rows of the last tile may be absent)
  int rec;       // partial-result record, or -1 when the unit writes the final output
};

struct AttnRange {
  long long g0, g1;   // this pair's global tiles
};

// Next unit of the pair from global tile `cursor` (advanced past the unit); false when done.
__device__ __forceinline__ bool attn_next_unit(const AttnKernelParams& p, int c, const AttnRange& rg,
                                               long long& cursor, AttnUnit& u) {
  if (cursor >= rg.g1) return false;
  const int TQ = p.tiles_per_q;
  u.bj = (int)cursor / TQ;   // G < 2^31
  const long long q0 = (long long)u.bj * TQ;
  const long long tb = min(rg.g1, q0 + TQ);
  u.row0 = (int)(cursor - q0) * kAttnTileRows;
  u.nrows = min(p.K, (int)(tb - q0) * kAttnTileRows) - u.row0;
  const bool piece = q0 < rg.g0 || q0 + TQ > rg.g1;
  u.rec = piece ? 2 * c + (cursor == rg.g0 ? 0 : 1) : -1;
  cursor = tb;
  return true;
}

// e4m3x2 (two codes in the low 16 bits) -> two fp32, exactly (through f16x2)
__device__ __forceinline__ void e4m3x2_to_f32(uint32_t codes, float& lo, float& hi) {
  uint32_t h2;
  asm("{\n\t.reg .b16 c;\n\tcvt.u16.u32 c, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, c;\n\t}" : "=r"(h2) : "r"(codes));
  asm("{\n\t.reg .b16 l16, h16;\n\tmov.b32 {l16, h16}, %2;\n\tcvt.f32.f16 %0, l16;\n\tcvt.f32.f16 %1, h16;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(h2));
}

__device__ __forceinline__ void cp_async4_hint(uint32_t dst, const void* src, uint64_t policy) {
  asm volatile("cp.async.ca.shared.global.L2::cache_hint [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "l"(policy)
               : "memory");
}

template <int DL, int DR, bool KV8>
__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attend_kernel(const __grid_constant__ AttnMaps maps, const AttnKernelParams p) {
  static_assert(kAttnThreads == 576, "role layout assumes 18 warps");
  using Lay = AttnLayout<DL, DR>;
  using Sm = AttnSmem<Lay>;
  using Tm = AttnTmem<Lay>;
  extern __shared__ __align__(1024) uint8_t smem[];
  AttnBarriers* sb = reinterpret_cast<AttnBarriers*>(smem + Sm::kOffBar);
  int32_t* rows_tab = reinterpret_cast<int32_t*>(smem + Sm::kOffRows);        // [max rows]
  uint32_t* mask_tab = reinterpret_cast<uint32_t*>(smem + Sm::kOffMask);      // [2][max rows/32]
  int32_t* fneg_tab = reinterpret_cast<int32_t*>(smem + Sm::kOffFirstNeg);    // [2][gather warps]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int cluster_id = blockIdx.x >> 1;
  const bool rope = Lay::has_rope((int)rank);
  const int DC = p.DL + p.DR;

  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) report(p.status, SIA_DEV_INTERNAL);
    return;  // both CTAs of the pair see the same base alignment and leave together
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sb->c_full[s], kProducerWarps * 32);  // one cp.async completion per gather thread
      mbar_init(&sb->c_empty[s], 1);
    }
    for (int s = 0; s < kRopeSlots; ++s) mbar_init(&sb->r_empty[s], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sb->s_full[s], 1);
      mbar_init(&sb->s_empty[s], 4);           // the 4 exchange warps (one arrival per warp)
      mbar_init(&sb->stash_full[s], 4);        // the 4 exchange warps
      mbar_init(&sb->own_free[s], 4 + 1);      // the 4 softmax warps and the copy's issuer
      mbar_init(&sb->tab_full[s], kProducerWarps);
      mbar_init(&sb->tab_free[s], 8 + 2);     // the softmax warps and both MMA threads
    }
    mbar_init(&sb->p_full, 4);
    mbar_init(&sb->p_empty, 1);
    mbar_init(&sb->epi_sync, 8);
    mbar_init(&sb->q_full, 8);         // the 8 warps writing q into TMEM
    mbar_init(&sb->q_tma, 1);          // the rope TMA (or a plain arrive when this CTA has none)
    mbar_init(&sb->q_empty, 1);
    mbar_init(&sb->o_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sb->sx_ready[s], 1);   // the peer's copy: its issuer's arrive + the bytes
      mbar_init(&sb->sx_free[s], 4);    // the peer's 4 softmax warps
    }
    mbar_init(&sb->g_sync, kProducerWarps);
    mbar_init(&sb->mma_done, 1);
    mbar_init(&sb->pv_done, 1);
    mbar_init(&sb->g_loaded[0], kProducerWarps);
    mbar_init(&sb->g_loaded[1], kProducerWarps);
    sb->abort = 0;
    fence_mbarrier_init();
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
  const WaitCtl wc{abort, p.status, p.wait_ns};
  // The next kernel (the split merge, or the next call's first kernel) waits for this grid's
  // completion before its loads, so it may be scheduled now and only its launch overlaps ours.
  pdl_launch_dependents();

  // Only the gather warps read what the previous kernel on the stream (Top-K) writes; they wait
  // for it below.  The query rows are inputs written before the previous kernels were launched.

  // number of 64-row tiles of unit buffer `buf`: rows up to the first -1 entry of the list
  auto unit_tiles = [&](int buf) {
    int first_neg = 1 << 30;
#pragma unroll
    for (int w = 0; w < kProducerWarps; ++w) first_neg = min(first_neg, fneg_tab[buf * kProducerWarps + w]);
    return first_neg;
  };

  if (warp >= kFirstProducerWarp && warp < kFirstProducerWarp + kProducerWarps) {
    // ---------------------------------------------------------------- gather (8 warps)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kGatherRegs));
    const int ptid = threadIdx.x - kFirstProducerWarp * 32;   // 0..255
    const int pwarp = warp - kFirstProducerWarp;
    const uint8_t* kv = static_cast<const uint8_t*>(p.kv);
    // One tile of gathers: consecutive threads take consecutive 16-byte pieces of a row, so a
    // warp reads whole 512-byte runs of a latent row at a time.  A thread's pieces are the same
    // for every tile, so their row, source offset and destination (latent stage or rope slot)
    // are packed once: row [0,6), source/16 [6,13), rope flag 13, destination/16 [14,26), and
    // bit 26 when the piece exists.
    // latent rows are read once per call: evict them first, so the split partials this kernel
    // writes stay in L2 for the merge
    const uint64_t stream_policy = l2_evict_first_policy();
    const int nch = rank == 0 ? Lay::kChunks0 : Lay::kChunks1;
    constexpr int kPer = (kRows * (Lay::kChunks0 > Lay::kChunks1 ? Lay::kChunks0 : Lay::kChunks1) +
                          kProducerWarps * 32 - 1) / (kProducerWarps * 32);
    uint32_t piece[kPer];
    auto make_pieces = [&]() {
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = ptid + j * kProducerWarps * 32;
        const int row = i / nch, k = i - row * nch;
        const bool lat = k < Lay::kLatChunks;
        piece[j] = i < kRows * nch
                       ? (uint32_t)row | ((uint32_t)Lay::chunk_src((int)rank, k) / 16u) << 6 | (lat ? 0u : 1u) << 13 |
                             (Lay::chunk_dst(row, k) / 16u) << 14 | 1u << 26
                       : 0u;
      }
    };
    auto gather_tile = [&](uint32_t lat_base, uint32_t rope_base, const int32_t* rows) {
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const uint32_t pc = piece[j];
        if (pc >> 26) {
          const uint8_t* src = kv + (size_t)(uint32_t)rows[pc & 63u] * (DC * 2) + ((pc >> 6) & 127u) * 16u;
          cp_async16_hint(((pc >> 13) & 1u ? rope_base : lat_base) + ((pc >> 14) & 4095u) * 16u, src, stream_policy);
        }
      }
    };
    int it = 0, u_it = 0, q_issued = 0;
    bool ok = true;
    bool waited = false;
    const AttnRange rg{attn_pair_start(p.split, cluster_id), attn_pair_start(p.split, cluster_id + 1)};
    long long cursor = rg.g0;
    AttnUnit un;
    // Touch every cache page of sequence b (one line of this CTA's half per page): the address
    // translations and the page-table row are then warm when the unit's rows are gathered.  A
    // unit that started on cold translations waited microseconds for its first tile.
    auto touch_pages = [&](int b) {
      const int L = p.seq_lens[b];
      const int npages = min(p.max_pages, (L + p.P - 1) / p.P);
      const int32_t* pt_row = p.page_table + (long long)b * p.max_pages;
      for (int i = ptid; i < npages; i += kProducerWarps * 32) {
        const int pg = pt_row[i];
        if (pg >= 0 && pg < p.num_pages)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(kv + ((size_t)pg * p.P * DC + (size_t)rank * (p.DL / 2)) * (KV8 ? 1 : 2)));
      }
    };
    // while the previous kernel still runs: the sequences of all of this pair's units, and the
    // latent half of their query rows that this CTA loads into TMEM at each unit's start
    if (cursor < rg.g1) {
      const int bj_lo = (int)(rg.g0 / p.tiles_per_q), bj_hi = (int)((rg.g1 - 1) / p.tiles_per_q);
      for (int b = bj_lo / p.J; b <= bj_hi / p.J; ++b) touch_pages(b);
      constexpr int kLines = Lay::kLatDims * 2 >= 128 ? Lay::kLatDims * 2 / 128 : 1;   // 128-byte lines per head row
      for (int bj = bj_lo; bj <= bj_hi; ++bj)
        for (int i = ptid; i < p.H * kLines; i += kProducerWarps * 32)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const uint8_t*>(p.q) +
                                                        ((size_t)bj * p.H + i / kLines) * (DC * 2) +
                                                        (size_t)rank * Lay::kLatDims * 2 + (i % kLines) * 128));
    }
    while (ok && attn_next_unit(p, cluster_id, rg, cursor, un)) {
      const int bj = un.bj;
      const int b = bj / p.J;
      const int L = p.seq_lens[b];
      const long long row_base = (long long)bj * p.K;
      const int row0 = un.row0;
      const int nrows = un.nrows;
      const int nrows_pad = (nrows + kRows - 1) / kRows * kRows;
      const int buf = u_it & 1;
      // rope part of the query rows of all heads (TMA; independent of the Top-K list)
      if (ptid == 0) {
        if (mbar_wait(&sb->q_empty, ((uint32_t)u_it & 1u) ^ 1u, wc)) {
          if (rope) {
            mbar_arrive_expect_tx(&sb->q_tma, Sm::kQRopeBytes);
            tma_load_2d(smem + Sm::kOffQ, &maps.q_rope, &sb->q_tma, Lay::rope_x((int)rank), bj * p.H);
          } else {
            mbar_arrive(&sb->q_tma);
          }
          ++q_issued;
        }
      }
      if (!waited) {
        pdl_wait_primary();  // the Top-K lists come from the previous kernel on the stream
        waited = true;
      }
      // resolve this unit's Top-K entries to physical cache rows: 8 entries per thread, all
      // loads of a thread in flight at once
      if (!mbar_wait_warp(&sb->tab_free[buf], ((uint32_t)(u_it >> 1) & 1u) ^ 1u, wc)) { ok = false; break; }
      int32_t* rt = rows_tab;
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
      // the row table is rewritten once every gather thread has issued the previous unit's tiles
      if (u_it > 0 && !mbar_wait_warp(&sb->g_sync, (uint32_t)(u_it - 1) & 1u, wc)) { ok = false; break; }
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
      mbar_arrive_warp(&sb->tab_full[buf]);
      if (!mbar_wait_warp(&sb->tab_full[buf], (uint32_t)(u_it >> 1) & 1u, wc)) { ok = false; break; }
      const int ntiles = (unit_tiles(buf) + kRows - 1) / kRows;
      if constexpr (!KV8) {
        make_pieces();   // (after the table: the two never hold registers at the same time)
        for (int t = 0; t < ntiles; ++t, ++it) {
          const int stage = it % kStages, rslot = it % kRopeSlots;
          if (!mbar_wait_warp(&sb->c_empty[stage], ((uint32_t)(it / kStages) & 1u) ^ 1u, wc)) { ok = false; break; }
          if (!mbar_wait_warp(&sb->r_empty[rslot], ((uint32_t)(it / kRopeSlots) & 1u) ^ 1u, wc)) { ok = false; break; }
          gather_tile(smem_u32(smem + Sm::kOffC + stage * Sm::kCStageBytes),
                      smem_u32(smem + Sm::kOffR + rslot * Sm::kCRopeBytes), rt + t * kRows);
          asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&sb->c_full[stage])) : "memory");
        }
      } else {
        // FP8 main cache ("Rapid Adaptation and Inference Optimization", tiered quantisation
        // table: FP8 with one scale per 128-element block of the row).  Tile t's e4m3 codes land
        // by cp.async in the upper half of its own latent stage and rope slot, and the scale of
        // each of this thread's pieces in a slot of the thread's own at the start of the latent
        // stage.  One tile later, once this thread's copies of tile t are complete, it reads its
        // codes and scales, every gather thread agrees that the staging has been read
        // (g_loaded), and each writes its pieces as bf16 (code x scale, rounded once) into the
        // swizzled K-major layout the MMAs read.
        const int npr = Lay::kLatPieces8 + Lay::rope_pieces8((int)rank);
        constexpr int kP8 = (kRows * (Lay::kLatPieces8 + Lay::kMaxRopePieces8) + kProducerWarps * 32 - 1) /
                            (kProducerWarps * 32);
        static_assert((kProducerWarps * 32) * kP8 * 4 <= Sm::kCStageBytes / 2, "scale slots overflow the stage");
        const uint8_t* kv8 = static_cast<const uint8_t*>(p.kv);
        auto staged = [&](int row, int k, uint32_t lat_base, uint32_t rope_base) -> uint32_t {
          return k < Lay::kLatPieces8 ? lat_base + Sm::kCStageBytes / 2 + row * (Lay::kLatPieces8 * 16) + 16 * k
                                      : rope_base + Sm::kCRopeBytes / 2 + row * Lay::kRopeCodeBytes + 16 * (k - Lay::kLatPieces8);
        };
        auto issue8 = [&](uint32_t lat_base, uint32_t rope_base, const int32_t* rows) {
#pragma unroll
          for (int j = 0; j < kP8; ++j) {
            const int i = ptid + j * kProducerWarps * 32;
            if (i < kRows * npr) {
              const int row = i / npr, k = i - (i / npr) * npr;
              const uint32_t pr = (uint32_t)rows[row];
              const int src = Lay::piece_src8((int)rank, k);
              cp_async16_hint(staged(row, k, lat_base, rope_base), kv8 + (size_t)pr * DC + src, stream_policy);
              cp_async4_hint(lat_base + (uint32_t)(ptid * kP8 + j) * 4u,
                             p.kv_scale + (size_t)pr * p.nblk + src / 128, stream_policy);
            }
          }
          asm volatile("cp.async.commit_group;" ::: "memory");
        };
        auto convert8 = [&](int stage, int rslot, int it_) -> bool {
          const uint32_t lat_base = smem_u32(smem + Sm::kOffC + stage * Sm::kCStageBytes);
          const uint32_t rope_base = smem_u32(smem + Sm::kOffR + rslot * Sm::kCRopeBytes);
          uint4 code[kP8];
          float sc[kP8];
#pragma unroll
          for (int j = 0; j < kP8; ++j) {
            const int i = ptid + j * kProducerWarps * 32;
            code[j] = make_uint4(0, 0, 0, 0);
            sc[j] = 0.0f;
            if (i < kRows * npr) {
              const int row = i / npr, k = i - (i / npr) * npr;
              asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(code[j].x), "=r"(code[j].y), "=r"(code[j].z), "=r"(code[j].w)
                           : "r"(staged(row, k, lat_base, rope_base)));
              asm volatile("ld.shared.f32 %0, [%1];" : "=f"(sc[j]) : "r"(lat_base + (uint32_t)(ptid * kP8 + j) * 4u));
            }
          }
          mbar_arrive_warp(&sb->g_loaded[it_ & 1]);
          if (!mbar_wait_warp(&sb->g_loaded[it_ & 1], (uint32_t)(it_ >> 1) & 1u, wc)) return false;
#pragma unroll
          for (int j = 0; j < kP8; ++j) {
            const int i = ptid + j * kProducerWarps * 32;
            if (i < kRows * npr) {
              const int row = i / npr, k = i - (i / npr) * npr;
              const uint32_t cw[4] = {code[j].x, code[j].y, code[j].z, code[j].w};
              uint32_t o[8];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                float a, b, c, d;
                e4m3x2_to_f32(cw[q] & 0xffffu, a, b);
                e4m3x2_to_f32(cw[q] >> 16, c, d);
                o[2 * q] = pack_bf16x2(a * sc[j], b * sc[j]);
                o[2 * q + 1] = pack_bf16x2(c * sc[j], d * sc[j]);
              }
              const bool lat = k < Lay::kLatPieces8;
              const uint32_t base = lat ? lat_base : rope_base;
              const int c0 = lat ? 2 * k : Lay::kLatChunks + 2 * (k - Lay::kLatPieces8);
              st_shared_v4(base + Lay::chunk_dst(row, c0), o[0], o[1], o[2], o[3]);
              st_shared_v4(base + Lay::chunk_dst(row, c0 + 1), o[4], o[5], o[6], o[7]);
            }
          }
          fence_proxy_async_smem();   // the MMAs read the stage through the async proxy
          mbar_arrive(&sb->c_full[stage]);
          return true;
        };
        int prev_stage = 0, prev_rslot = 0;
        for (int t = 0; t < ntiles; ++t, ++it) {
          const int stage = it % kStages, rslot = it % kRopeSlots;
          if (!mbar_wait_warp(&sb->c_empty[stage], ((uint32_t)(it / kStages) & 1u) ^ 1u, wc)) { ok = false; break; }
          if (!mbar_wait_warp(&sb->r_empty[rslot], ((uint32_t)(it / kRopeSlots) & 1u) ^ 1u, wc)) { ok = false; break; }
          issue8(smem_u32(smem + Sm::kOffC + stage * Sm::kCStageBytes),
                 smem_u32(smem + Sm::kOffR + rslot * Sm::kCRopeBytes), rt + t * kRows);
          if (t > 0) {
            asm volatile("cp.async.wait_group 1;" ::: "memory");   // this thread's copies of tile t-1
            if (!convert8(prev_stage, prev_rslot, it - 1)) { ok = false; break; }
          }
          prev_stage = stage;
          prev_rslot = rslot;
        }
        if (!ok) break;
        if (ntiles > 0) {
          asm volatile("cp.async.wait_group 0;" ::: "memory");
          if (!convert8(prev_stage, prev_rslot, it - 1)) { ok = false; break; }
        }
      }
      if (!ok) break;
      mbar_arrive_warp(&sb->g_sync);   // this warp is done with the row table
      ++u_it;
    }
    // our copies have landed before we may leave, whether or not the CTA is aborting: every
    // cp.async of this thread, and the rope TMA of the last unit (one unit's q at a time: the
    // next is only issued once the products of this one are done)
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (ptid == 0 && q_issued > 0) mbar_drain(&sb->q_tma, (uint32_t)(q_issued - 1) & 1u, p.status);
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- S = Q . C^T issuer
    // (O += P . C has its own issuing warp, so a logit tile never waits for P of an earlier
    // tile and P never waits for a logit tile being issued)
    if (lane == 0) {
      const uint32_t idesc_qk = umma_idesc(1, 1, false, false, kRows, 128);
      const uint32_t qr_base = smem_u32(smem + Sm::kOffQ);
      int it = 0, u_it = 0;
      bool ok = true;
      const AttnRange rg{attn_pair_start(p.split, cluster_id), attn_pair_start(p.split, cluster_id + 1)};
    long long cursor = rg.g0;
      AttnUnit un;
      for (; ok && attn_next_unit(p, cluster_id, rg, cursor, un); ++u_it) {
        const int buf = u_it & 1;
        if (!mbar_wait(&sb->tab_full[buf], (uint32_t)(u_it >> 1) & 1u, wc)) { ok = false; break; }
        const int ntiles = (unit_tiles(buf) + kRows - 1) / kRows;
        mbar_arrive(&sb->tab_free[buf]);
        if (!mbar_wait(&sb->q_full, (uint32_t)u_it & 1u, wc)) { ok = false; break; }
        if (!mbar_wait(&sb->q_tma, (uint32_t)u_it & 1u, wc)) { ok = false; break; }
        tc_fence_after();
        for (int t = 0; t < ntiles; ++t, ++it) {
          const int stage = it % kStages;
          const int sbuf = it & 1;
          if (!mbar_wait(&sb->c_full[stage], (uint32_t)(it / kStages) & 1u, wc)) { ok = false; break; }
          if (!mbar_wait(&sb->s_empty[sbuf], ((uint32_t)(it >> 1) & 1u) ^ 1u, wc)) { ok = false; break; }
          fence_proxy_async_smem();   // the gathered rows were written by cp.async
          tc_fence_after();
          const uint32_t c_base = smem_u32(smem + Sm::kOffC + stage * Sm::kCStageBytes);
          const uint32_t d = tmem_base + Tm::kS + (uint32_t)(sbuf * kRows);
          constexpr int kSub = Lay::kLatKbw / 32;   // 16-element K steps per swizzled block
#pragma unroll
          for (int g = 0; g < Lay::kLatDims / 16; ++g) {
            const uint64_t bd = umma_smem_desc(c_base + (g / kSub) * Sm::kCLatBytes + (g % kSub) * 32, 16,
                                               8 * Lay::kLatKbw, umma_layout_type(Lay::kLatKbw));
            umma_f16_ts(d, tmem_base + Tm::kQ + (uint32_t)(8 * g), bd, idesc_qk, g > 0);
          }
          const int rslot = it % kRopeSlots;
          if (rope) {
            const uint32_t r_base = smem_u32(smem + Sm::kOffR + rslot * Sm::kCRopeBytes);
#pragma unroll
            for (int ks = 0; ks < Lay::kRopeKbw / 32; ++ks) {
              const uint64_t ad = umma_smem_desc(qr_base + ks * 32, 16, 8 * Lay::kRopeKbw, umma_layout_type(Lay::kRopeKbw));
              const uint64_t bd = umma_smem_desc(r_base + ks * 32, 16, 8 * Lay::kRopeKbw, umma_layout_type(Lay::kRopeKbw));
              umma_f16(d, ad, bd, idesc_qk, true);
            }
          }
          umma_commit(&sb->s_full[sbuf]);
          umma_commit(&sb->r_empty[rslot]);
        }
        if (!ok) break;
        umma_commit(&sb->q_empty);  // q reusable once this unit's products are done
      }
      umma_commit(&sb->mma_done);
      mbar_drain(&sb->mma_done, 0, p.status);   // every S = Q . C^T product done
    }
    __syncwarp();
  } else if (warp == kPvWarp) {
    // ---------------------------------------------------------------- O += P . C issuer
    if (lane == 0) {
      const uint32_t idesc_pv = umma_idesc(1, 1, false, true, Lay::kPvN, 128);
      const uint32_t p_base = smem_u32(smem + Sm::kOffP);
      int it = 0, u_it = 0;
      bool ok = true;
      const AttnRange rg{attn_pair_start(p.split, cluster_id), attn_pair_start(p.split, cluster_id + 1)};
    long long cursor = rg.g0;
      AttnUnit un;
      for (; ok && attn_next_unit(p, cluster_id, rg, cursor, un); ++u_it) {
        const int buf = u_it & 1;
        if (!mbar_wait(&sb->tab_full[buf], (uint32_t)(u_it >> 1) & 1u, wc)) { ok = false; break; }
        const int ntiles = (unit_tiles(buf) + kRows - 1) / kRows;
        mbar_arrive(&sb->tab_free[buf]);
        for (int t = 0; t < ntiles; ++t, ++it) {
          if (!mbar_wait(&sb->p_full, (uint32_t)it & 1u, wc)) { ok = false; break; }
          fence_proxy_async_smem();   // the row stage (cp.async) and P (st.shared)
          tc_fence_after();
          const int stage = it % kStages;
          const uint32_t c_base = smem_u32(smem + Sm::kOffC + stage * Sm::kCStageBytes);
#pragma unroll
          for (int ks = 0; ks < kRows / 16; ++ks) {
            const uint64_t ad = umma_smem_desc(p_base + ks * 32, 16, 1024, umma_layout_type(128));
            const uint64_t bd = umma_smem_desc(c_base + ks * 16 * Lay::kLatKbw, Sm::kCLatBytes,
                                               8 * Lay::kLatKbw, umma_layout_type(Lay::kLatKbw));
            umma_f16(tmem_base + Tm::kO, ad, bd, idesc_pv, t > 0 || ks > 0);
          }
          umma_commit(&sb->c_empty[stage]);
          umma_commit(&sb->p_empty);
          if (t + 1 == ntiles) umma_commit(&sb->o_full);
        }
      }
      umma_commit(&sb->pv_done);
      mbar_drain(&sb->pv_done, 0, p.status);    // every O += P . C product done
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax + exchange
    // Two warpgroups, thread = head h = TMEM lane in both.  The exchange warpgroup (warps 4-7)
    // reads each tile's partial logits out of TMEM (the S buffer is free again at once), encodes
    // them as int16 with one power-of-two scale per head (relative error at most 2^-15 of the
    // head's largest partial in the tile) into a local stash, and bulk-copies the stash into the
    // peer CTA's buffer.  The softmax warpgroup (warps 0-3) decodes its own stash and the peer's
    // block and adds them: both CTAs add the same two values, so their logits are bit-identical.
    // Per unit both warpgroups load half of q into TMEM and write half of the output columns.
    // One copy of the warpgroups' code per role, each behind its own register count.
    auto role = [&](auto wg_c) __attribute__((always_inline)) {
    constexpr int wg = decltype(wg_c)::value;
    const int quad = warp & 3;
    const int h = quad * 32 + lane;   // head = TMEM lane
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quad * 32) << 16);
    const uint32_t sx_peer = mapa_shared(smem_u32(smem + Sm::kOffSx), peer);
    const bool leader = threadIdx.x == 128;   // issues the exchange warpgroup's bulk copies
    float* lbuf = reinterpret_cast<float*>(smem + Sm::kOffL);     // [sum, max][128]
    int s_it = 0, u_it = 0, o_it = 0, e_it = 0;
    bool ok = true;

    const AttnRange rg{attn_pair_start(p.split, cluster_id), attn_pair_start(p.split, cluster_id + 1)};
    long long cursor = rg.g0;
    AttnUnit un;
    for (; ok && attn_next_unit(p, cluster_id, rg, cursor, un); ++u_it) {
      const int bj = un.bj;
      const int buf = u_it & 1;
      {
        // q: head h's dims [rank * kLatDims, +kLatDims) as bf16 pairs, 16 columns (64 bytes) per
        // TMEM store; the warpgroups split the column groups.  All of a thread's loads are in
        // flight at once (the gather warps fetched the rows into L2 at the start).
        constexpr int kGroups = Lay::kLatDims / 32;
        constexpr int kGPer = (kGroups + 1) / 2;
        const int g_lo = wg == 0 ? 0 : kGPer, g_hi = wg == 0 ? kGPer : kGroups;
        const bool real = h < p.H;
        const size_t q_off = ((size_t)(real ? h : 0)) * (DC * 2) + (size_t)rank * Lay::kLatDims * 2;
        const uint8_t* qrow = static_cast<const uint8_t*>(p.q) + (size_t)bj * p.H * (DC * 2) + q_off;
        uint4 qv[kGPer][4];
#pragma unroll
        for (int j = 0; j < kGPer; ++j)
#pragma unroll
          for (int i = 0; i < 4; ++i)
            qv[j][i] = real && g_lo + j < g_hi ? ld_nc_v4(qrow + (g_lo + j) * 64 + 16 * i) : make_uint4(0, 0, 0, 0);
        if (!mbar_wait_warp(&sb->q_empty, ((uint32_t)u_it & 1u) ^ 1u, wc)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < kGPer; ++j) {
          if (g_lo + j < g_hi) {   // warp-uniform
            const uint32_t w[16] = {qv[j][0].x, qv[j][0].y, qv[j][0].z, qv[j][0].w, qv[j][1].x, qv[j][1].y,
                                    qv[j][1].z, qv[j][1].w, qv[j][2].x, qv[j][2].y, qv[j][2].z, qv[j][2].w,
                                    qv[j][3].x, qv[j][3].y, qv[j][3].z, qv[j][3].w};
            tmem_st16(lane_addr + Tm::kQ + (uint32_t)(16 * (g_lo + j)), w);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive_warp(&sb->q_full);
      }
      if (!mbar_wait_warp(&sb->tab_full[buf], (uint32_t)(u_it >> 1) & 1u, wc)) { ok = false; break; }
      const int first_neg = unit_tiles(buf);
      const int ntiles = (first_neg + kRows - 1) / kRows;
      const uint32_t* mt = mask_tab + buf * (kAttnMaxSplitRows / 32);
      float m = -INFINITY, l = 0.0f;   // the softmax warpgroup's running max and sum of head h
      const int it0 = s_it;
      if (wg == 1) {
        // ---- exchange warpgroup
        for (int t = 0; t < ntiles; ++t) {
          const int it = it0 + t, sb1 = it & 1;
          if (!mbar_wait_warp(&sb->s_full[sb1], (uint32_t)(it >> 1) & 1u, wc)) { ok = false; break; }
          tc_fence_after();
          uint32_t r[4][16];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld16(lane_addr + Tm::kS + sb1 * kRows + c * 16, r[c]);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive_warp(&sb->s_empty[sb1]);   // the S buffer may be refilled
          // the stash of tile it - 2 is free once the softmax decoded it and its copy to the
          // peer read it (the most recent copy, tile it - 1's, may still be in flight)
          if (it >= 2) {
            if (leader) {
              bulk_wait_read_prior();
              mbar_arrive(&sb->own_free[sb1]);
            }
            if (!mbar_wait_warp(&sb->own_free[sb1], (uint32_t)((it >> 1) - 1) & 1u, wc)) { ok = false; break; }
          }
          uint8_t* xs = smem + Sm::kOffStash + sb1 * Sm::kSxBlock;
          {
            float amax = 0.0f;
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
              for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(__uint_as_float(r[c][i])));
            amax *= fabsf(p.scale_log2);
            // e with amax 2^e < 2^14: amax < 2^E for E = (biased exponent of amax) - 126
            const int E = (int)((__float_as_uint(amax) >> 23) & 0xffu) - 126;
            const int e = amax > 0.0f ? min(max(14 - E, -100), 100) : 0;
            const float sc = p.scale_log2 * __uint_as_float((uint32_t)(127 + e) << 23);
#pragma unroll
            for (int gi = 0; gi < kRows / 8; ++gi) {   // 16-byte group gi: rows [8 gi, 8 gi + 8)
              uint32_t enc[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int j = 8 * gi + 2 * i;
                const float y0 = fmaf(__uint_as_float(r[j >> 4][j & 15]), sc, kMagic);
                const float y1 = fmaf(__uint_as_float(r[(j + 1) >> 4][(j + 1) & 15]), sc, kMagic);
                enc[i] = prmt(__float_as_uint(y0), __float_as_uint(y1), 0x5410u);
              }
              st_shared_v4(smem_u32(xs + (gi * 128 + h) * 16), enc[0], enc[1], enc[2], enc[3]);
            }
            *reinterpret_cast<int*>(xs + Sm::kSxCodes + h * 4) = e;
          }
          fence_proxy_async_smem();   // the copy reads the stash through the async proxy
          mbar_arrive_warp(&sb->stash_full[sb1]);
          bool sent = true;
          if (leader) {
            // the peer's buffer of this parity was last released either after its softmax
            // decoded tile it - 2 (nothing to order against the copy) or, when that tile ended
            // the previous unit (it is this unit's second tile), after the peer staged its
            // output through it (generic stores: acquire them)
            const uint32_t par = ((uint32_t)(it >> 1) & 1u) ^ 1u;
            sent = mbar_wait(&sb->stash_full[sb1], (uint32_t)(it >> 1) & 1u, wc) &&
                   (t == 1 ? mbar_wait<true>(&sb->sx_free[sb1], par, wc) : mbar_wait(&sb->sx_free[sb1], par, wc));
            if (sent) {
              mbar_arrive_expect_tx_remote(&sb->sx_ready[sb1], peer, Sm::kSxBlock);
              bulk_copy_to_cluster(sx_peer + (uint32_t)(sb1 * Sm::kSxBlock), smem_u32(xs), Sm::kSxBlock,
                                   mapa_shared(smem_u32(&sb->sx_ready[sb1]), peer));
              bulk_commit();
            }
          }
          if (!__shfl_sync(0xffffffffu, sent, 0)) { ok = false; break; }
        }
      } else {
        // ---- softmax warpgroup: all 64 rows of each tile per thread.  Online softmax in base 2
        // with lazy rescaling of O (only when a head's max grows by more than 2^8).
        for (int t = 0; t < ntiles; ++t) {
          const int it = it0 + t, sbuf = it & 1;
          uint32_t valid0 = mt[2 * t], valid1 = mt[2 * t + 1];
          const int live = first_neg - t * kRows;   // rows past the first -1 are padding
          if (live < 32) {
            valid0 &= live > 0 ? (1u << live) - 1u : 0u;
            valid1 = 0u;
          } else if (live < 64) {
            valid1 &= (1u << (live - 32)) - 1u;
          }
          // this CTA's partials (stash) plus the peer's (its bulk copy; the barrier's completion
          // makes the bytes visible): logit = decoded own + decoded peer, in that order on both
          if (!mbar_wait_warp(&sb->stash_full[sbuf], (uint32_t)(it >> 1) & 1u, wc)) { ok = false; break; }
          if (!mbar_wait_warp(&sb->sx_ready[sbuf], (uint32_t)(it >> 1) & 1u, wc)) { ok = false; break; }
          float s[kRows];
          {
            const uint8_t* own = smem + Sm::kOffStash + sbuf * Sm::kSxBlock;
            const uint8_t* prx = smem + Sm::kOffSx + sbuf * Sm::kSxBlock;
            const int e0 = *reinterpret_cast<const int*>(own + Sm::kSxCodes + h * 4);
            const int e1 = *reinterpret_cast<const int*>(prx + Sm::kSxCodes + h * 4);
            const float dn0 = __uint_as_float((uint32_t)(127 - e0) << 23), bias0 = -kMagic * dn0;
            const float dn1 = __uint_as_float((uint32_t)(127 - e1) << 23), bias1 = -kMagic * dn1;
            // rank 0 adds (own, peer) and rank 1 (peer, own): the same two values in the same
            // order on both CTAs
            const uint8_t* first = rank == 0 ? own : prx;
            const uint8_t* second = rank == 0 ? prx : own;
            const float dnA = rank == 0 ? dn0 : dn1, biasA = rank == 0 ? bias0 : bias1;
            const float dnB = rank == 0 ? dn1 : dn0, biasB = rank == 0 ? bias1 : bias0;
#pragma unroll
            for (int gi = 0; gi < kRows / 8; ++gi) {
              const uint4 a4 = *reinterpret_cast<const uint4*>(first + (gi * 128 + h) * 16);
              const uint4 b4 = *reinterpret_cast<const uint4*>(second + (gi * 128 + h) * 16);
              const uint32_t qa[4] = {a4.x, a4.y, a4.z, a4.w}, qb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float a0 = fmaf(__uint_as_float(prmt(qa[i], 0x4B000000u, 0x7610u)), dnA, biasA);
                const float a1 = fmaf(__uint_as_float(prmt(qa[i], 0x4B000000u, 0x7632u)), dnA, biasA);
                const float b0 = fmaf(__uint_as_float(prmt(qb[i], 0x4B000000u, 0x7610u)), dnB, biasB);
                const float b1 = fmaf(__uint_as_float(prmt(qb[i], 0x4B000000u, 0x7632u)), dnB, biasB);
                s[8 * gi + 2 * i] = a0 + b0;
                s[8 * gi + 2 * i + 1] = a1 + b1;
              }
            }
          }
          // both blocks are in registers: the stash may be rewritten (with the copy's read) and
          // the peer may refill our buffer; after the unit's last tile the peer's block first
          // stages the epilogue's output (released there)
          mbar_arrive_warp(&sb->own_free[sbuf]);
          if (t + 1 < ntiles) mbar_arrive_cluster_relaxed_warp(&sb->sx_free[sbuf], peer);
          float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          if ((valid0 & valid1) == ~0u) {
#pragma unroll
            for (int i = 0; i < kRows; ++i) mx[i & 3] = fmaxf(mx[i & 3], s[i]);
          } else {
#pragma unroll
            for (int i = 0; i < kRows; ++i) {
              s[i] = (((i < 32 ? valid0 : valid1) >> (i & 31)) & 1u) ? s[i] : -INFINITY;
              mx[i & 3] = fmaxf(mx[i & 3], s[i]);
            }
          }
          const float mt_ = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
          float alpha = 1.0f;
          const bool need = mt_ > m + 8.0f;
          if (need) {
            alpha = fast_exp2(m - mt_);   // 0 when m is -inf
            m = mt_;
          }
          float ps[4] = {0.f, 0.f, 0.f, 0.f};
          if (m != -INFINITY) {
            // masked logits are -inf and m is finite: their exp2 is exactly 0
#pragma unroll
            for (int i = 0; i < kRows; ++i) {
              s[i] = fast_exp2(s[i] - m);
              ps[i & 3] += s[i];
            }
          } else {
#pragma unroll
            for (int i = 0; i < kRows; ++i) s[i] = 0.0f;
          }
          l = l * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));

          // P . C of the previous tile must be done: it reads the P buffer, and O is rescaled
          if (!mbar_wait_warp(&sb->p_empty, ((uint32_t)it & 1u) ^ 1u, wc)) { ok = false; break; }
          tc_fence_after();
          if (__any_sync(0xffffffffu, need && t > 0)) {
            // O holds the tiles < t of this unit
#pragma unroll 1
            for (int c = 0; c < Lay::kPvN; c += 16) {
              uint32_t rr[16];
              tmem_ld16(lane_addr + Tm::kO + c, rr);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
              tmem_st16(lane_addr + Tm::kO + c, rr);
            }
            tmem_wait_st();
          }
          // P (bf16) into shared memory: head h's row, K columns = the tile's 64 rows
#pragma unroll
          for (int k = 0; k < kRows / 8; ++k)
            st_shared_v4(smem_u32(smem + Sm::kOffP + swizzled_offset((uint32_t)h, (uint32_t)k * 16, 128)),
                         pack_bf16x2(s[8 * k], s[8 * k + 1]), pack_bf16x2(s[8 * k + 2], s[8 * k + 3]),
                         pack_bf16x2(s[8 * k + 4], s[8 * k + 5]), pack_bf16x2(s[8 * k + 6], s[8 * k + 7]));
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive_warp(&sb->p_full);   // P written (and O rescaled) by this warp
        }
      }
      s_it = it0 + ntiles;
      if (!ok) break;
      mbar_arrive_warp(&sb->tab_free[buf]);
      // ---- unit epilogue: normalise O and write it out
      if (ntiles > 0) {
        if (!mbar_wait_warp(&sb->o_full, (uint32_t)o_it & 1u, wc)) { ok = false; break; }
        ++o_it;
        // the softmax warpgroup has decoded the last tile (so the peer-logit buffer may stage
        // output), and the exchange warpgroup takes each head's max and sum from it
        if (wg == 0) {
          lbuf[h] = l;
          lbuf[128 + h] = m;
        }
        mbar_arrive_warp(&sb->epi_sync);
        if (!mbar_wait_warp(&sb->epi_sync, (uint32_t)e_it & 1u, wc)) { ok = false; break; }
        ++e_it;
        if (wg == 1) {
          l = lbuf[h];
          m = lbuf[128 + h];
        }
      }
      tc_fence_after();
      const bool any = ntiles > 0 && l > 0.0f;
      const float inv = any ? 1.0f / l : 0.0f;
      const float lse = any ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
      const bool real_head = h < p.H;
      // O rows (the bf16 output, or a piece's normalised fp32 partial): each warpgroup writes
      // half of this CTA's columns, staged through a 128B-swizzled 4 KB slice per warp
      // (the softmax warpgroup in the P buffer, free once the unit's last P . C is done; the
      // exchange warpgroup in the last tile's peer-logit block, released to the peer only
      // afterwards) so that each global store writes four whole 128-byte runs
      const bool partial = un.rec >= 0;
      const int c_lo = wg * (Lay::kPvN / 2), c_hi = (wg + 1) * (Lay::kPvN / 2);
      if (ntiles > 0) {
        uint8_t* slice = (wg == 0 ? smem + Sm::kOffP : smem + Sm::kOffSx + ((it0 + ntiles - 1) & 1) * Sm::kSxBlock) + quad * 4096;
        if (!partial) {
          // the output, bf16: 64 columns (128 bytes) per head and round
          uint16_t* obase = p.out + (long long)bj * p.H * p.DL + rank * Lay::kPvN;
#pragma unroll 1
          for (int c = c_lo; c < c_hi; c += 64) {
            uint32_t w[32];
            {
              // four loads in flight per TMEM wait (a wait per load made the epilogue latency bound)
              uint32_t r[4][16];
#pragma unroll
              for (int q = 0; q < 4; ++q) tmem_ld16(lane_addr + Tm::kO + c + 16 * q, r[q]);   // past c_hi: not stored
              tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int i = 0; i < 8; ++i)
                  w[8 * q + i] = pack_bf16x2(__uint_as_float(r[q][2 * i]) * inv, __uint_as_float(r[q][2 * i + 1]) * inv);
            }
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 8; ++k)
              st_shared_v4(smem_u32(slice + lane * 128 + ((k ^ (lane & 7)) * 16)), w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int r = 4 * k + (lane >> 3), blk = lane & 7;
              const int head = quad * 32 + r;
              const uint4 v = *reinterpret_cast<const uint4*>(slice + r * 128 + ((blk ^ (r & 7)) * 16));
              if (head < p.H && c + 8 * blk < c_hi)
                *reinterpret_cast<uint4*>(obase + (long long)head * p.DL + c + 8 * blk) = v;
            }
          }
        } else {
          // a piece, fp32 (the merge rounds once, to the bf16 output): 32 columns per round
          float* obase = p.part_o + (long long)un.rec * p.H * p.DL + rank * Lay::kPvN;
#pragma unroll 1
          for (int c = c_lo; c < c_hi; c += 32) {
            uint32_t w[32];
            {
              uint32_t r[2][16];
#pragma unroll
              for (int q = 0; q < 2; ++q) tmem_ld16(lane_addr + Tm::kO + c + 16 * q, r[q]);   // past c_hi: not stored
              tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < 2; ++q)
#pragma unroll
                for (int i = 0; i < 16; ++i) w[16 * q + i] = __float_as_uint(__uint_as_float(r[q][i]) * inv);
            }
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 8; ++k)
              st_shared_v4(smem_u32(slice + lane * 128 + ((k ^ (lane & 7)) * 16)), w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int r = 4 * k + (lane >> 3), blk = lane & 7;
              const int head = quad * 32 + r;
              const uint4 v = *reinterpret_cast<const uint4*>(slice + r * 128 + ((blk ^ (r & 7)) * 16));
              if (head < p.H && c + 4 * blk < c_hi)
                *reinterpret_cast<uint4*>(obase + (long long)head * p.DL + c + 4 * blk) = v;
            }
          }
        }
      } else if (real_head) {
        // empty list: zeros (the exchange buffer may already hold the peer's next logits)
        if (!partial) {
          uint16_t* obase = p.out + (long long)bj * p.H * p.DL + rank * Lay::kPvN;
          for (int c = c_lo; c < c_hi; c += 8)
            *reinterpret_cast<uint4*>(obase + (long long)h * p.DL + c) = make_uint4(0, 0, 0, 0);
        } else {
          float* obase = p.part_o + (long long)un.rec * p.H * p.DL + rank * Lay::kPvN;
          for (int c = c_lo; c < c_hi; c += 4)
            *reinterpret_cast<uint4*>(obase + (long long)h * p.DL + c) = make_uint4(0, 0, 0, 0);
        }
      }
      if (real_head && wg == 0) {
        // a piece records the log-sum-exp of each CTA of the pair (their logits differ in the
        // last bits: each adds its own exact partial to the peer's decoded one)
        if (partial) p.part_lse[((long long)un.rec * 2 + rank) * p.H + h] = lse;
        else if (p.lse && rank == 0) p.lse[(long long)bj * p.H + h] = lse;
      }
      if (ntiles > 0 && wg == 1) {
        // the exchange warpgroup staged its output through the peer-logit buffer of the last
        // tile: it releases that buffer to the peer now (deferred from the tile)
        __syncwarp();
        fence_proxy_async_smem();   // the peer's next bulk copy into this buffer comes after our stores
        mbar_arrive_cluster_warp(&sb->sx_free[(it0 + ntiles - 1) & 1], peer);
      }
      tc_fence_before();   // our reads of O come before the next unit's first P . C
    }
    // drain: this CTA's bulk copies into the peer are complete before the final cluster barrier
    if (leader) bulk_wait_all();
    };
    if (warp < 4) {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
      role(std::integral_constant<int, 0>{});
    } else {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kExchangeRegs));
      role(std::integral_constant<int, 1>{});
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer no longer writes into our shared memory or arrives on our barriers
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Lay::kTmemCols);
  }
}

// Log-sum-exp merge of the pieces of the queries that straddle a CTA-pair boundary.  One
// (boundary, head) per DL/8 threads, 8 output dims per thread (two 16-byte loads of the fp32
// partials); the first boundary inside a query merges all of that query's pieces: the last unit
// of the pair before it, then the first unit of every pair that starts inside the query.
constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const CombineKernelParams p) {
  // every pair's first tile, computed once per CTA (one 64-bit division per thread at most)
  __shared__ long long starts[kAttnMaxPairs + 1];
  const int TQ = p.tiles_per_q, C = p.split.C;
  for (int i = threadIdx.x; i <= C; i += kCombineThreads) starts[i] = attn_pair_start(p.split, i);
  __syncthreads();
  pdl_launch_dependents();  // the dependent waits for this grid's completion before its loads
  pdl_wait_primary();
  const int tph = p.DL / 8;                               // threads per (boundary, head)
  const long long bh = (long long)blockIdx.x * (kCombineThreads / tph) + threadIdx.x / tph;
  const int d8 = (threadIdx.x % tph) * 8;
  if (bh >= (long long)(C - 1) * p.H) return;
  const int c = 1 + (int)(bh / p.H), h = (int)(bh % p.H);
  const long long g = starts[c];
  const long long q0 = (long long)((int)g / TQ) * TQ;     // G < 2^31
  if (g == q0) return;                                   // a boundary at a query start
  if (starts[c - 1] > q0) return;                        // an earlier boundary owns this query
  const int bj = (int)(q0 / TQ);
  const int rank = d8 >= p.DL / 2 ? 1 : 0;               // the CTA that computed these dims
  float mx = -INFINITY, wsum = 0.0f, o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int recs[4];
  int n = 0;
  auto merge = [&]() {
    // the log-sum-exps and partial vectors of up to four pieces are loaded together, so a
    // merge of up to four pieces waits for one memory latency
    float ls[4];
    uint4 v[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool in = i < n;
      const long long e = in ? recs[i] : 0;
      ls[i] = in ? p.part_lse[(e * 2 + rank) * p.H + h] : -INFINITY;
      const float* src = p.part_o + (e * p.H + h) * p.DL + d8;
      v[i][0] = in ? ld_nc_v4(src) : make_uint4(0, 0, 0, 0);
      v[i][1] = in ? ld_nc_v4(src + 4) : make_uint4(0, 0, 0, 0);
    }
    n = 0;
    float m_new = mx;
#pragma unroll
    for (int i = 0; i < 4; ++i) m_new = fmaxf(m_new, ls[i]);
    if (m_new == -INFINITY) return;   // every piece so far is empty
    const float cf = mx == -INFINITY ? 0.0f : expf(mx - m_new);
    wsum *= cf;
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j] *= cf;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float wgt = ls[i] == -INFINITY ? 0.0f : expf(ls[i] - m_new);
      const uint32_t w8[8] = {v[i][0].x, v[i][0].y, v[i][0].z, v[i][0].w, v[i][1].x, v[i][1].y, v[i][1].z, v[i][1].w};
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] += wgt * __uint_as_float(w8[k]);
      wsum += wgt;
    }
    mx = m_new;
  };
  // pair c - 1 holds the query's first piece: its last unit, or its only one when it starts at q0
  recs[n++] = 2 * (c - 1) + (starts[c - 1] == q0 ? 0 : 1);
  for (int cc = c; cc < C && starts[cc] < q0 + TQ; ++cc) {
    recs[n++] = 2 * cc;   // every later pair's first unit
    if (n == 4) merge();
  }
  if (n > 0) merge();
  const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
  const long long row = (long long)bj * p.H + h;
  *reinterpret_cast<uint4*>(p.out + row * p.DL + d8) =
      make_uint4(pack_bf16x2(o[0] * inv, o[1] * inv), pack_bf16x2(o[2] * inv, o[3] * inv),
                 pack_bf16x2(o[4] * inv, o[5] * inv), pack_bf16x2(o[6] * inv, o[7] * inv));
  if (d8 == 0 && p.lse) p.lse[row] = wsum > 0.0f ? mx + logf(wsum) : -INFINITY;
}

// The dynamic shared memory of a launch: at most two CTAs per SM may share the 512 TMEM columns
// (kTmemCols each <= 256 when two fit), so a small layout still takes 100 KB.
template <int DL, int DR>
size_t attend_launch_smem() {
  using Sm = AttnSmem<AttnLayout<DL, DR>>;
  return Sm::kBytes < 100 * 1024 ? 100 * 1024 : Sm::kBytes;
}

// How many 2-CTA clusters of the kernel the device holds at once (0 if the runtime cannot say).
// A cluster's CTAs must sit in one GPC, so this can be below half the SM count.
template <int DL, int DR, bool KV8>
int attend_clusters_impl() {
  const size_t smem = attend_launch_smem<DL, DR>();
  if (cudaFuncSetAttribute(sparse_attend_kernel<DL, DR, KV8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kAttnThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, sparse_attend_kernel<DL, DR, KV8>, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return n;
}

template <int DL, int DR, bool KV8>
cudaError_t launch_attend_impl(const AttnKernelParams& p, const CUtensorMap& q_rope, int n_clusters,
                               bool pdl, cudaStream_t stream) {
  {
    // the warpgroup register split assumes the launch allocation kLaunchRegs per thread
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, sparse_attend_kernel<DL, DR, KV8>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  }
  const size_t smem = attend_launch_smem<DL, DR>();
  cudaError_t e = cudaFuncSetAttribute(sparse_attend_kernel<DL, DR, KV8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  AttnMaps m;
  m.q_rope = q_rope;
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
  return cudaLaunchKernelEx(&cfg, sparse_attend_kernel<DL, DR, KV8>, m, p);
}

}  // namespace

size_t attend_smem_bytes(int dl, int dr) {
  if (dl == 512 && dr == 64) return AttnSmem<AttnLayout<512, 64>>::kBytes;
  if (dl == 64 && dr == 16) return AttnSmem<AttnLayout<64, 16>>::kBytes;
  return 0;
}

int attend_max_clusters(int dl, int dr, bool kv8) {
  if (dl == 512 && dr == 64)
    return kv8 ? attend_clusters_impl<512, 64, true>() : attend_clusters_impl<512, 64, false>();
  if (dl == 64 && dr == 16)
    return kv8 ? attend_clusters_impl<64, 16, true>() : attend_clusters_impl<64, 16, false>();
  return 0;
}

cudaError_t launch_sparse_attend(const AttnKernelParams& p, const CUtensorMap& q_rope,
                                 int n_clusters, bool pdl, cudaStream_t stream) {
  if (p.DL == 512 && p.DR == 64)
    return p.kv_fp8 ? launch_attend_impl<512, 64, true>(p, q_rope, n_clusters, pdl, stream)
                    : launch_attend_impl<512, 64, false>(p, q_rope, n_clusters, pdl, stream);
  if (p.DL == 64 && p.DR == 16)
    return p.kv_fp8 ? launch_attend_impl<64, 16, true>(p, q_rope, n_clusters, pdl, stream)
                    : launch_attend_impl<64, 16, false>(p, q_rope, n_clusters, pdl, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_combine(const CombineKernelParams& p, bool pdl, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  const long long per_cta = kCombineThreads / (p.DL / 8);
  cfg.gridDim = dim3((unsigned)(((long long)(p.split.C - 1) * p.H + per_cta - 1) / per_cta), 1, 1);
  cfg.blockDim = dim3(kCombineThreads, 1, 1);
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
