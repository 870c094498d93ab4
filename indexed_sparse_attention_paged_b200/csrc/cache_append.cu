// cache_append.cu -- writes the new tokens' index keys and latent rows into the paged caches,
// quantising them on the way in when the cache is FP8.
//
// This is the step before page-table translation: the runtime keeps an index cache and a main
// (latent) cache in pages ("Day0 Inference Adaptation and Performance Optimization for a New
// Hybrid-Attention LLM Architecture", on the new cache structures; "Rapid Adaptation and
// Inference Optimization", section IV.4.2, coordinating the sparse attention with paged cache
// management), and the quantised formats of the pages' tiered quantisation table: per-token FP8
// index keys, MXFP8 index keys (one E8M0 scale per 32 elements), and an FP8 main cache with one
// scale per 128-element block of the token's row ("Day 0 Inference Adaptation and Performance
// Optimization for Hybrid Sparse Attention LLMs", section 5).
//
// Token j of the J new tokens of sequence b sits at position p = seq_lens[b] - J + j and goes to
// row p % P of page page_table[b][p / P].  The quantisers are dynamic absmax ones:
//   - FP8 index key: scale = the smallest power of two s with amax <= 448 s (1 for an all-zero
//     key), codes = e4m3(x / s) (an exact division);
//   - MXFP8 index key, per group of 32: E = floor(log2 amax) - 8 clamped to [-127, 127] (the
//     OCP shared exponent; 8 is the largest e4m3 exponent), scale code E + 127 (127 for an
//     all-zero group), codes = e4m3(x / 2^E);
//   - FP8 main cache, per 128-element block: s = fp32(amax / 448) (1 for an all-zero block),
//     codes = e4m3(fp32(x / s));
// e4m3 rounds to nearest, ties to even, and saturates at +-448 (cvt.rn.satfinite).
//
// Design: one CTA of 128 threads per new token; the work is a few hundred bytes per token, so
// the kernel is launch-latency bound and is kept to a single launch for both caches.
#include <cuda_runtime.h>

#include "sia_internal.h"
#include "sia_ptx.cuh"

namespace sia {
namespace {

constexpr int kAppendThreads = 128;
constexpr int kKvBlock = 128;
constexpr int kMaxKvBlocks = 8;   // d_kv <= 1024

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// e4m3 code of x: round to nearest even, saturating to the largest finite value.
__device__ __forceinline__ uint8_t e4m3_code(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return (uint8_t)(r & 0xffu);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__global__ void __launch_bounds__(kAppendThreads) cache_append_kernel(const AppendKernelParams p) {
  __shared__ float red[kAppendThreads / 32][kMaxKvBlocks + 1];
  const int tok = blockIdx.x;
  const int b = tok / p.J, j = tok - (tok / p.J) * p.J;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait_primary();
  pdl_launch_dependents();
  const int pos = p.seq_lens[b] - p.J + j;
  if (pos < 0 || (long long)pos >= (long long)p.max_pages * p.P) {
    if (tid == 0) report(p.status, SIA_DEV_BAD_POSITION);
    return;
  }
  const int page = p.page_table[(long long)b * p.max_pages + pos / p.P];
  if (page < 0 || page >= p.num_pages) {
    if (tid == 0) report(p.status, SIA_DEV_BAD_PAGE);
    return;
  }
  const long long row = (long long)page * p.P + pos % p.P;

  // ---------------------------------------------------------------- index key (D <= 256)
  {
    const uint16_t* x = static_cast<const uint16_t*>(p.new_k) + (long long)tok * p.D;
    float v[2];
    int n = 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int d = tid + i * kAppendThreads;
      v[i] = d < p.D ? bf16_to_f32(x[d]) : 0.0f;
      n += d < p.D;
    }
    if (p.key_format == SIA_KEY_BF16) {
      uint16_t* dst = static_cast<uint16_t*>(p.k_cache) + row * p.D;
      for (int i = 0; i < n; ++i) dst[tid + i * kAppendThreads] = x[tid + i * kAppendThreads];
    } else if (p.key_format == SIA_KEY_FP8_POW2) {
      float a = warp_max(fmaxf(fabsf(v[0]), fabsf(v[1])));
      if (lane == 0) red[warp][0] = a;
      __syncthreads();
      float amax = 0.0f;
#pragma unroll
      for (int w = 0; w < kAppendThreads / 32; ++w) amax = fmaxf(amax, red[w][0]);
      // smallest e with amax <= 448 * 2^e: with amax = m 2^E (m in [0.5, 1)) and 448 = 0.875 2^9,
      // e = E - 9 when m <= 0.875, else E - 8
      int e = 0;
      if (amax > 0.0f) {
        int E;
        const float m = frexpf(amax, &E);
        e = m <= 0.875f ? E - 9 : E - 8;
      }
      uint8_t* dst = static_cast<uint8_t*>(p.k_cache) + row * p.D;
      for (int i = 0; i < n; ++i) dst[tid + i * kAppendThreads] = e4m3_code(ldexpf(v[i], -e));
      if (tid == 0) static_cast<float*>(p.k_scale)[row] = ldexpf(1.0f, e);
      __syncthreads();   // red[] is reused below
    } else {   // SIA_KEY_MXFP8: thread d's group is d / 32, i.e. its warp (plus 4 for d >= 128)
      uint8_t* dst = static_cast<uint8_t*>(p.k_cache) + row * p.D;
      uint8_t* sdst = static_cast<uint8_t*>(p.k_scale) + row * (p.D / 32);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int d0 = warp * 32 + i * kAppendThreads;   // warp-uniform
        if (d0 >= p.D) break;
        const float amax = warp_max(fabsf(v[i]));
        int E = 0;
        if (amax > 0.0f) {
          int f;
          frexpf(amax, &f);   // amax = m 2^f, m in [0.5, 1): floor(log2 amax) = f - 1
          E = min(127, max(-127, f - 1 - 8));
        }
        dst[d0 + lane] = e4m3_code(ldexpf(v[i], -E));
        if (lane == 0) sdst[d0 / 32] = (uint8_t)(E + 127);
      }
    }
  }

  // ---------------------------------------------------------------- main latent row
  {
    const uint16_t* x = static_cast<const uint16_t*>(p.new_kv) + (long long)tok * p.DC;
    if (p.kv_format == SIA_KV_BF16) {
      uint16_t* dst = static_cast<uint16_t*>(p.kv_cache) + row * p.DC;
      for (int d = tid; d < p.DC; d += kAppendThreads) dst[d] = x[d];
      return;
    }
    // block k covers elements [128k, 128k + 128): thread t holds element 128k + t of each block
    const int nblk = (p.DC + kKvBlock - 1) / kKvBlock;
    float v[kMaxKvBlocks];
#pragma unroll
    for (int k = 0; k < kMaxKvBlocks; ++k) {
      const int d = k * kKvBlock + tid;
      v[k] = (k < nblk && d < p.DC) ? bf16_to_f32(x[d]) : 0.0f;
      const float a = warp_max(fabsf(v[k]));
      if (lane == 0) red[warp][k] = a;
    }
    __syncthreads();
    uint8_t* dst = static_cast<uint8_t*>(p.kv_cache) + row * p.DC;
#pragma unroll
    for (int k = 0; k < kMaxKvBlocks; ++k) {
      if (k >= nblk) break;
      float amax = 0.0f;
#pragma unroll
      for (int w = 0; w < kAppendThreads / 32; ++w) amax = fmaxf(amax, red[w][k]);
      const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
      const int d = k * kKvBlock + tid;
      if (d < p.DC) dst[d] = e4m3_code(__fdiv_rn(v[k], s));
      if (tid == 0) p.kv_scale[row * nblk + k] = s;
    }
  }
}

}  // namespace

cudaError_t launch_cache_append(const AppendKernelParams& p, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3((unsigned)((long long)p.B * p.J), 1, 1);
  cfg.blockDim = dim3(kAppendThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, cache_append_kernel, p);
}

}  // namespace sia
