/*
 * sia.h -- C ABI of libsia, the B200 (sm_100a) library for indexed sparse attention over
 *          paged caches: a lightweight indexer that scores every causal history position
 *          from a paged index-K cache and keeps each query's Top-K positions, followed by an
 *          MLA-style attention that gathers only those rows of the paged latent KV cache.
 *
 * Source of the operations (titles and sections of the pages describing the method):
 *   - "Day0 Inference Adaptation and Performance Optimization for New-Architecture LLMs",
 *     section 2 (index-based sparse attention branch) and section 3.1 (fused indexer);
 *   - "Rapid Adaptation and Inference Optimization: Key Engineering Practices for Day0 LLM
 *     Support", sections IV.4.1 (indexer fusion: read the paged key cache directly, output
 *     only the final Top-K indices) and IV.4.2 (sparse attention reads the selected rows of the
 *     main KV cache through the paged cache management, with no extra copies);
 *   - "Day 0 Inference Adaptation and Performance Optimization for Hybrid Sparse Attention
 *     LLMs", section "Operator Fusion and Multi-Stream Scheduling" (the five-step decode chain
 *     score -> head-weighted sum -> Top-K -> gather -> sparse attention, and its fusion into
 *     an index operator plus a sparse attention operator, each with BF16 and quantised paths);
 *   - "Day0 Inference Adaptation and Performance Optimization for a New Hybrid-Attention LLM
 *     Architecture", section 4.1 (the fused_indexer(q_quant, k, head_weight) call).
 * The score is fixed as  I[t,s] = sum_h w[t,h] * ReLU(q[t,h] . k[s])  (one index key per
 * position, shared by every head), and Top-K ties go to the lower position.
 *
 * Conventions for every call:
 *   - every pointer in the argument structs is a DEVICE pointer owned by the caller; the
 *     library never allocates, frees or synchronises; `stream` is a cudaStream_t passed as
 *     void*; all work is enqueued asynchronously on it;
 *   - argument errors are found on the host, before anything is launched, and returned as a
 *     status code; a CUDA launch error returns SIA_ERR_CUDA;
 *   - data errors that only the device can see (a page id outside [0, num_pages), a query
 *     position or Top-K entry at or past seq_len) never trap: the kernel ORs a SIA_DEV_* bit
 *     into *dev_status (when dev_status is not NULL), treats the offending row as absent and
 *     carries on; the caller reads *dev_status after synchronising;
 *   - every wait inside a kernel is bounded (two seconds unless sia_set_wait_limit_ns says
 *     otherwise); a wait that gives up sets SIA_DEV_TIMEOUT and the kernel returns early,
 *     leaving its outputs undefined (before it returns, every CTA still waits, with a bound of
 *     its own, for the asynchronous copies and tensor-core operations it issued); when
 *     SIA_DEV_TIMEOUT or SIA_DEV_INTERNAL is set, every output of the call is undefined;
 *   - layout: row-major, innermost dimension last, no padding between rows.
 */
#ifndef SIA_H
#define SIA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SIA_OK = 0,
    SIA_ERR_INVALID_ARGUMENT = 1, /* a NULL pointer, a bad size, mismatched arguments        */
    SIA_ERR_UNSUPPORTED = 2,      /* a shape or dtype this build has no kernel for            */
    SIA_ERR_CUDA = 3,             /* a CUDA runtime call or kernel launch failed              */
    SIA_ERR_WORKSPACE = 4         /* workspace NULL, too small or not 256-byte aligned        */
} sia_status;

/* Bits OR-ed into *dev_status by the kernels. */
#define SIA_DEV_BAD_PAGE 0x1      /* a page-table entry used by the call is outside the pool  */
#define SIA_DEV_BAD_POSITION 0x2  /* a query position or Top-K entry is >= seq_len          */
#define SIA_DEV_TIMEOUT 0x4       /* a bounded in-kernel wait gave up                         */
#define SIA_DEV_INTERNAL 0x8      /* a kernel could not set itself up (its shared-memory base
                                     was not 1024-byte aligned) and returned at once           */

typedef enum {
    SIA_BF16 = 0,                 /* bfloat16                                                 */
    SIA_FP8_E4M3 = 1,             /* OCP FP8 E4M3 ("fn": no infinities), one byte per value   */
    SIA_MXFP8 = 2                 /* E4M3 codes with one E8M0 scale per 32 elements (OCP MX)  */
} sia_dtype;

/*
 * Stage 1: the lightweight indexer with fused Top-K.
 *
 * For every sequence b and query j at position p = q_pos[b][j] (default seq_lens[b]-n_q+j):
 *   I[s] = q_scale[b][j] * k_scale[s] * sum_h w[b][j][h] * ReLU(q[b][j][h] . k[s]),  s <= p
 * where k[s] is row (s % page_size) of page page_table[b][s / page_size] of k_cache, and
 * topk_out[b][j] receives the positions of the top_k largest I[s] (ties: lower s first) in
 * ascending order, padded with -1 when fewer than top_k positions are visible (p+1 < top_k).
 *
 * dtype SIA_MXFP8 (the pages' MXFP8 indexing path: "Rapid Adaptation and Inference
 * Optimization", tiered quantisation table; "Day 0 Inference Adaptation and Performance
 * Optimization for Hybrid Sparse Attention LLMs", section 5.1): q and k_cache hold E4M3 codes and
 * every 32 consecutive elements of a q head vector or of a key share one E8M0 scale 2^(e - 127)
 * (q_mx, k_mx; q_scale and k_scale must be NULL); elements are dequantised, then scored by the
 * same formula.  head_dim must be 64 or 128.  Each query is scored on its own (the keys are
 * read once per query token, so J = 2 reads them twice).
 */
typedef struct {
    int32_t batch;              /* B >= 1                                                    */
    int32_t n_q;                /* query tokens per sequence J >= 1 (decode 1-2, prefill T)  */
    int32_t n_heads;            /* indexer heads H, 1..64                                    */
    int32_t head_dim;           /* D; bf16: 32, 64 or 128; fp8: 64, 128 or 256               */
    int32_t page_size;          /* P, a power of two, 8..4096                                */
    int32_t max_pages_per_seq;  /* columns of page_table                                     */
    int32_t num_pages;          /* pages in k_cache (the pool), for the device bounds check  */
    int32_t top_k;              /* K >= 1                                                    */
    sia_dtype dtype;            /* element type of both q and k_cache                        */
    const void* q;              /* [B, J, H, D] of dtype                                     */
    const float* q_scale;       /* NULL (= 1) or [B, J], positive                            */
    const float* w;             /* [B, J, H] fp32 head weights (any sign)                    */
    const void* k_cache;        /* [num_pages, P, D] of dtype                                */
    const float* k_scale;       /* NULL (= 1) or [num_pages, P] fp32, positive               */
    const int32_t* page_table;  /* [B, max_pages_per_seq]; entries past the context unused   */
    const int32_t* seq_lens;    /* [B], 0 <= seq_lens[b] <= max_pages_per_seq * P            */
    const int32_t* q_pos;       /* NULL or [B, J] with q_pos < seq_lens[b]                   */
    int32_t* topk_out;          /* [B, J, K] int32 output                                    */
    float* scores_out;          /* NULL, or [B, J, max_pages_per_seq * P] fp32: receives I[s]
                                   for s <= p (other entries are left unwritten)             */
    const uint8_t* q_mx;        /* SIA_MXFP8 only: E8M0 scale codes [B, J, H, D / 32]        */
    const uint8_t* k_mx;        /* SIA_MXFP8 only: E8M0 scale codes [num_pages, P, D / 32]   */
} sia_index_args;

/*
 * Stage 2: MLA-style sparse attention over the selected latent rows.
 *
 * For every (b, j, head h), with c[s] = row (s % P) of page page_table[b][s / P] of kv_cache:
 *   z_s = softmax_scale * q[b][j][h] . c[s]   over all d_latent + d_rope dims,
 *   out[b][j][h] = sum_s softmax(z)_s * c[s][0 : d_latent]     (bf16, fp32 accumulation),
 *   lse[b][j][h] = ln sum_s exp(z_s)                            (-inf if the list is empty)
 * over the positions s listed in topk[b][j] (valid entries first, -1 padding after them; the
 * list need not be sorted).  The main cache is bf16, or FP8 with block scales (kv_scale): "Rapid
 * Adaptation and Inference Optimization", tiered quantisation table, and "Day 0 Inference
 * Adaptation and Performance Optimization for Hybrid Sparse Attention LLMs", section 5.2.
 */
typedef struct {
    int32_t batch;              /* B >= 1                                                    */
    int32_t n_q;                /* J >= 1                                                    */
    int32_t n_heads;            /* attention heads, 1..128                                   */
    int32_t d_latent;           /* (d_latent, d_rope) = (512, 64) or (64, 16)                */
    int32_t d_rope;
    int32_t page_size;          /* P >= 1                                                    */
    int32_t max_pages_per_seq;
    int32_t num_pages;          /* pages in kv_cache                                         */
    int32_t top_k;              /* K >= 1, the row length of topk                            */
    float softmax_scale;
    const void* q;              /* bf16 [B, J, n_heads, d_latent + d_rope]                   */
    const void* kv_cache;       /* bf16 [num_pages, P, d_latent + d_rope]                    */
    const int32_t* page_table;  /* [B, max_pages_per_seq]                                    */
    const int32_t* seq_lens;    /* [B]                                                       */
    const int32_t* topk;        /* [B, J, K] int32                                           */
    void* out;                  /* bf16 [B, J, n_heads, d_latent] output                     */
    float* lse;                 /* NULL or fp32 [B, J, n_heads] output                       */
    const float* kv_scale;      /* NULL: kv_cache is bf16.  Else kv_cache holds FP8 E4M3 codes
                                   [num_pages, P, d_latent + d_rope] and kv_scale fp32
                                   [num_pages, P, ceil((d_latent + d_rope) / 128)]: element d of
                                   a row is its decoded code times the scale of block d / 128 of
                                   that row (the pages' FP8 main cache, one scale per 128-element
                                   block); it is rounded once to bf16 before the products     */
} sia_attend_args;

/*
 * Paged cache append: the step before page-table translation.  Writes the J new tokens of every
 * sequence into the index-K cache and the main latent cache, quantising on the way in when a
 * cache is FP8 ("Day0 Inference Adaptation and Performance Optimization for a New
 * Hybrid-Attention LLM Architecture", new cache structures kept in pages; "Rapid Adaptation and
 * Inference Optimization", section IV.4.2, paged cache management; the formats are those of the
 * pages' tiered quantisation table).  Token j of sequence b sits at position
 * p = seq_lens[b] - n_q + j (seq_lens counts the new tokens) and goes to row p % page_size of
 * page page_table[b][p / page_size] of both caches; no other row is written.
 *   SIA_KEY_BF16      k_cache bf16 [num_pages, P, head_dim] (a copy), k_scale NULL;
 *   SIA_KEY_FP8_POW2  k_cache e4m3 codes, k_scale fp32 [num_pages, P]: per token the smallest
 *                     power of two s with max|x| <= 448 s (1 for an all-zero key), codes of x / s;
 *   SIA_KEY_MXFP8     k_cache e4m3 codes, k_scale uint8 E8M0 [num_pages, P, head_dim / 32]: per
 *                     group of 32 elements E = floor(log2 max|x|) - 8 clamped to [-127, 127],
 *                     code E + 127 (127 for an all-zero group), codes of x / 2^E;
 *   SIA_KV_BF16       kv_cache bf16 [num_pages, P, d_kv] (a copy), kv_scale NULL;
 *   SIA_KV_FP8_BLOCK128  kv_cache e4m3 codes, kv_scale fp32 [num_pages, P, ceil(d_kv / 128)]:
 *                     per 128-element block of the row s = fp32(max|x| / 448) (1 for an all-zero
 *                     block), codes of fp32(x / s).
 * e4m3 codes round to nearest, ties to even, and saturate at +-448.  A token whose position is
 * outside [0, max_pages_per_seq * P) or whose page id is outside the pool is skipped and sets
 * SIA_DEV_BAD_POSITION / SIA_DEV_BAD_PAGE.  No workspace.
 */
typedef enum { SIA_KEY_BF16 = 0, SIA_KEY_FP8_POW2 = 1, SIA_KEY_MXFP8 = 2 } sia_key_format;
typedef enum { SIA_KV_BF16 = 0, SIA_KV_FP8_BLOCK128 = 1 } sia_kv_format;

typedef struct {
    int32_t batch;              /* B >= 1                                                    */
    int32_t n_q;                /* new tokens per sequence J >= 1                            */
    int32_t head_dim;           /* index key length: 32..256, a multiple of 32               */
    int32_t d_kv;               /* main-cache row length (d_latent + d_rope): 16..1024, even */
    int32_t page_size;          /* P >= 1                                                    */
    int32_t max_pages_per_seq;
    int32_t num_pages;          /* pages in each pool                                        */
    sia_key_format key_format;
    sia_kv_format kv_format;
    const void* new_k;          /* bf16 [B, J, head_dim]                                     */
    const void* new_kv;         /* bf16 [B, J, d_kv]                                         */
    const int32_t* page_table;  /* [B, max_pages_per_seq]                                    */
    const int32_t* seq_lens;    /* [B], including the J new tokens                          */
    void* k_cache;              /* see key_format                                            */
    void* k_scale;              /* see key_format                                            */
    void* kv_cache;             /* see kv_format                                             */
    float* kv_scale;            /* see kv_format                                             */
} sia_append_args;

sia_status sia_cache_append(const sia_append_args* a, int32_t* dev_status, void* stream);

/* Workspace bytes a call needs (0 for a NULL argument).  The workspace is caller-owned device
 * memory, 256-byte aligned, whose contents need no initialisation and may be reused by the
 * next call on the same stream. */
size_t sia_index_workspace_size(const sia_index_args* a);
size_t sia_attend_workspace_size(const sia_attend_args* a);
size_t sia_workspace_size(const sia_index_args* ia, const sia_attend_args* aa);

/* Stage 1: score every causal position and write each query's Top-K list. */
sia_status sia_sparse_index_topk(const sia_index_args* a, void* workspace, size_t ws_bytes,
                                 int32_t* dev_status, void* stream);

/* The scoring step of stage 1 alone: writes I[t,s] for every causal position s <= p(t) of
 * every query into a->scores_out (required; positions past p(t) are left untouched) and no
 * Top-K list ("Day 0 Inference Adaptation and Performance Optimization for Hybrid Sparse
 * Attention LLMs", section "Operator Fusion and Multi-Stream Scheduling", the score-and-
 * aggregate steps before the selection).  For a prefill chunk this is the dense causal q.k
 * contraction on the tensor cores.  a->topk_out and a->top_k are ignored; a->scores_out NULL
 * -> SIA_ERR_INVALID_ARGUMENT. */
sia_status sia_index_scores(const sia_index_args* a, int32_t* dev_status, void* stream);

/* Stage 2: sparse MLA attention over a Top-K list. */
sia_status sia_sparse_mla_attend(const sia_attend_args* a, void* workspace, size_t ws_bytes,
                                 int32_t* dev_status, void* stream);

/* Stage 1 for callers that cannot allocate device memory while they run (a serving loop with a
 * fixed preallocated arena, a C runtime without a device allocator, a loop that must not stall
 * on cudaMalloc/cudaFree): same operation and arguments as sia_sparse_index_topk, but the
 * per-position scores live in a 16 MiB array inside the library, so no workspace is passed and
 * nothing is allocated.  The pages describing the method have no counterpart of this call.
 *   - limit: batch * n_q * max_pages_per_seq * page_size * 4 bytes <= 16 MiB, else
 *     SIA_ERR_WORKSPACE before any launch (ignored when scores_out is given);
 *   - the array is shared by every call in the process: calls whose kernels may overlap on the
 *     GPU (other streams, other host threads) race on it and must be serialised by the caller;
 *   - the first call on each device (and the first after that device's context was reset)
 *     loads the array's module -- which is when the 16 MiB are reserved on the device -- and
 *     looks up the array's device address (cudaGetSymbolAddress); make that first call at
 *     start-up, before carving a memory arena out of the device and before any stream capture;
 *   - once reserved, the 16 MiB stay reserved on that device until the process exits. */
sia_status sia_sparse_index_topk_noalloc(const sia_index_args* a, int32_t* dev_status, void* stream);

/* Both stages back to back on one stream (programmatic dependent launch between kernels, no
 * host synchronisation; capturable in a CUDA graph).  Stream order is kept: the first kernel of
 * this call (and of sia_sparse_index_topk and sia_index_scores) may be scheduled while the
 * previous kernel on the stream drains, but it reads and writes no global memory before that
 * kernel has completed.  The two argument sets must describe the
 * same sequences: equal batch, n_q, page_size, max_pages_per_seq, top_k, page_table and
 * seq_lens, with aa->topk == ia->topk_out. */
sia_status sia_fused_decode(const sia_index_args* ia, const sia_attend_args* aa,
                            void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream);

/* The bound of every pipeline wait inside the kernels of calls made after this one, from any
 * host thread, in nanoseconds of the GPU's global timer; 0 restores the default of two seconds.
 * Returns the previous bound.  For testing the timeout path (a tiny bound makes the first wait
 * that does not succeed at once give up and report SIA_DEV_TIMEOUT); a serving caller leaves it
 * alone.  Not a counterpart of anything in the pages describing the method. */
uint64_t sia_set_wait_limit_ns(uint64_t ns);

/* Static description of a status code. */
const char* sia_status_string(sia_status s);

/* The detail message of the last failing call made by this host thread ("" if none). */
const char* sia_last_error(void);

/* Library version as MAJOR * 10000 + MINOR * 100 + PATCH. */
int32_t sia_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SIA_H */
