/*
 * mla_decode.h -- C ABI of the B200 (sm_100a) MLA decode library
 * (libmla_decode_b200.so).
 *
 * Multi-head Latent Attention decoding over a paged KV cache: for each
 * sequence of a batch, s_q new query tokens x h_q heads (576-dim bf16 queries)
 * attend to one shared latent KV head of 576 dims (512 latent "NoPE" dims +
 * 64 RoPE dims) stored in 64-token pages reached through a block table; the
 * values are the first 512 dims of the same cache rows.  Each call returns
 * the 512-dim output and the softmax log-sum-exp of every (token, head) row.
 *
 * Sources for the operations:
 *  - get_mla_metadata / flash_mla_with_kvcache call sequence, block size 64,
 *    causal flag, dv, the (o, lse) result: "Was ist FlashMLA?" (topnet.top),
 *    sections "Hauptmerkmale von FlashMLA", "2. MLA-Metadaten abrufen",
 *    "3. MLA-Decodierung ausführen".
 *  - FP8 cache rows (512 e4m3 + 4 fp32 scales + 64 bf16 RoPE) and the sparse
 *    path driven by an indices tensor: FlashMLA walkthrough (sao.pub),
 *    section "二、核心功能与架构".
 *
 * Conventions shared by every entry point:
 *  - Pointers are DEVICE pointers unless a parameter says "host".  The caller
 *    owns every buffer; the library allocates no device memory and keeps no
 *    per-call state (it caches the SM count and kernel attributes).
 *  - Every launch is asynchronous on `stream` (a cudaStream_t passed as
 *    void*; NULL = legacy default stream).  Argument errors are detected on
 *    the host and returned synchronously before anything is launched.
 *  - Data errors found on the device never trap: the kernels OR an
 *    MLA_DEVERR_* bit into *err_word (caller-zeroed int32) and treat the
 *    offending key as masked.
 *  - Thread safety: calls may come from several host threads; each call only
 *    reads its arguments.
 */
#ifndef MLA_DECODE_H
#define MLA_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Symbols of the shared library (everything else in it is hidden). */
#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#define MLA_PAGE_SIZE 64          /* tokens per cache page */
#define MLA_D_QK 576              /* query/key dims: 512 NoPE + 64 RoPE */
#define MLA_D_V 512               /* value/output dims (first 512 key dims) */
#define MLA_FP8_ROW_BYTES 656     /* 512 e4m3 + 4 x fp32 scale + 64 x bf16 */
#define MLA_MD_WORDS 8            /* int32 words per tile_md row */
#define MLA_FIXED_SPLIT_COST 5    /* scheduler cost of one split, in pages */

/* Status codes returned by every entry point. */
enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, bad dim */
  MLA_ERR_UNSUPPORTED = 2,   /* h_kv != 1, d_v != 512, indices with a bf16 cache ... */
  MLA_ERR_WORKSPACE = 3,     /* workspace smaller than mla_workspace_bytes() */
  MLA_ERR_CUDA = 4           /* a CUDA runtime call or launch failed */
};

/* Bits the kernels OR into *err_word. */
#define MLA_DEVERR_BLOCK_TABLE 1  /* block_table entry outside [0, num_blocks) or page beyond the table width */
#define MLA_DEVERR_INDEX 2        /* sparse index outside [0, L) and not -1 */
#define MLA_DEVERR_TIMEOUT 4      /* a pipeline wait gave up (kernel returned early) */
#define MLA_DEVERR_SEQLEN 8       /* negative cache_seqlens entry (treated as 0) */
#define MLA_DEVERR_INTERNAL 16    /* shared-memory alignment or TMEM allocation problem */

/*
 * Host-only.  Shape of the split plan for one decode step: how many rows the
 * tile_scheduler_metadata tensor of the metadata call has, and how long
 * num_splits is ("Was ist FlashMLA?" (topnet.top), section
 * "2. MLA-Metadaten abrufen": get_mla_metadata returns both; their sizes are
 * this library's own, the pages do not give them).
 *   batch, s_q, h_q, h_kv : problem sizes (h_kv must be 1)
 *   topk                  : 0 for the dense path, else indices per query token
 *   num_sm_parts          : <= 0 = choose from the current device's SM count;
 *                           > 0 forces that many partitions (tests)
 *   *num_parts_out        : rows of tile_md (each MLA_MD_WORDS int32)
 *   *num_splits_len_out   : entries of num_splits = units + 1, where a unit
 *                           is a sequence (dense) or a (sequence, token) pair
 *                           (sparse)
 */
MLA_API int mla_metadata_shape(int batch, int s_q, int h_q, int h_kv, int topk, int num_sm_parts,
                       int* num_parts_out, int* num_splits_len_out);

/*
 * Split-KV tile-scheduler metadata ("2. MLA-Metadaten abrufen": computed once
 * per decode step and reused by every layer).  One small kernel on `stream`.
 *   cache_seqlens : int32 [batch] (device)
 *   num_parts     : from mla_metadata_shape
 *   tile_md       : int32 [num_parts, 8] output; row p =
 *                   {unit_begin, page_begin, unit_end, page_end (exclusive
 *                    pair), first_split_index, 0, 0, 0}
 *   num_splits    : int32 [units + 1] output; exclusive prefix sum of the
 *                   number of splits of each unit
 * The plan: unit u with n_u pages (ceil(L/64), or ceil(topk/64) on the sparse
 * path) costs n_u + MLA_FIXED_SPLIT_COST; partition boundary p sits at cost
 * position floor(p * total / num_parts).
 */
MLA_API int mla_get_metadata(const int32_t* cache_seqlens, int batch, int s_q, int h_q, int h_kv, int topk,
                     int num_parts, int32_t* tile_md, int32_t* num_splits, void* stream);

/*
 * Host-only.  Bytes of workspace a decode with this plan needs: fp32 partial
 * outputs and log-sum-exps for at most (units + num_parts) splits.  The pages
 * split the key range through num_splits ("Was ist FlashMLA?" (topnet.top),
 * sections "2. MLA-Metadaten abrufen" and "3. MLA-Decodierung ausführen")
 * without saying where partial results live; this scratch is the library's
 * own.  Returns MLA_ERR_UNSUPPORTED for more than 4 * 65535 query rows per
 * unit (s_q * h_q dense, h_q sparse), which the combine grid cannot span.
 */
MLA_API int mla_workspace_bytes(int batch, int s_q, int h_q, int topk, int num_parts, size_t* bytes);

/* Arguments of a decode call (a host struct; the pointers it holds are device pointers). */
typedef struct mla_decode_args {
  const void* q;                /* bf16 [batch, s_q, h_q, 576]; (s_q, h_q, 576) contiguous, 16-B aligned */
  int64_t q_batch_stride;       /* elements between batch entries (>= s_q*h_q*576, multiple of 8) */
  const void* k_cache;          /* bf16 [num_blocks, 64, 1, 576]  or, with is_fp8,
                                   uint8 [num_blocks, 64, 1, 656]; 16-B aligned */
  int64_t k_block_stride;       /* bytes between pages (multiple of 16, >= one page) */
  int32_t num_blocks;           /* pages in the cache */
  const int32_t* block_table;   /* int32 [batch, block_table_stride] */
  int32_t block_table_stride;   /* int32 entries between rows */
  int32_t block_table_width;    /* valid columns per row; pages beyond are errors */
  const int32_t* cache_seqlens; /* int32 [batch] */
  const int32_t* indices;       /* int32 [batch, s_q, topk] logical positions, -1 = pad; NULL = dense */
  int32_t topk;                 /* indices per query token (0 when dense) */
  const int32_t* tile_md;       /* from mla_get_metadata */
  const int32_t* num_splits;    /* from mla_get_metadata */
  int32_t num_parts;            /* from mla_metadata_shape */
  void* out;                    /* bf16 [batch, s_q, h_q, 512] contiguous (output) */
  float* lse;                   /* fp32 [batch, h_q, s_q] contiguous (output), natural log */
  void* workspace;              /* scratch, 256-B aligned */
  size_t workspace_bytes;       /* >= mla_workspace_bytes() */
  int32_t* err_word;            /* int32, caller-zeroed; MLA_DEVERR_* bits (output) */
  int32_t batch, s_q, h_q, h_kv, d_v;
  float softmax_scale;          /* logits = softmax_scale * q.k; finite and > 0 */
  int32_t causal;               /* dense s_q > 1: token i sees keys t <= L - s_q + i */
  int32_t is_fp8;               /* k_cache holds FP8 rows: read through indices
                                   (sparse) or, with indices == NULL, walked page
                                   by page like the bf16 cache (dense; causal
                                   applies).  The logits carry no dequantisation
                                   rounding: codes enter the MMA as exact f16,
                                   each 128-value group keeps its own fp32 sum,
                                   the fp32 scales multiply the sums, and q is
                                   scaled per row by a power of two into the f16
                                   range, so any finite scale and any bf16 q are
                                   accepted.  V enters PV as f16 code x scale
                                   (x a per-group power of two), which rounds
                                   only the output. */
} mla_decode_args;

/*
 * flash_mla_with_kvcache ("3. MLA-Decodierung ausführen"): the attention
 * kernel followed by the split-combine kernel, both on `stream`.
 * out/lse of a row whose key set is empty are 0 and -inf.
 */
MLA_API int mla_decode(const mla_decode_args* args, void* stream);

/* The attention kernel alone (split results go to the workspace). */
MLA_API int mla_decode_attention(const mla_decode_args* args, void* stream);

/* The LSE-weighted combine of split results alone (after mla_decode_attention). */
MLA_API int mla_decode_combine(const mla_decode_args* args, void* stream);

/*
 * Decode (same arguments and results as mla_decode) for callers that cannot
 * allocate device memory themselves: code that is handed its buffers by a
 * host program and may not create allocations of its own (a plugin inside a
 * serving process whose memory is budgeted up front), or code that must stay
 * off cudaMalloc / cudaFree because those calls can synchronise the device.
 * The pages have no counterpart to this entry point.
 *
 * args->workspace and args->workspace_bytes are ignored: the split-KV
 * partial results go to one scratch array built into the library, of
 * MLA_NOALLOC_SCRATCH_BYTES bytes on every GPU that loads the library, held
 * until the process exits.  A plan needing more than that (see
 * mla_workspace_bytes) returns MLA_ERR_WORKSPACE before anything is
 * launched.  No allocation is made by this call.
 *  - The first call in a CUDA context looks the array's device address up
 *    with cudaGetSymbolAddress, with that context current, and keeps it with
 *    the context's unique id.  A cudaDeviceReset, or a context the caller
 *    makes current through the driver API, has a new id, so the next call
 *    looks the address up again (the module and its array may have moved).
 *    Make the first call in each context before any stream capture begins.
 *  - All calls share the one array, and it keeps whatever the last call left
 *    in it.  Nothing in it needs to start at zero: every slot the combine
 *    kernel reads is written earlier in the same call.  Calls whose kernels
 *    overlap on the GPU (different streams, no ordering between them) race
 *    on the array and corrupt each other's results; order them.
 */
#define MLA_NOALLOC_SCRATCH_BYTES (64u << 20)
MLA_API int mla_decode_noalloc(const mla_decode_args* args, void* stream);

/*
 * FP8 cache writer: quantise n new key rows into the FP8 cache row format
 * (FlashMLA walkthrough (sao.pub), section "二、核心功能与架构": 512 e4m3
 * NoPE values + 4 float32 scales, one per 128 values + 64 bf16 RoPE values =
 * 656 bytes) and store row i at slot_mapping[i] = page * 64 + row.  The pages
 * fix the format; the scales follow the plainest reading: scale = max|x| / 448
 * per 128-value group (float32), code = e4m3 round-to-nearest-even of
 * x / scale (IEEE float32 division), saturating; an all-zero group gets scale
 * 0 and codes 0; RoPE is copied.  (The decode reads these rows back with
 * is_fp8.)
 *
 *   k_new         bf16 [n, 576] (device), rows k_row_stride elements apart
 *                 (multiple of 8, >= 576), 16-B aligned; values finite
 *   slot_mapping  int32 [n] (device); -1 skips a row; a slot outside
 *                 [0, num_blocks * 64) is skipped and sets MLA_DEVERR_BLOCK_TABLE
 *   kv_cache      uint8 [num_blocks, 64, 1, 656] (device, written), pages
 *                 k_block_stride bytes apart (multiple of 16, >= 64 * 656),
 *                 16-B aligned
 *   err_word      int32 (device), caller-zeroed
 * Asynchronous on `stream`; n == 0 launches nothing.  Two rows mapped to the
 * same slot race.  Returns MLA_OK, MLA_ERR_INVALID_ARG or MLA_ERR_CUDA.
 * (No counterpart call on the pages: it is the step that produces the cache
 * the FP8 decode reads.)
 */
MLA_API int mla_fp8_cache_write(const void* k_new, int64_t k_row_stride, int32_t n, const int32_t* slot_mapping,
                                void* kv_cache, int64_t k_block_stride, int32_t num_blocks, int32_t* err_word,
                                void* stream);

/*
 * Give-up limit, in nanoseconds, of the decode kernels' pipeline waits for
 * every decode call launched after this one (0 restores the default of 2 s).
 * A wait that runs past it makes its CTA raise MLA_DEVERR_TIMEOUT in
 * *err_word, drain its own copies and MMAs (those drains always keep the 2 s
 * bound), free its tensor memory and return; the call's out/lse are then
 * undefined, and the next call with the default limit computes normally.
 * This exists to exercise that failure path: the bounded waits are the
 * library's failure detection (a stuck pipeline ends the kernel with an
 * error bit instead of hanging the GPU), and a short limit makes them give
 * up on ordinary inputs.  Limits below 1 ms make the waits poll without
 * suspending the waiting thread (slower, but each test is short enough to
 * see such a limit pass).  It is process-wide and not meant to change while
 * calls from other threads are being launched.  The pages have no
 * counterpart to it.  Returns MLA_OK.
 */
MLA_API int mla_set_pipeline_wait_limit(uint64_t ns);

/* Human-readable name of a status code (static string). */
MLA_API const char* mla_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DECODE_H */
