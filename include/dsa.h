/*
 * dsa.h - C ABI of the DSA sparse-attention step for NVIDIA B200 (sm_100a).
 *
 * The step (GLM-5 decoder attention with DeepSeek-style sparse attention):
 *   1. indexer scores   score[s] = sum_h w[h] * max(0, q_idx[h] . k_idx[s])
 *   2. exact top-k      keep the k best tokens (all of them when fewer exist);
 *                       equal scores resolve to the lower token index
 *   3. absorbed MLA     attention in the compressed latent space over the
 *                       kept tokens only:
 *                         z[h,j]   = scale * q[h,:] . L[idx_j, :]      (all R+P columns)
 *                         out[h,:] = sum_j softmax_j(z[h,:]) * L[idx_j, 0:R]
 *                         lse[h]   = log sum_j exp(z[h,j])            (natural log)
 *
 * Sources: "GLM on an A100, in Vx", section "The model" (an indexer scores
 * every earlier token; each query attends to the 2,048 highest-scoring tokens;
 * below 2,048 tokens everything is kept; keys and values share one latent
 * vector per token) and section "How do we know it is right?" (ReLU inside the
 * indexer; ties follow a stable argsort of -scores).  "Self-contained GLM-5
 * serving stack: Just Vx kernels compiled to PTX", file list (absorbed MLA
 * decode, compressed request-local KV, DSA indexer selection) and GPU-code
 * paragraph (split online-softmax compressed MLA).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - bf16 tensors are passed as raw 16-bit patterns (uint16_t).
 *  - Every tensor pointer is DEVICE memory owned by the caller.  The library
 *    allocates nothing, keeps no mutable global state and is thread-safe.
 *  - Every call is asynchronous on `stream`.  A NULL stream means the
 *    per-thread default stream, never the legacy default stream.
 *  - Arguments (shapes, ranges, 16-byte alignment) are checked on the host
 *    before anything is launched; a rejected call has no side effects and
 *    returns DSA_ERR_INVALID_ARG or DSA_ERR_UNSUPPORTED.  Launch failures
 *    return DSA_ERR_CUDA.  No C++ exception crosses this interface.
 *  - Checks made on the device (a page id or token index out of range, a
 *    bounded wait that gave up) never fault: the kernel skips the access,
 *    records the event in the workspace status block and finishes.  Read it
 *    with dsa_workspace_check().
 *
 * Paged caches
 * ------------
 * Both caches are pools of 64-token pages that share one block table:
 *   k_idx_pages   [num_pages, 64, D_I]   bf16  indexer keys, one per token
 *   latent_pages  [num_pages, 64, R + P] bf16  latent rows [c_kv (R) | k_rope (P)]
 * Token s of sequence b lives in physical page block_table[b, s / 64], slot s % 64.
 *
 * Query rows
 * ----------
 * Decode (dims.causal == 0): row b is the newest token of sequence b; it sits
 *   at position seq_lens[b] - 1 and sees tokens 0 .. seq_lens[b]-1.
 * Prefill (dims.causal == 1): the rows are T consecutive tokens of sequence 0;
 *   row t sits at position q_pos0 + t and sees tokens 0 .. q_pos0 + t.
 *
 * Index output: the kept token positions of each row in ascending order,
 * padded with -1 when the row sees fewer than k tokens.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

/* cudaStream_t without pulling in the CUDA headers. */
typedef struct CUstream_st *dsa_stream_t;

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,  /* bad pointer, shape, alignment or range (host check) */
  DSA_ERR_UNSUPPORTED = 2,  /* valid request outside what the kernels implement   */
  DSA_ERR_CUDA = 3,         /* a CUDA runtime call or a launch failed              */
  DSA_ERR_WORKSPACE = 4,    /* workspace missing, misaligned or too small          */
  DSA_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up (from the status block) */
  DSA_ERR_DEVICE_CHECK = 6  /* a device-side range check failed (from the status block)   */
} dsa_status_t;

/* Paged-cache view.  Pointers are device memory. */
typedef struct {
  int32_t num_seqs;            /* sequences (decode: B; prefill: 1)                  */
  const int32_t *seq_lens;     /* [num_seqs] tokens in the cache, current included   */
  const int32_t *block_table;  /* [num_seqs, max_pages] physical page ids             */
  int32_t max_pages;           /* row stride of block_table                           */
  int32_t page_size;           /* tokens per page; must be 64                          */
  int32_t num_pages;           /* physical pages in each pool (device range check)    */
  int32_t max_seq_len;         /* host-side upper bound on every seq_lens[b]; sizes grids */
} dsa_cache_t;

/* Problem dimensions. */
typedef struct {
  int32_t n_q;     /* query rows: decode B (== num_seqs); prefill T                 */
  int32_t H_I;     /* indexer heads, 1..64                                            */
  int32_t D_I;     /* indexer head dim: 32, 64 or 128                                 */
  int32_t topk;    /* k: 1..4096                                                      */
  int32_t H;       /* MLA heads, 1..64 (tiles always hold 64 head columns)            */
  int32_t R;       /* latent (kv_lora) rank, multiple of 64, <= 512                   */
  int32_t P;       /* rope part, multiple of 16, R + P <= 576                          */
  int32_t causal;  /* 0 = decode rows, 1 = causal prefill rows of sequence 0           */
  int32_t q_pos0;  /* prefill: position of row 0                                       */
  float scale;     /* softmax scale applied to q . L                                   */
} dsa_dims_t;

/* Operation ids for dsa_workspace_bytes(). */
typedef enum {
  DSA_OP_INDEXER_SCORES = 0,
  DSA_OP_TOPK = 1,
  DSA_OP_SPARSE_MLA_DECODE = 2,
  DSA_OP_SPARSE_MLA_PREFILL = 3,
  DSA_OP_ATTENTION_FORWARD = 4,
  DSA_OP_CACHE_APPEND = 5,
  DSA_OP_INDEXER_SCORES_K8 = 6,   /* dsa_indexer_scores_k8 */
  DSA_OP_ATTENTION_FORWARD_K8 = 7, /* dsa_attention_forward_k8 */
  DSA_OP_ATTENTION_FORWARD_HOST = 8, /* dsa_attention_forward_host */
  DSA_OP_ATTENTION_FORWARD_FP8 = 9   /* dsa_attention_forward_fp8 */
} dsa_op_t;

/* Library version (major * 10000 + minor * 100 + patch). */
DSA_API int dsa_version(void);

/* Human-readable name of a status code (static string). */
DSA_API const char *dsa_status_string(dsa_status_t status);

/* The last CUDA error a call of this library met on the calling thread (a
 * failed launch or kernel attribute), as "where: message (code)"; an empty
 * string when there was none.  The text behind a DSA_ERR_CUDA status.  Valid
 * until the thread's next failing call. */
DSA_API const char *dsa_last_cuda_error(void);

/* Bytes of device workspace `op` needs for these dims and cache.  Every
 * workspace starts with a 256-byte status block; the rest is scratch whose
 * contents are undefined between calls.  The status block also holds the
 * indexer's work counter (CTAs take part of the key tiles from it), which
 * every indexer launch leaves at zero: a workspace serves one call at a time,
 * so calls that share one are queued on one stream.  Returns 0 for invalid
 * input. */
DSA_API size_t dsa_workspace_bytes(dsa_op_t op, const dsa_dims_t *dims, const dsa_cache_t *cache);

/* Number of kernels one dsa_attention_forward (op = DSA_OP_ATTENTION_FORWARD),
 * dsa_attention_forward_k8 (DSA_OP_ATTENTION_FORWARD_K8) or
 * dsa_attention_forward_fp8 (DSA_OP_ATTENTION_FORWARD_FP8) call launches for
 * these dims and cache on the current device: the indexer (plus the E4M3
 * query split for FP8 keys), the top-k, the sparse MLA, and the split merge
 * when a row's partial results meet in global memory.  A query of the launch
 * plan with no counterpart on the pages; launches nothing.  Returns -1 for
 * invalid input. */
DSA_API int32_t dsa_forward_launches(dsa_op_t op, const dsa_dims_t *dims, const dsa_cache_t *cache);

/* Clear the status block of a workspace (asynchronous on `stream`).  Call it
 * once after allocating a workspace and after reading an error. */
DSA_API dsa_status_t dsa_workspace_init(void *ws, size_t ws_bytes, dsa_stream_t stream);

/* Wait for `stream`, then read the status block: DSA_OK, DSA_ERR_TIMEOUT or
 * DSA_ERR_DEVICE_CHECK.  `info` (may be NULL) receives the first recorded
 * event code.  Synchronous. */
DSA_API dsa_status_t dsa_workspace_check(const void *ws, dsa_stream_t stream, uint32_t *info);

/* Step 1 - indexer scores ("GLM on an A100, in Vx", "The model"; ReLU per
 * indexer head from "How do we know it is right?").
 *   q_idx        [n_q, H_I, D_I] bf16
 *   w            [n_q, H_I]      fp32 head weights (any 1/sqrt scale folded in)
 *   k_idx_pages  [num_pages, 64, D_I] bf16, rows 16-byte aligned
 *   scores       [n_q, ld] fp32 output; entry (r, s) is written for every
 *                token s the row sees (s < seq_lens[r], or s <= q_pos0 + r);
 *                entries past that are left untouched.  ld >= max tokens seen,
 *                multiple of 4.
 * Uses tcgen05 tensor-core tiles fed by TMA; exact for integer-valued inputs
 * whose partial sums stay below 2^24. */
DSA_API dsa_status_t dsa_indexer_scores(const uint16_t *q_idx, const float *w,
                                const uint16_t *k_idx_pages, const dsa_cache_t *cache,
                                const dsa_dims_t *dims, float *scores, int64_t ld,
                                void *ws, size_t ws_bytes, dsa_stream_t stream);

/* Step 2 - exact top-k with the stable lower-index tie rule ("GLM on an A100,
 * in Vx", "The model" and "How do we know it is right?").
 *   scores     [n_q, ld] fp32; row r uses its first len(r) entries, where
 *              len(r) = valid_len[r] if valid_len != NULL, else causal_base + r + 1
 *              (clamped to [0, ld]).  -0.0 and +0.0 compare equal; NaN is undefined.
 *   idx        [n_q, k] int32 output: kept positions ascending, -1 padded.
 * Scores are read, never modified. */
DSA_API dsa_status_t dsa_topk(const float *scores, int64_t ld, int32_t n_q, const int32_t *valid_len,
                      int32_t causal_base, int32_t k, int32_t *idx, void *ws, size_t ws_bytes,
                      dsa_stream_t stream);

/* Step 3 - absorbed MLA decode over the kept latent rows ("Self-contained
 * GLM-5 serving stack ...", file list and GPU-code paragraph).
 *   q            [n_q, H, R + P] bf16 absorbed queries, rows 16-byte aligned
 *   latent_pages [num_pages, 64, R + P] bf16
 *   idx          [n_q, topk] int32 token positions (-1 = unused slot); a position
 *                outside the row's context is skipped and flagged on the device.
 *                Row r reads only its first min(topk, len(r)) slots, len(r) the
 *                number of tokens the row sees (a row keeps at most that many;
 *                dsa_topk emits them first, then -1)
 *   out          [n_q, H, R] fp32, lse [n_q, H] fp32 (natural log).  A row with
 *                no kept token gets out = 0 and lse = -inf.
 * Precision: bf16 products of q and the latent rows, accumulated in fp32; the
 * softmax weights enter the PV product as two bf16 terms (hi + lo, about 16
 * significant bits). 
 * dims.causal must be 0; row b reads sequence b of the cache. */
DSA_API dsa_status_t dsa_sparse_mla_decode(const uint16_t *q, const uint16_t *latent_pages,
                                   const dsa_cache_t *cache, const int32_t *idx,
                                   const dsa_dims_t *dims, float *out, float *lse,
                                   void *ws, size_t ws_bytes, dsa_stream_t stream);

/* Step 3 for causal prefill rows: as dsa_sparse_mla_decode with dims.causal == 1;
 * every row reads sequence 0 of the cache and may only keep tokens <= q_pos0 + t. */
DSA_API dsa_status_t dsa_sparse_mla_prefill(const uint16_t *q, const uint16_t *latent_pages,
                                    const dsa_cache_t *cache, const int32_t *idx,
                                    const dsa_dims_t *dims, float *out, float *lse,
                                    void *ws, size_t ws_bytes, dsa_stream_t stream);

/* The whole step: indexer scores -> exact top-k -> sparse MLA, one call, all
 * launches on `stream`.  idx_out [n_q, topk] (may be NULL) receives the kept
 * positions; out/lse as above.  Bit-identical to calling the three steps in
 * order with the same workspace sizes. */
DSA_API dsa_status_t dsa_attention_forward(const uint16_t *q_idx, const float *w,
                                   const uint16_t *k_idx_pages, const uint16_t *q,
                                   const uint16_t *latent_pages, const dsa_cache_t *cache,
                                   const dsa_dims_t *dims, int32_t *idx_out, float *out,
                                   float *lse, void *ws, size_t ws_bytes, dsa_stream_t stream);

/* The whole step with host buffers, for callers whose per-step inputs and
 * results live in host memory.  On `stream`, in order: the inputs are copied
 * into the workspace, the step runs (as dsa_attention_forward), the results are
 * copied back to host memory.  Host buffers the device can address (page-locked
 * and mapped, as pinned allocations are under unified addressing) are moved by
 * one small kernel each way, the SMs reading and writing them over the host
 * link (a copy-engine transfer costs microseconds of latency per buffer);
 * any other host buffer by its own cudaMemcpyAsync, which for pageable memory
 * waits for the host.  A mapped q_h (only the sparse MLA reads it) is copied
 * by a spare warp of every indexer CTA while the keys are scanned, so that its
 * transfer over the host link overlaps the scan.  The call returns once
 * everything is queued: the host
 * results are valid after the stream has passed it (e.g. cudaStreamSynchronize).
 *   q_idx_h [n_q, H_I, D_I] bf16, w_h [n_q, H_I] fp32, q_h [n_q, H, R + P] bf16:
 *             host copies of dsa_attention_forward's inputs (any alignment)
 *   cache_h   as dsa_cache_t, except that seq_lens and block_table point to
 *             HOST memory (4-byte aligned); they are copied with the inputs
 *   k_idx_pages, latent_pages: the device page pools, as dsa_attention_forward
 *   idx_h [n_q, topk] i32 (may be NULL), out_h [n_q, H, R] fp32, lse_h [n_q, H]
 *             fp32: host results
 *   ws        device workspace of dsa_workspace_bytes(DSA_OP_ATTENTION_FORWARD_HOST):
 *             the step's workspace, then the staged inputs and results
 * Errors as dsa_attention_forward; a failed host check copies nothing, and a
 * failed copy returns DSA_ERR_CUDA. */
DSA_API dsa_status_t dsa_attention_forward_host(const uint16_t *q_idx_h, const float *w_h,
                                        const uint16_t *k_idx_pages, const uint16_t *q_h,
                                        const uint16_t *latent_pages, const dsa_cache_t *cache_h,
                                        const dsa_dims_t *dims, int32_t *idx_h, float *out_h,
                                        float *lse_h, void *ws, size_t ws_bytes,
                                        dsa_stream_t stream);

/* FP8 index keys: the indexer, and the whole step, over an index-key cache
 * held as E4M3 bytes with one fp32 scale per token ("GLM on an A100, in Vx",
 * section "INT4, FP8 and BF16": E4M3 bytes with a float32 scale per block;
 * here a block is one token's key).  Key s of a page is dequantized as
 * k_scale[row] * e4m3(k8_pages[row, :]) with row = page * 64 + slot, so
 *   score[r, s] = k_scale[row(s)] * sum_h w[r, h] * max(0, q_idx[r, h] . e4m3(k8[row(s)]))
 * (the scale is taken out of the ReLU and the head sum; a scale must be > 0).
 *   k8_pages  [num_pages, 64, D_I] uint8 E4M3 codes (sign, 4 exponent bits with
 *             bias 7, 3 mantissa bits; 0x7F / 0xFF are NaN), 16-byte aligned
 *   k_scale   [num_pages * 64] fp32, 16-byte aligned
 * Everything else as dsa_indexer_scores / dsa_attention_forward; workspaces
 * from dsa_workspace_bytes(DSA_OP_INDEXER_SCORES_K8 / _ATTENTION_FORWARD_K8).
 * D_I must be 128.  The tensor cores multiply the keys as E4M3 (half the
 * bytes and MMA time of bf16 keys); the query enters as two E4M3 terms,
 * q * 2^s = hi + lo, s a power-of-two scale per (row, head) folded into w, so
 * a query element is carried exactly unless it is nonzero and below about
 * 2^-11 of its head's largest magnitude (then to a multiple of 2^(-9 - s)).
 * Scores are exact whenever the bf16 path's would be, the query elements are
 * so carried and every key scale is a power of two. */
DSA_API dsa_status_t dsa_indexer_scores_k8(const uint16_t *q_idx, const float *w,
                                   const uint8_t *k8_pages, const float *k_scale,
                                   const dsa_cache_t *cache, const dsa_dims_t *dims,
                                   float *scores, int64_t ld, void *ws, size_t ws_bytes,
                                   dsa_stream_t stream);
DSA_API dsa_status_t dsa_attention_forward_k8(const uint16_t *q_idx, const float *w,
                                      const uint8_t *k8_pages, const float *k_scale,
                                      const uint16_t *q, const uint16_t *latent_pages,
                                      const dsa_cache_t *cache, const dsa_dims_t *dims,
                                      int32_t *idx_out, float *out, float *lse, void *ws,
                                      size_t ws_bytes, dsa_stream_t stream);

/* FP8 latent cache: the sparse MLA step, and the whole step with both caches
 * in FP8, over a latent cache held as E4M3 bytes with one fp32 scale per token
 * ("GLM on an A100, in Vx", section "INT4, FP8 and BF16": E4M3 bytes with a
 * float32 scale per block; here a block is one token's whole latent row
 * [c_kv | k_rope]).  Token row `row` = page * 64 + slot stands for
 *   L[row, :] = latent_scale[row] * e4m3(latent8_pages[row, :])
 * and serves as key (all R + P columns) and value (the first R) exactly as a
 * bf16 row does.
 *   latent8_pages [num_pages, 64, R + P] uint8 E4M3 codes, 16-byte aligned
 *   latent_scale  [num_pages * 64] fp32 (finite, any sign), 4-byte aligned
 * Everything else as dsa_sparse_mla_decode / _prefill (workspaces from
 * DSA_OP_SPARSE_MLA_DECODE / _PREFILL) and, for dsa_attention_forward_fp8,
 * as dsa_attention_forward_k8 with the FP8 index keys (workspace from
 * DSA_OP_ATTENTION_FORWARD_FP8, the same size as DSA_OP_ATTENTION_FORWARD_K8).  The kernel widens each gathered E4M3 row to
 * bf16 in shared memory (exact) and applies the token's scale to its logit and
 * to its PV weight, so the latent rows cost 580 bytes per kept token instead
 * of 1,152. */
DSA_API dsa_status_t dsa_sparse_mla_decode_l8(const uint16_t *q, const uint8_t *latent8_pages,
                                      const float *latent_scale, const dsa_cache_t *cache,
                                      const int32_t *idx, const dsa_dims_t *dims, float *out,
                                      float *lse, void *ws, size_t ws_bytes, dsa_stream_t stream);
DSA_API dsa_status_t dsa_sparse_mla_prefill_l8(const uint16_t *q, const uint8_t *latent8_pages,
                                       const float *latent_scale, const dsa_cache_t *cache,
                                       const int32_t *idx, const dsa_dims_t *dims, float *out,
                                       float *lse, void *ws, size_t ws_bytes, dsa_stream_t stream);
DSA_API dsa_status_t dsa_attention_forward_fp8(const uint16_t *q_idx, const float *w,
                                       const uint8_t *k8_pages, const float *k_scale,
                                       const uint16_t *q, const uint8_t *latent8_pages,
                                       const float *latent_scale, const dsa_cache_t *cache,
                                       const dsa_dims_t *dims, int32_t *idx_out, float *out,
                                       float *lse, void *ws, size_t ws_bytes, dsa_stream_t stream);

/* Cache append: write the new tokens' index keys and latent rows into the
 * paged caches, the step in front of the indexer ("Self-contained GLM-5
 * serving stack ...", file list: absorbed MLA decode over compressed
 * request-local KV, which the engine grows by one compressed row per token).
 *   k_idx_new    [n_q, D_I]    bf16 index key of each new token
 *   latent_new   [n_q, R + P]  bf16 latent row ([c_kv | k_rope]) of each new token
 *   k_idx_pages, latent_pages  the page pools, written in place
 * Row r goes to the position the step gives its query: decode row b to
 * position seq_lens[b] - 1 of sequence b (seq_lens already counts it);
 * prefill row t (dims.causal = 1) to position q_pos0 + t of sequence 0.
 * Position s of a sequence lives in page block_table[seq][s / 64], slot
 * s % 64.  A page id outside [0, num_pages) or a position outside the block
 * table skips that row and is reported as DSA_ERR_DEVICE_CHECK by the next
 * dsa_workspace_check.  Distinct rows must target distinct slots.  Only
 * dims.n_q, D_I, R, P, causal and q_pos0 are used.  Launched with
 * programmatic dependent launch, so a following dsa_attention_forward on the
 * same stream starts its prologue while the append finishes. */
DSA_API dsa_status_t dsa_cache_append(const uint16_t *k_idx_new, const uint16_t *latent_new,
                              uint16_t *k_idx_pages, uint16_t *latent_pages,
                              const dsa_cache_t *cache, const dsa_dims_t *dims, void *ws,
                              size_t ws_bytes, dsa_stream_t stream);

/* Workspace of the entry points that need only the status block
 * (dsa_absorb_query, dsa_project_values; also what dsa_workspace_bytes returns
 * for DSA_OP_INDEXER_SCORES, DSA_OP_TOPK and DSA_OP_CACHE_APPEND). */
#define DSA_STATUS_WORKSPACE_BYTES 256

/* Query absorption, the product in front of the logits: the per-head key
 * up-projection folded into the query, so the step scores queries against the
 * compressed latent rows directly ("Self-contained GLM-5 serving stack ...",
 * file list: absorbed MLA decode over compressed request-local KV).
 *   q_nope  [n_q, H, d_nope] bf16, q_rope [n_q, H, P] bf16 (may be NULL when P = 0)
 *   w_uk    [H, d_nope, R] bf16 (row d of head h maps q_nope[., h, d] onto the R latent columns)
 *   q_abs   [n_q, H, R + P] bf16 output, the step's q:
 *           q_abs[b, h, 0:R] = bf16(sum_d q_nope[b, h, d] * w_uk[h, d, :]) (fp32 accumulate,
 *           round to nearest even), q_abs[b, h, R:] = q_rope[b, h, :]
 * d_nope: multiple of 64, <= 512; R: multiple of 64, <= 512; P: multiple of 16,
 * R + P <= 576; H <= 128.  All pointers 16-byte aligned.  tcgen05 tensor cores
 * (D^T = W^T . q^T per head, the weight tile as the MN-major A operand). */
DSA_API dsa_status_t dsa_absorb_query(const uint16_t *q_nope, const uint16_t *q_rope,
                              const uint16_t *w_uk, uint16_t *q_abs, int32_t n_q, int32_t H,
                              int32_t d_nope, int32_t R, int32_t P, void *ws, size_t ws_bytes,
                              dsa_stream_t stream);

/* Value projection, the product after the split merge: the per-head value
 * up-projection applied to the latent-space output (same pages as above).
 *   o_lat   [n_q, H, R] fp32 (the `out` of the step), 16-byte aligned
 *   w_uv    [H, R, d_v] bf16, 16-byte aligned
 *   v_out   [n_q, H, d_v] fp32 output: v_out[b, h, :] = sum_r o_lat[b, h, r] * w_uv[h, r, :]
 * o_lat enters the tensor cores as two bf16 terms (hi + lo), so its precision
 * is kept to about 2^-17 relative.  R: multiple of 64, <= 512; d_v: multiple of
 * 64, <= 512; H <= 128. */
DSA_API dsa_status_t dsa_project_values(const float *o_lat, const uint16_t *w_uv, float *v_out,
                                int32_t n_q, int32_t H, int32_t R, int32_t d_v, void *ws,
                                size_t ws_bytes, dsa_stream_t stream);

/* Context-parallel decode of one long sequence whose keys are split over
 * ranks (GPUs), the key range of rank i before that of rank i + 1 ("GLM on an
 * A100, in Vx", "The model": contexts of up to 1,048,576 tokens, each query
 * keeping its 2,048 best-scoring earlier tokens).  Each rank runs
 * dsa_indexer_scores and dsa_topk over its own keys (local positions); then
 *   1. dsa_cp_candidates: its kept local positions idx_local [n_q, k] become
 *      (score, global index) pairs cand_scores / cand_idx [n_q, k] (pads:
 *      -inf, -1); offsets [n_q] = the global position of the rank's first key;
 *   2. the caller all-gathers the pairs, rank by rank: all_scores / all_idx
 *      [ranks, n_q, k];
 *   3. dsa_cp_select: the exact global top-k of the pairs (the lower global
 *      index wins ties, as in dsa_topk) into gidx [n_q, k] (ascending, -1
 *      padded), and in own_idx [n_q, k] this rank's share of it as local
 *      positions, ascending, first in the row (-1 after them); my_offsets / my_lens [n_q]
 *      give this rank's key range.  Workspace: dsa_cp_workspace_bytes;
 *   4. dsa_sparse_mla_decode with own_idx over the rank's latent rows, then
 *      the caller all-gathers (out, lse): outs [ranks, n_q, H, dv], lses
 *      [ranks, n_q, H];
 *   5. dsa_cp_merge: out = sum_r exp(lse_r - L) out_r, L = log sum_r
 *      exp(lse_r) (natural log; a rank with no kept token has lse = -inf).
 * The global top-k lies within the union of the local top-ks, so the result
 * is the one-device step's.  Pointers 4-byte aligned; ranks <= 1024. */
DSA_API size_t dsa_cp_workspace_bytes(int32_t ranks, int32_t n_q, int32_t k);
DSA_API dsa_status_t dsa_cp_candidates(const float *scores, int64_t ld, int32_t n_q,
                               const int32_t *idx_local, int32_t k, const int32_t *offsets,
                               float *cand_scores, int32_t *cand_idx, void *ws, size_t ws_bytes,
                               dsa_stream_t stream);
DSA_API dsa_status_t dsa_cp_select(const float *all_scores, const int32_t *all_idx,
                           int32_t ranks, int32_t n_q, int32_t k, const int32_t *my_offsets,
                           const int32_t *my_lens, int32_t *gidx, int32_t *own_idx, void *ws,
                           size_t ws_bytes, dsa_stream_t stream);
DSA_API dsa_status_t dsa_cp_merge(const float *outs, const float *lses, int32_t ranks,
                          int32_t n_q, int32_t H, int32_t dv, float *out, float *lse, void *ws,
                          size_t ws_bytes, dsa_stream_t stream);

/* Sparse MLA decode for callers that cannot allocate device memory.
 *
 * The pages have no counterpart of this entry point: it exists for callers
 * that cannot call cudaMalloc (or any allocator) at the point where they run
 * the step, e.g. code inside a memory pool that must not grow, or a host that
 * hands the library only its input and output buffers.  It computes what
 * dsa_sparse_mla_decode computes, always with the pipelined kernel that call
 * uses for large batches (results agree within the step's tolerance), and
 * takes no workspace: its scratch (the
 * per-split partial results and a status block) is a fixed 16 MiB array in
 * the library's own device memory, present on every GPU that loads the
 * library until the process exits.
 *
 *   Arguments as for dsa_sparse_mla_decode, without ws / ws_bytes.
 *   Returns DSA_ERR_WORKSPACE, before launching anything, when the partial
 *   results of this call would not fit in the 16 MiB array.  Partials exist
 *   only when few rows hold long selections: each row is then split over more
 *   CTAs than one cluster holds, and every split leaves n_q * splits * 64 *
 *   R' * 4 bytes (R' = R rounded up to a multiple of 128).  One row of
 *   top-8,192 (64 splits, 8.4 MB) fits; two rows of top-65,536 (64 splits
 *   each, 16.8 MB) are rejected.  Rows split over one cluster (e.g. a batch of
 *   32 at top-2,048) or not split at all need only the status block.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  All calls on a device share the one array, and it keeps the last
 * call's contents: calls whose executions overlap on the GPU (different
 * streams, or different host threads) race on it and must be ordered by the
 * caller.  Device-side range-check events (a token index or page id out of
 * range) and bounded-wait time-outs of this call are recorded in the array's
 * status block, which is cleared at the start of every call; read it back
 * with dsa_noalloc_status() after the call.
 * Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call. */
DSA_API dsa_status_t dsa_sparse_mla_decode_noalloc(const uint16_t *q, const uint16_t *latent_pages,
                                           const dsa_cache_t *cache, const int32_t *idx,
                                           const dsa_dims_t *dims, float *out, float *lse,
                                           dsa_stream_t stream);

/* The device-side status of the last dsa_sparse_mla_decode_noalloc call on the
 * current device (the status block of its built-in array), read on `stream`:
 * synchronises `stream`, then returns DSA_OK, DSA_ERR_DEVICE_CHECK (an index
 * or page id was out of range and skipped) or DSA_ERR_TIMEOUT (a bounded wait
 * gave up), with the first event's code in *info when info is not NULL.
 * Like the entry point it has no counterpart on the pages, and allocates
 * nothing (one 256-byte device-to-host copy into the caller's stack). */
DSA_API dsa_status_t dsa_noalloc_status(dsa_stream_t stream, uint32_t *info);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
