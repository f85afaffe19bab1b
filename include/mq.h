/*
 * mq — quantized-KV decode attention for NVIDIA B200 (sm_100a).
 *
 * A C ABI over hand-written CUDA kernels for the per-token decode step of an
 * inference engine whose KV cache stores keys as int8 and values as int4:
 *
 *   mq_kv_append    quantize-on-append of new K/V tokens into a paged cache
 *   mq_kv_export    cached tokens read back in the codec's canonical packing
 *   mq_decode_attn  attention of a few query tokens per sequence (1 = decode,
 *                   n > 1 = verification of n speculative draft tokens, causal
 *                   among the drafts) against the cache, split over the
 *                   sequence and merged by log-sum-exp
 *   mq_prefill_attn attention of many query tokens per sequence (a prompt or a
 *                   prompt chunk), causal, in tiles of 128 query rows
 *   mq_decode_attn_cascade  the same for sessions sharing a cached prefix: the
 *                   shared pages are read once for all of them
 *   mq_draft_ngram  history-based drafts (the tokens that followed the latest
 *                   earlier occurrence of a sequence's last n tokens), to verify
 *                   with mq_decode_attn
 *   mq_tune         on-device choice of the decode launch shape under a
 *                   wall-clock budget, accepting only bit-identical candidates
 *                   (or, on request, candidates within alpha times the output
 *                   movement of a one-step perturbation of the stored cache),
 *                   with the choice kept in a store file keyed by the device,
 *                   driver, toolchain and library build
 *
 * Where the operations come from.  The blog.123qwe.co.kr deep dive on
 * magnitudedev/magnitude, section 5 ("core mechanism 3: speculative decoding,
 * quantized KV, prefix sharing"), reports the decode attention unit
 * attention_decode_k8v4 with the codec "Key 8-bit, Value 4-bit, group 32, f16
 * scale", the guarantee that verifying several draft tokens costs one decode
 * step because decode is bandwidth-bound, and sessions sharing a prefix cache.
 * Its section 3 ("core mechanism 1: the 60 s first-load tuner") describes the
 * tuner: a 60 s wall-clock budget, candidates measured on the device, a cost
 * summed over serving shapes (4k/64k decode, verification width) weighted by
 * their time at the default configuration, timing passes sized beyond the
 * last-level cache, and results stored and reused by later loads until the
 * driver or toolchain identity changes.  Its section 4 ("core mechanism 2: the
 * precision system") gives the alpha = 8 admission rule.  The paper-digest.app
 * summary ("Core Mechanics") adds that the tuner keeps only configurations that
 * do not change model output.
 *
 * The codec's arithmetic is this library's fixed reading (the pages name the
 * codec only):
 *   K, per (token, kv-head) vector: s = fp16_rn(max|x| / 127), computed as an
 *     IEEE fp32 division then rounded to fp16; code = clamp(rne(x / s), -127,
 *     127) with an IEEE fp32 division; s == 0 gives code 0.
 *   V, per (token, kv-head, 32 consecutive channels): s = fp16_rn(max|x| / 7),
 *     code = clamp(rne(x / s), -8, 7), stored as 4-bit two's complement nibbles,
 *     two per byte.  Which two codes share a byte is the page layout's choice
 *     (below: the codes of one channel for two tokens); mq_kv_export writes the
 *     codec's canonical packing, channel 2j in the low nibble of byte j and
 *     channel 2j + 1 in the high nibble.
 *   Symmetric (no zero point).  NaN inputs give code 0; scales that overflow
 *     fp16 become +inf and give code 0 (inputs beyond 65504*127 for K or
 *     65504*7 for V are outside the codec's domain).
 *
 * Conventions
 *   - Every pointer argument is a DEVICE pointer owned by the caller unless
 *     stated otherwise; the library never frees caller memory.  The opaque
 *     mq_cache handle is a host object allocated by mq_cache_create.
 *   - Every call returns an mq_status and never throws.  Host-side validation
 *     happens before any CUDA call; a failed validation launches nothing.
 *   - Calls that launch work are asynchronous on `stream` (a cudaStream_t; NULL
 *     is the legacy default stream).  Faults inside kernels surface at the next
 *     synchronization; conditions a kernel detects itself (an out-of-range
 *     block id or position, a wait that ran out of time) set a device error
 *     word that mq_device_status() reads and clears.
 *   - A cache handle is not thread-safe; distinct handles are independent.
 */
#ifndef MQ_H
#define MQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (CUDA's runtime stream handle); NULL is the legacy default stream. */
typedef struct CUstream_st* mq_stream;

typedef enum mq_status {
    MQ_OK = 0,
    MQ_ERR_INVALID_ARG = 1,     /* null pointer, bad size or count, inconsistent arguments     */
    MQ_ERR_UNSUPPORTED = 2,     /* head_dim not 128/256, page size not 16, dtype, too many rows  */
    MQ_ERR_CAPACITY = 3,        /* pool too small for n_blocks, max_seq_len beyond the table     */
    MQ_ERR_WORKSPACE = 4,       /* workspace null, too small or misaligned                      */
    MQ_ERR_CUDA = 5,            /* a CUDA runtime call or kernel launch failed                   */
    MQ_ERR_DEVICE = 6,          /* a kernel flagged a bad block id/position/length or a timeout  */
    MQ_TUNE_BUDGET_EXHAUSTED = 7, /* warning: the tuner's budget ran out before every candidate   */
    MQ_ERR_IO = 8               /* the tuning store could not be written                        */
} mq_status;

typedef enum mq_dtype { MQ_F32 = 0, MQ_BF16 = 1, MQ_F16 = 2 } mq_dtype;

/* Tokens per page; fixed. */
#define MQ_PAGE_TOKENS 16

/* ---------------------------------------------------------------------------
 * Cache layout
 *
 * The pool is an array of n_blocks blocks; a block holds MQ_PAGE_TOKENS
 * consecutive token positions of one sequence for every kv-head, as n_kv_heads
 * pages of mq_page_bytes(head_dim) bytes: page (block, h) starts at byte
 * (block * n_kv_heads + h) * mq_page_bytes(head_dim).  A page holds the 16
 * tokens of one (block, kv-head):
 *     K codes   16*D bytes      int8
 *     K scales  16 * 2 bytes    fp16, one per token
 *     V codes   16*D/2 bytes    int4 pairs
 *     V scales  16*D/32 * 2     fp16, one per (token, 32-channel group)
 * = 25*D + 32 bytes (3232 for D = 128, 6432 for D = 256), against 64*D for
 * fp16 K+V: 0.395x (D = 128) and 0.393x (D = 256) — "more than half" smaller,
 * as the trawling.dev Launch HN page (per-device tuning and performance claims)
 * reports for this codec.  The page is laid out for the decode kernel's tensor
 * cores as two records of 8 tokens (tokens 0-7 at byte 0, tokens 8-15 at byte
 * R = 12.5*D + 16; R = 1616 for D = 128, 3216 for D = 256).  In the record of
 * token tau (tt = tau % 8, NG = D/32 groups):
 *     K code of (tau, channel c): byte (c/16)*128 + tt*16 + c%16 — 8-row x
 *       16-byte blocks, so the K codes of consecutive records form one K-major
 *       int8 matrix operand whose 8-token groups are R bytes apart
 *     V codes: one 32-bit word per channel c at byte 8*D + 4*c holding the 8
 *       tokens' 4-bit two's-complement codes, token tt at bit 4*(tt/2) + 16*(tt%2)
 *     K scale of tau: fp16 at byte 12*D + 2*tt
 *     V scale of (tau, group g): fp16 at byte 12*D + 16 + 2*(tt*NG + g)
 * The codes and scales themselves are exactly the codec's.
 *
 * A block_table is int32 [n_seqs][max_blocks_per_seq]: entry [b][i] is the
 * physical block holding positions [16 i, 16 i + 16) of sequence b.  Several
 * sequences may name the same physical block (a shared prefix: the deep dive's
 * section 5 and the Launch HN page describe sessions sharing a prefix cache);
 * the library only reads through block tables and never owns blocks.
 * ------------------------------------------------------------------------- */
typedef struct mq_cache mq_cache;

typedef struct mq_cache_desc {
    int32_t n_kv_heads;   /* >= 1                                                     */
    int32_t head_dim;     /* 128 or 256                                               */
    int32_t page_tokens;  /* must be MQ_PAGE_TOKENS                                   */
    int64_t n_blocks;     /* >= 1                                                     */
    void* pool;           /* device memory, caller-owned, 256-byte aligned            */
    size_t pool_bytes;    /* >= mq_cache_pool_bytes(n_kv_heads, head_dim, n_blocks)   */
} mq_cache_desc;

/* Bytes of one page: 25*head_dim + 32, or 0 for an unsupported head_dim. */
size_t mq_page_bytes(int32_t head_dim);

/* Bytes the pool must hold: n_blocks * n_kv_heads * mq_page_bytes(head_dim)
 * (0 for invalid arguments). */
size_t mq_cache_pool_bytes(int32_t n_kv_heads, int32_t head_dim, int64_t n_blocks);

/* Validates the descriptor and returns a new host handle in *out (which is set
 * to NULL on error).  Binds the handle to the current CUDA device.  Does not
 * touch the pool's contents.  Errors: INVALID_ARG (null, n_kv_heads < 1,
 * n_blocks < 1, misaligned pool), UNSUPPORTED (head_dim, page_tokens),
 * CAPACITY (pool_bytes too small), CUDA. */
mq_status mq_cache_create(const mq_cache_desc* desc, mq_cache** out);

/* Frees the handle (never the pool).  NULL is accepted. */
mq_status mq_cache_destroy(mq_cache* cache);

/* ---------------------------------------------------------------------------
 * mq_kv_append — quantize-on-append
 *
 * Quantizes n_tokens new K/V vectors and writes them into their pages.
 *   k, v         [n_tokens][n_kv_heads][head_dim], dtype `dtype` (F32, BF16 or
 *                F16), packed by sequence in order b = 0 .. n_seqs-1
 *   cu_new       int32 [n_seqs + 1], exclusive prefix sum of the tokens each
 *                sequence appends (cu_new[0] = 0, cu_new[n_seqs] = n_tokens)
 *   start_pos    int32 [n_seqs], the position of sequence b's first new token
 *   block_table  int32 [n_seqs][max_blocks_per_seq] (see above)
 * Token i of sequence b goes to position start_pos[b] + i, i.e. page
 * block_table[b][pos / 16], slot pos % 16.  Two calls (or two tokens) that
 * write the same position race; writing a position of a shared block changes
 * it for every sequence that names the block.
 * Work: one warp per (8-token half page, kv-head) the new tokens touch.  A half
 * page the call covers entirely is written with plain stores; the others (the
 * ragged ends of each sequence's range) replace each 4-bit code with atomic bit
 * operations, so appends split over several calls give the same pages as one.
 * Errors: INVALID_ARG (null pointers, n_seqs < 1 or > 65535, n_tokens < 0,
 * dtype), CUDA.  n_tokens == 0 launches nothing.  A position outside
 * [0, max_blocks_per_seq*16) or a block id outside [0, n_blocks) is skipped by
 * the kernel, and a sequence whose cu_new range leaves [0, n_tokens] is skipped
 * whole (none of its K/V is read); both are reported through mq_device_status()
 * as MQ_ERR_DEVICE.
 * ------------------------------------------------------------------------- */
mq_status mq_kv_append(mq_cache* cache, const void* k, const void* v, mq_dtype dtype, int32_t n_seqs,
                       int32_t n_tokens, const int32_t* cu_new, const int32_t* start_pos,
                       const int32_t* block_table, int32_t max_blocks_per_seq, mq_stream stream);

/* ---------------------------------------------------------------------------
 * mq_kv_export — cached tokens read back in the codec's canonical form
 *
 * The codec (deep dive, section 5: "Key 8-bit, Value 4-bit, group 32, f16
 * scale") packs V codes two per byte; the page layout above groups them by
 * channel for the decode kernel.  This call reads tokens back with V packed
 * channel by channel, as the codec paragraph at the top of this header defines
 * it, and copies codes and scales unchanged (no arithmetic on values): for
 * offloading or inspecting a cache, and for checking it byte for byte.
 *   cu_tok       int32 [n_seqs + 1], exclusive prefix sum of the tokens read per
 *                sequence (like mq_kv_append's cu_new)
 *   start_pos    int32 [n_seqs], position of sequence b's first token read
 *   block_table  int32 [n_seqs][max_blocks_per_seq]
 *   k_codes      out int8   [n_tokens][n_kv_heads][head_dim]
 *   k_scales     out uint16 [n_tokens][n_kv_heads]          (fp16 bits)
 *   v_packed     out uint8  [n_tokens][n_kv_heads][head_dim / 2]: byte j =
 *                (code[2j] & 15) | (code[2j + 1] & 15) << 4
 *   v_scales     out uint16 [n_tokens][n_kv_heads][head_dim / 32] (fp16 bits)
 * All pointers are device pointers owned by the caller; asynchronous on
 * `stream`.  Token i of sequence b is position start_pos[b] + i.  Reading a
 * position no append has written returns whatever the pool holds there.
 * Errors: INVALID_ARG (null pointers, n_seqs < 1 or > 65535, n_tokens < 0,
 * max_blocks_per_seq < 1), CUDA.  n_tokens == 0 launches nothing.  A token
 * outside its sequence's cu_tok range, a position outside [0,
 * max_blocks_per_seq*16) or a block id outside [0, n_blocks) is not read: its
 * outputs are zero and mq_device_status() reports MQ_ERR_DEVICE.
 * ------------------------------------------------------------------------- */
mq_status mq_kv_export(const mq_cache* cache, int32_t n_seqs, int32_t n_tokens, const int32_t* cu_tok,
                       const int32_t* start_pos, const int32_t* block_table, int32_t max_blocks_per_seq,
                       int8_t* k_codes, uint16_t* k_scales, uint8_t* v_packed, uint16_t* v_scales,
                       mq_stream stream);

/* ---------------------------------------------------------------------------
 * mq_decode_attn — attention of n_q_per_seq[b] query tokens of every sequence
 * against its quantized cache
 *
 *   q            [sum_b n_q_per_seq[b]][n_q_heads][head_dim], dtype q_dtype
 *                (F32, BF16 or F16), packed by sequence in order
 *   seq_lens     int32 [n_seqs]: L_b, the tokens in sequence b's cache,
 *                INCLUDING its n_q_per_seq[b] query tokens, whose K/V must
 *                already be appended
 *   n_q_per_seq  int32 [n_seqs]: n_b, 1 <= n_b <= min(L_b, max_q_per_seq)
 *   total_q      host: the rows of q and out (sum_b n_b); a row index at or beyond
 *                it is never read or written (such rows are reported through
 *                mq_device_status())
 *   max_q_per_seq, max_seq_len   host bounds on n_b and L_b (they size the grid)
 *   block_table  int32 [n_seqs][max_blocks_per_seq]
 *   softmax_scale  the logit scale (1/sqrt(head_dim) for standard attention)
 *   out          fp32 [sum_b n_b][n_q_heads][head_dim]
 *   lse          fp32 [sum_b n_b][n_q_heads], natural-log log-sum-exp of the
 *                scaled logits; may be NULL
 *   workspace    device scratch of at least mq_decode_workspace_bytes(...)
 *                bytes, 256-byte aligned, holding the CTA partials of the
 *                split reduction (see mq_decode_workspace_bytes).  It needs no
 *                initialization and can be reused by later calls of any shape
 *                that fits it.  Calls that share a workspace must not overlap.
 *   workspace_bytes  its size; a workspace smaller than the query for this
 *                shape is refused with MQ_ERR_WORKSPACE.
 * Stream order: the kernels are launched as programmatic dependent launches and
 * let the kernel after them start its set-up early.  Every page read and every
 * write waits until the preceding kernel on the stream has completed, but the set-up
 * reads q, block_table, seq_lens and n_q_per_seq before that wait.  When the
 * preceding work on the stream is another mq_decode_attn or mq_kv_append call, these
 * four inputs must not be that call's outputs (e.g. its out used as this call's q).
 * Any other kernel in between restores plain stream order.
 * Query token j of sequence b (0-based) attends to positions 0 .. L_b - n_b + j:
 * the history plus drafts 0..j (causal among the drafts).  q-head h reads
 * kv-head h / (n_q_heads / n_kv_heads).  The result is bit-identical for every
 * launch configuration the tuner may choose under its default admission rule
 * (see mq_tune).
 * Errors: INVALID_ARG (null pointers, n_seqs < 1 or > 65535, n_q_heads not a
 * multiple of n_kv_heads, total_q < 1, max_q_per_seq < 1, max_seq_len <
 * max_q_per_seq, a non-finite softmax_scale, out not 16-byte aligned), UNSUPPORTED
 * (n_q_heads/n_kv_heads * max_q_per_seq > 64, q dtype), CAPACITY (max_seq_len >
 * max_blocks_per_seq * 16), WORKSPACE, CUDA.  A sequence whose L_b / n_b break
 * the bounds above is skipped by the kernel and reported by mq_device_status().
 * ------------------------------------------------------------------------- */
size_t mq_decode_workspace_bytes(const mq_cache* cache, int32_t n_seqs, int32_t n_q_heads, int32_t max_q_per_seq,
                                 int32_t max_seq_len);

/* Number of kernels one mq_decode_attn call with these bounds launches (1 when no
 * unit is split across CTAs, else 2: the decode kernel and the merge of the split
 * partials); 0 for arguments the call would refuse. */
int32_t mq_decode_kernel_count(const mq_cache* cache, int32_t n_seqs, int32_t n_q_heads, int32_t max_q_per_seq,
                               int32_t max_seq_len);

mq_status mq_decode_attn(const mq_cache* cache, const void* q, mq_dtype q_dtype, int32_t n_seqs, int32_t n_q_heads,
                         int32_t total_q, int32_t max_q_per_seq, int32_t max_seq_len, const int32_t* block_table,
                         int32_t max_blocks_per_seq, const int32_t* seq_lens, const int32_t* n_q_per_seq,
                         float softmax_scale, float* out, float* lse, void* workspace, size_t workspace_bytes,
                         mq_stream stream);

/* ---------------------------------------------------------------------------
 * mq_prefill_attn — attention of a prompt's query tokens against the quantized
 * cache (prefill, or a chunk of it)
 *
 * The deep dive (section 3, the first-load tuner) counts 4k and 64k prompt
 * prefill among the serving terms the tuner weighs; the stork.ai page quotes
 * prefill rates.  The arithmetic is mq_decode_attn's, for any number of query
 * tokens per sequence: query token j of sequence b (0-based, n_b of them) attends
 * to positions 0 .. L_b - n_b + j, where L_b counts the prompt's own tokens, whose
 * K/V must already be appended (mq_kv_append).  n_b = L_b is a whole prompt; a
 * smaller n_b is a prompt chunk after a cached history.
 *   q, seq_lens, n_q_per_seq, total_q, block_table, softmax_scale, out, lse
 *                as mq_decode_attn (q packed by sequence; out fp32, lse may be NULL)
 *   max_q_per_seq, max_seq_len   host bounds on n_b and L_b
 * No workspace: one CTA takes a tile of 128 query rows (query token, q-head of a
 * kv-head) over every key its rows see.  Keys enter the tensor cores as exact
 * fp16 codes, q as fp16 scaled by a power of two per row (exact for the BF16 and
 * F16 q this call accepts), values as two fp16 parts hi + lo of code * s_v (about
 * 22 significant bits), the softmax weights as fp16 with l summed from the same
 * rounded weights.  Asynchronous on `stream`, launched as a programmatic
 * dependent launch like mq_decode_attn (see its stream-order note).
 * Errors: those of mq_decode_attn's host checks; UNSUPPORTED for F32 q, head_dim
 * other than 128, or a group size n_q_heads / n_kv_heads that does not divide 128.  A
 * sequence whose L_b / n_b break the bounds is skipped and reported by
 * mq_device_status(), as are unusable block ids (their tokens are masked).
 * ------------------------------------------------------------------------- */
mq_status mq_prefill_attn(const mq_cache* cache, const void* q, mq_dtype q_dtype, int32_t n_seqs, int32_t n_q_heads,
                          int32_t total_q, int32_t max_q_per_seq, int32_t max_seq_len, const int32_t* block_table,
                          int32_t max_blocks_per_seq, const int32_t* seq_lens, const int32_t* n_q_per_seq,
                          float softmax_scale, float* out, float* lse, mq_stream stream);

/* ---------------------------------------------------------------------------
 * mq_decode_attn_static: mq_decode_attn without a caller workspace.
 *
 * The method on the pages has no counterpart to this call; it is a convenience
 * of this library.  It is for callers that cannot give the library a device
 * allocation when they decode: a server that has reserved nearly all free HBM
 * for its KV pool, a C host program with no device allocator of its own, or a
 * decode loop that cannot afford the device synchronization cudaMalloc and
 * cudaFree may cause.  The call allocates nothing.  Its scratch is one fixed
 * array of MQ_DECODE_STATIC_SCRATCH_BYTES (16 MiB) per device inside the
 * library, whose address is looked up on the first call on each device.
 *
 * Arguments, layouts, ownership and results are those of mq_decode_attn,
 * without workspace and workspace_bytes; the outputs equal mq_decode_attn's.
 * The call launches the decode kernels on `stream` with the array as their
 * workspace.
 * Make the first call on each device before any stream capture that is to
 * contain a later call: that first call does the address lookup.  The lookup is
 * repeated when the device's context has changed since (after cudaDeviceReset),
 * so make the first call after a reset outside a capture too.
 * The scratch is shared by every call on a device: calls whose executions may
 * overlap (different streams or host threads without ordering between them)
 * race on it and give wrong results.  Order them, or use mq_decode_attn with a
 * workspace per stream.
 * Errors: those of mq_decode_attn, and WORKSPACE when the shape needs more than
 * MQ_DECODE_STATIC_SCRATCH_BYTES of scratch (mq_decode_workspace_bytes() above
 * that limit); nothing is launched then.
 * ------------------------------------------------------------------------- */
#define MQ_DECODE_STATIC_SCRATCH_BYTES ((size_t)16 << 20)

mq_status mq_decode_attn_static(const mq_cache* cache, const void* q, mq_dtype q_dtype, int32_t n_seqs,
                                int32_t n_q_heads, int32_t total_q, int32_t max_q_per_seq, int32_t max_seq_len,
                                const int32_t* block_table, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                const int32_t* n_q_per_seq, float softmax_scale, float* out, float* lse,
                                mq_stream stream);

/* ---------------------------------------------------------------------------
 * mq_decode_attn_cascade: mq_decode_attn for sessions that share a cached prefix,
 * reading the shared pages once.
 *
 * The pages report concurrent sessions sharing one prefix cache (the deep dive,
 * section 5; trawling.dev "Launch HN: Magnitude", per-device kernel tuning).  With
 * mq_decode_attn every session reads the shared pages again.  Here the step is
 *   1. one pass over the prefix pages for the query tokens of every session together
 *      (no causal mask: every query token of a session already sees its whole prefix),
 *   2. the plain decode over each session's own pages after the prefix, causal among
 *      its drafts as in mq_decode_attn,
 *   3. a merge of the two results per (query token, q-head) by their log-sum-exps:
 *      out = (o1 e^lse1 + o2 e^lse2) / (e^lse1 + e^lse2), lse = log(e^lse1 + e^lse2).
 * The result equals mq_decode_attn's within fp32 rounding (not bit-identical: the
 * summation order differs).
 *
 * Arguments are those of mq_decode_attn plus
 *   prefix_len   tokens of the shared prefix, a positive multiple of 16.  Every
 *                sequence's block table starts with the same prefix_len / 16 blocks
 *                (the caller's promise; the prefix pages are read through row 0), and
 *                every sequence has L_b - n_b >= prefix_len (its queries lie after the
 *                prefix; a sequence that breaks this is skipped and reported by
 *                mq_device_status()).
 *   workspace    at least mq_decode_cascade_workspace_bytes(...) bytes, 256-byte
 *                aligned, no initialization needed; it holds both passes' CTA partials
 *                and the prefix pass's out and lse.
 * Errors: those of mq_decode_attn; INVALID_ARG also for a prefix_len that is not a
 * positive multiple of 16, total_q > prefix_len, max_seq_len - prefix_len <
 * max_q_per_seq, or total_q < max_q_per_seq; UNSUPPORTED when (n_q_heads / n_kv_heads)
 * x total_q > 64 (the prefix pass's query rows per kv-head).
 * Launches: the two decode passes (one or two kernels each) and one merge kernel.
 * ------------------------------------------------------------------------- */
size_t mq_decode_cascade_workspace_bytes(const mq_cache* cache, int32_t n_seqs, int32_t n_q_heads, int32_t total_q,
                                         int32_t max_q_per_seq, int32_t max_seq_len, int32_t prefix_len);

mq_status mq_decode_attn_cascade(const mq_cache* cache, const void* q, mq_dtype q_dtype, int32_t n_seqs,
                                 int32_t n_q_heads, int32_t total_q, int32_t max_q_per_seq, int32_t max_seq_len,
                                 const int32_t* block_table, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                 const int32_t* n_q_per_seq, int32_t prefix_len, float softmax_scale, float* out,
                                 float* lse, void* workspace, size_t workspace_bytes, mq_stream stream);

/* ---------------------------------------------------------------------------
 * mq_draft_ngram: history-based drafting (speculative decoding).
 *
 * The deep dive (section 5, the drafting guarantees) lists history-based drafters
 * among those whose draft step costs only the bytes they read; the drafts are then
 * verified by one mq_decode_attn launch (n_q_per_seq = 1 + the number of drafts).
 * The pages give no algorithm; this library's reading: for each sequence b with
 * history tokens[b][0 .. L_b), find the most recent earlier occurrence of its last
 * `ngram` tokens,
 *   i* = max { i : 0 <= i < L_b - ngram, tokens[b][i + j] == tokens[b][L_b - ngram + j]
 *              for every j < ngram },
 * and propose the tokens that followed it:
 *   drafts[b][j] = tokens[b][i* + ngram + j],  j < n_drafts[b] = min(max_draft, L_b - i* - ngram).
 *   tokens     int32 [n_seqs][max_len] (device), token ids compared as int32 values
 *   seq_lens   int32 [n_seqs] (device), L_b
 *   drafts     int32 [n_seqs][max_draft] (device); entries at or past n_drafts[b]
 *              are not written
 *   n_drafts   int32 [n_seqs] (device): the count, 0 when nothing matches or
 *              L_b <= ngram, -1 when L_b is outside [0, max_len]
 * Runs one kernel on `stream` (the current device); reads each history once.
 * Errors: INVALID_ARG (null pointers, max_len < 1, n_seqs < 1, ngram outside
 * [1, 64], max_draft < 1), CUDA.
 * ------------------------------------------------------------------------- */
mq_status mq_draft_ngram(const int32_t* tokens, int32_t max_len, const int32_t* seq_lens, int32_t n_seqs,
                         int32_t ngram, int32_t max_draft, int32_t* drafts, int32_t* n_drafts, mq_stream stream);

/* ---------------------------------------------------------------------------
 * Launch configuration and tuning
 *
 * The decode kernel cuts every sequence into chunks of 128 tokens; one CTA takes a
 * contiguous range of chunks of one (sequence, kv-head, row block) and the CTA
 * partials are combined by one fixed binary tree over the split index.
 *   ring_stages    2 .. 8: chunks (8 pages each) a CTA keeps in flight, cut
 *                  to what fits in shared memory; never changes the output
 *   splits_per_sm  1, 2 or 4: the split count along the sequence is chosen so
 *                  that about splits_per_sm x (number of SMs) CTAs run.  Row
 *                  blocks of up to 8 rows (one query token per sequence at GQA
 *                  <= 8, head_dim 128; GQA <= 4 at head_dim 256) merge fixed runs
 *                  of chunks over one fixed binary tree whose shape depends on the
 *                  sequence length alone, a CTA taking an aligned power-of-two run
 *                  of them: there the split count never changes the output.  With
 *                  2 to 64 sequences in such a call the CTAs are one flat grid of
 *                  about splits_per_sm x (CTAs per SM) x (number of SMs), and at
 *                  least 4 per (sequence, kv-head) on average (up to 4 per
 *                  CTA slot): the
 *                  device reads every sequence's length and gives each (sequence,
 *                  kv-head) CTAs in proportion to its own length (the run of
 *                  chunks per CTA is the smallest power of two whose CTAs fit).  The
 *                  wider blocks (draft verification) accumulate each CTA's range in
 *                  token order, so there it sets the rounding of the output.
 *   softmax_warps  4 or 8: warps that turn one chunk's scores into weights; with
 *                  8, a block's rows are split over two groups of four (each row's
 *                  arithmetic is the same in either case, so this never changes
 *                  the output).  32-row blocks always use 8 and 4-row blocks 4.
 * The tuner keeps only candidates whose output bytes equal the current
 * configuration's (or, on request, within the alpha rule; see mq_tune).
 * There is one configuration per row class (query rows per kv-head, padded):
 * rows_class 0 = up to 8 rows, 1 = up to 16, 2 = up to 32.
 * ------------------------------------------------------------------------- */
typedef struct mq_decode_config {
    int32_t ring_stages;
    int32_t splits_per_sm;
    int32_t softmax_warps;
} mq_decode_config;

mq_status mq_get_decode_config(const mq_cache* cache, int32_t rows_class, mq_decode_config* cfg);
mq_status mq_set_decode_config(mq_cache* cache, int32_t rows_class, const mq_decode_config* cfg);

/* Admission rules for tuner candidates. */
#define MQ_ADMIT_BIT_IDENTICAL 0  /* out and lse bytes equal the default configuration's       */
#define MQ_ADMIT_ALPHA 1          /* every out and lse point within alpha x storage noise       */

typedef struct mq_tune_params {
    double budget_s;        /* wall-clock budget for everything the tuner does (e.g. 60) */
    int32_t n_q_heads;      /* query heads of the model the cache serves                */
    const char* log_path;   /* host path for the JSON evidence log, or NULL             */
    const char* store_path; /* host path of the persistent tuning store, or NULL        */
    int32_t admission;      /* MQ_ADMIT_BIT_IDENTICAL (0) or MQ_ADMIT_ALPHA             */
    double alpha;           /* the alpha of MQ_ADMIT_ALPHA; <= 0 selects 8              */
} mq_tune_params;

typedef struct mq_tune_result {
    mq_decode_config chosen[3];   /* per rows_class (unchanged if that class was not probed) */
    double cost;                  /* weighted cost of the chosen set (1.0 = the defaults)   */
    int32_t n_tried;              /* candidates measured                                      */
    int32_t n_rejected;           /* candidates the admission rule rejected                   */
    int32_t n_skipped;            /* candidates not reached inside the budget                 */
    double elapsed_s;
    int32_t from_store;           /* 1: the choice was read from the store, nothing measured */
} mq_tune_result;

/* On-device tuner.  Within params->budget_s of wall-clock time (allocation,
 * probe set-up, every measurement included) it measures the candidate launch
 * configurations on three probe shapes built from the cache's geometry and
 * params->n_q_heads — decode at 4K and at 64K tokens, and a speculative step: one
 * mq_draft_ngram launch over a 64K-token history followed by the verification of
 * 8 drafts at 64K — admits candidates by params->admission, and keeps the admitted
 * candidate set with the lowest cost (the deep dive's service cost)
 *     cost(c) = sum_p weight(p) * median_time(c, p),
 *     weight(p) = sum_t launches(t, p) / time_at_defaults(t)
 * over the terms t (decode 4K, decode 64K, the drafter launch, verification of 8
 * drafts, and prompt prefill of 4K and 64K tokens through mq_prefill_attn when the
 * geometry allows it), each of weight 1; reported relative to the defaults' cost.
 * No candidate changes the drafter or prefill launches: their terms are measured
 * once and enter every candidate's cost at that time.
 * The default is the configuration the cache holds when mq_tune is called.
 *
 * Admission.  MQ_ADMIT_BIT_IDENTICAL keeps a candidate only if its out and lse
 * bytes equal the default's on every probe.  MQ_ADMIT_ALPHA keeps it if, at every
 * point i of out and lse on every probe,
 *     |candidate_i - default_i| <= alpha * noise_i,
 * where noise_i, the storage-resolution noise, is how far the default output
 * moves at i when every stored element of the probe cache moves by one step of
 * its format (int8 K code and int4 V code by one code, fp16 scales by one unit in
 * the last place, each in a seeded random direction); noise_i is the larger of
 * two such perturbations.  The rule uses the stored data and its declared types
 * only.  A point whose noise is zero must match exactly.
 *
 * Timed launches read probe caches that together exceed twice the L2 size, so
 * no launch finds its data warm in L2.  The probes use their own device
 * buffers (allocated and freed here; the cache's pool is not touched).  The
 * chosen configurations are stored in the cache handle.  Returns MQ_OK, or
 * MQ_TUNE_BUDGET_EXHAUSTED when the budget ended the search early (the best
 * configuration measured so far is kept; the defaults if none).  Synchronizes
 * the device.  Writes a JSON record of every candidate to params->log_path
 * when it is not NULL.
 *
 * Persistence.  With params->store_path set, the tuner first looks up the
 * identity string of mq_tune_identity() in that store: on a match it applies the
 * stored choice to the cache, measures nothing, sets result->from_store and
 * returns MQ_OK.  Otherwise it searches and, when the search completed (MQ_OK),
 * writes its choice under that identity (a search the budget cut short is not
 * stored, so a later call with more budget searches again); a store that cannot
 * be written gives MQ_ERR_IO after the choice has been applied. */
mq_status mq_tune(mq_cache* cache, const mq_tune_params* params, mq_tune_result* result);

/* The identity a tuning choice is stored under: the GPU's name, SM count and
 * compute capability, the driver version, the CUDA runtime the library was built
 * with, the library version and source build id, the cache geometry (head_dim,
 * n_kv_heads), params->n_q_heads, the admission rule (with alpha), and the
 * configurations the cache holds (the defaults the candidates are compared with).
 * Any change to one of them gives another identity, so the choice is searched
 * again.  Written to buf as a NUL-terminated string of printable characters
 * without tabs; INVALID_ARG if buf_len is too small (512 bytes always suffice).
 * Queries the cache's device; launches nothing. */
mq_status mq_tune_identity(const mq_cache* cache, const mq_tune_params* params, char* buf, size_t buf_len);

/* The tuning store: a text file, one choice per line,
 *     <identity> TAB <r0>:<s0>:<w0> <r1>:<s1>:<w1> <r2>:<s2>:<w2> TAB <cost>
 * (ring_stages:splits_per_sm:softmax_warps of rows_class 0, 1, 2), after a header
 * line starting with '#'.  Host-only file access; no GPU is needed.
 * mq_tune_store_get: *found = 1 and chosen[0..2] set when a well-formed line with
 *   this identity exists (a line whose configurations are out of range counts as
 *   absent); *found = 0 otherwise, a missing or unreadable file included.
 * mq_tune_store_put: writes the file with this identity's line replaced (or
 *   added), every other line kept, through a temporary file in the same directory
 *   renamed over the store, so readers never see a partial file.  IO when the file
 *   cannot be written; INVALID_ARG for an identity holding a tab or newline, or an
 *   out-of-range configuration. */
mq_status mq_tune_store_get(const char* path, const char* identity, mq_decode_config chosen[3], int32_t* found);
mq_status mq_tune_store_put(const char* path, const char* identity, const mq_decode_config chosen[3], double cost);

/* ---------------------------------------------------------------------------
 * Diagnostics
 * ------------------------------------------------------------------------- */
/* Synchronizes `stream`, then reads and clears the device error word of the
 * cache's device: MQ_OK, MQ_ERR_DEVICE (a kernel flagged bad input or a timed
 * out wait since the last call), or MQ_ERR_CUDA. */
mq_status mq_device_status(const mq_cache* cache, mq_stream stream);

/* Static description of a status code. */
const char* mq_status_string(mq_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t mq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MQ_H */
