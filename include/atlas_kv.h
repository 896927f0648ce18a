/*
 * atlas_kv.h -- C ABI of the paged FP8 KV-cache decode / MTP-verify attention
 * library for NVIDIA B200 (sm_100a).  Library: libatlas_kv.so.
 *
 * What the library computes.  The Atlas pages describe an inference engine
 * with a "paged FP8 KV cache" and multi-token-prediction (MTP, K = 4 drafts)
 * verification (GB10 page: "Atlas Takes On vLLM With a Pure Rust/CUDA
 * Inference Engine on a Single GB10", deployment-path paragraph), a memory
 * pool of fixed-size preallocated blocks for the KV cache (Atlas deep-dive,
 * ainews.cool, "Memory architecture" paragraph), FP8 quantisation with scale
 * factors (same page, "Quantisation" paragraph) and dedicated MQA/GQA
 * attention kernels of the FlashAttention-2 family (same page, "Attention"
 * paragraph).  The pages fix no layout, page size, scale granularity,
 * rounding or mask convention; the readings used here are:
 *
 *   pages        uint8 E4M3 codes; K pages token-major
 *                [num_pages][num_kv_heads][page_size][head_dim], and with
 *                head_dim 128 each 128-byte token row stores its 16-byte
 *                chunk j (dims 16j..16j+15) at chunk position j XOR (slot % 8)
 *                (the tensor cores' 128-byte swizzle, so pages are copied
 *                into shared memory verbatim); V pages in 16-slot groups,
 *                head-dim-major inside a group:
 *                [num_pages][num_kv_heads][page_size/16][head_dim][16], slot t
 *                of a group at byte 4*((t%8)/2) + 2*(t/8) + t%2
 *   block table  int32 [batch][max_blocks_per_seq]; token p of sequence b is in
 *                page block_table[b][p / page_size], slot p % page_size
 *   scales       one float32 per KV head for K and one for V (static)
 *   encode       code = E4M3(fp32(x) / fp32(scale[h])), IEEE division, round to
 *                nearest even, |y| >= 448 saturates to +-448, sign of zero kept
 *   q, out       bf16 [batch][q_len][num_q_heads][head_dim]; q-head hq reads KV
 *                head hq / (num_q_heads / num_kv_heads)
 *   seq_lens     context length of each sequence INCLUDING the q_len new tokens,
 *                whose K/V must already be appended
 *   mask         new row i (0-based) sees key positions t <= seq_len - q_len + i
 *   softmax      s = sm_scale * q . k, fp32 online softmax, fp32 accumulation,
 *                bf16 output (round to nearest even); sm_scale <= 0 means
 *                1/sqrt(head_dim)
 *
 * Ownership.  Every buffer is owned by the caller; the library stores
 * pointers and never allocates or frees device memory.  A pool handle is
 * owned by the caller from atlas_kv_pool_create until atlas_kv_pool_destroy.
 *
 * Streams.  Every compute entry point only enqueues work on the given stream
 * (a cudaStream_t passed as void*; NULL = legacy default stream) and returns
 * without synchronising.  Only atlas_get_device_error synchronises.
 *
 * Errors.  Arguments are checked on the host before anything is enqueued;
 * a failed check returns a negative status and enqueues nothing.  Checks
 * that need device data (page ids inside the block table, per-sequence
 * lengths, append positions) are made by the kernels: an offending page or
 * sequence is skipped (its output rows are written as zeros or left
 * untouched, as documented per call) and a bit is set in the pool's device
 * error word, read with atlas_get_device_error.  No kernel traps.
 *
 * Threads.  A pool is immutable after creation except for its workspace.
 * Decode calls that share one pool share its workspace, so they must be
 * issued on one stream (or otherwise ordered); appends only set bits of the
 * workspace's error word.
 */
#ifndef ATLAS_KV_H
#define ATLAS_KV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATLAS_API __attribute__((visibility("default")))
#else
#define ATLAS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct atlas_kv_pool atlas_kv_pool_t;   /* opaque host-side descriptor */

typedef enum {
    ATLAS_OK = 0,
    ATLAS_ERR_INVALID_ARG = -1,   /* null pointer, bad size or alignment        */
    ATLAS_ERR_UNSUPPORTED = -2,   /* a shape this build has no kernel for       */
    ATLAS_ERR_WORKSPACE = -3,     /* workspace too small for the call           */
    ATLAS_ERR_CUDA = -4,          /* a CUDA runtime call failed                 */
    ATLAS_ERR_DEVICE_CHECK = -5   /* atlas_get_device_error found a device flag */
} atlas_status_t;

typedef enum { ATLAS_DTYPE_F32 = 0, ATLAS_DTYPE_BF16 = 1 } atlas_dtype_t;

/* Bits of the device error word. */
#define ATLAS_DEVERR_PAGE_ID   0x1   /* decode: block-table entry outside [0, num_pages) */
#define ATLAS_DEVERR_SEQ_LEN   0x2   /* decode: seq_len < q_len, > max_seq_len or > table */
#define ATLAS_DEVERR_APPEND    0x4   /* append: position or page id out of range          */
#define ATLAS_DEVERR_TIMEOUT   0x8   /* decode: a bounded wait for staged K/V ran out      */

/* Fields of atlas_paged_gqa_decode_plan's output array. */
#define ATLAS_PLAN_SPLIT_TOKENS  0   /* KV tokens per split / per CTA range           */
#define ATLAS_PLAN_NUM_SPLITS    1   /* splits (grid) or most ranges (balanced) of a  */
                                     /* max-length segment                            */
#define ATLAS_PLAN_KERNEL        2   /* 1 = FP8 warp-MMA kernel (mma.sync E4M3), grid */
                                     /* partition; 2 = the same, balanced partition;  */
                                     /* 3 = 5th-generation tensor-core kernel         */
                                     /* (tcgen05.mma, TMEM accumulators), grid        */
#define ATLAS_PLAN_ROWS_PER_CTA  3   /* query rows (q_len x group) per segment        */
#define ATLAS_PLAN_ROW_BLOCKS    4   /* segments per (sequence, KV head)              */
#define ATLAS_PLAN_LAUNCHES      5   /* kernel launches per decode call               */
#define ATLAS_PLAN_GRID_CTAS     6   /* CTAs launched                                 */
#define ATLAS_PLAN_FIELDS        7

/*
 * Bytes of workspace a pool needs so that decode calls with batch <=
 * max_batch, q_len <= max_q_len, the given head counts and head_dim and
 * max_seq_len <= max_seq_len fit with the automatic partition, and -- when
 * min_split_tokens > 0 -- with any split override >= min_split_tokens.
 * The workspace holds the split-KV partial results (float32 O rows and
 * log2-sum-exp values: one slot per split of every segment with the grid
 * partition, one per segment plus one per CTA with the balanced one), one
 * completion counter per segment (sequence, KV head, row block) and the
 * device error word.  The figure depends on the SM count of the current device (148 if
 * none is visible).  Returns 0 for invalid arguments.
 */
ATLAS_API size_t atlas_kv_workspace_bytes(int32_t max_batch, int32_t max_q_len,
                                          int32_t num_q_heads, int32_t num_kv_heads,
                                          int32_t head_dim, int32_t max_seq_len,
                                          int32_t min_split_tokens);

/*
 * Describe a page pool.  num_pages >= 1; page_size a multiple of 16 and
 * <= 1024; head_dim 64 or 128; num_kv_heads >= 1.  k_pages: device uint8
 * [num_pages][num_kv_heads][page_size][head_dim] (token-major; chunk-permuted
 * rows when head_dim is 128, see the page layout above); v_pages:
 * device uint8 [num_pages][num_kv_heads][page_size/16][head_dim][16] (16-slot
 * groups, head-dim-major inside a group); both 16-byte aligned.
 * k_scale / v_scale: device float32 [num_kv_heads] (used by append; decode
 * takes its own scale pointers).  max_batch, max_q_len, num_q_heads bound the
 * decode calls (they size the counter region).  workspace: device memory of
 * workspace_bytes >= atlas_kv_workspace_bytes(...), 256-byte aligned and
 * ZERO-FILLED by the caller before the first call; the library keeps its
 * counters at zero between calls.  No CUDA call is made here.
 */
ATLAS_API atlas_status_t atlas_kv_pool_create(atlas_kv_pool_t** pool, int32_t num_pages,
                                    int32_t page_size, int32_t num_kv_heads,
                                    int32_t head_dim, void* k_pages, void* v_pages,
                                    const float* k_scale, const float* v_scale,
                                    int32_t max_batch, int32_t max_q_len,
                                    int32_t num_q_heads, void* workspace,
                                    size_t workspace_bytes);

/* Free the host-side descriptor (not the caller's buffers).  NULL is a no-op. */
ATLAS_API atlas_status_t atlas_kv_pool_destroy(atlas_kv_pool_t* pool);

/*
 * Override the split length of later decode calls: splits of split_tokens KV
 * tokens (grid partition), or CTA ranges of about split_tokens tokens
 * (balanced partition: ceil(units / (split_tokens / 32)) CTAs, where units
 * counts 32-token units as if every sequence were max_seq_len long); 0
 * restores the automatic choice.  Must be 0 or a multiple of 64 in [64, 8192].
 * Meant for tuning and for split-invariance tests.
 */
ATLAS_API atlas_status_t atlas_kv_pool_set_split_tokens(atlas_kv_pool_t* pool, int32_t split_tokens);

/* Tuning options for atlas_kv_pool_set_option. */
#define ATLAS_OPT_SPLIT_TOKENS   1   /* same as atlas_kv_pool_set_split_tokens           */
#define ATLAS_OPT_STAGES         2   /* K/V staging depth per stream: 0 = auto, 2 or 3   */
                                     /* (tensor-core kernel: depth of the K ring, auto 3; */
                                     /* its V ring always has 2 stages)                  */
#define ATLAS_OPT_WAVES          3   /* automatic sizing, 0 = 1, up to 8: balanced: CTAs */
                                     /* per resident CTA slot; grid: splits sized for     */
                                     /* 2 x this many waves of resident CTAs; more, smaller */
                                     /* parts need more partial slots in the workspace    */
                                     /* (ATLAS_ERR_WORKSPACE if they do not fit)          */
#define ATLAS_OPT_PARTITION      4   /* 0 = auto, 1 = grid (CTA = one split of one      */
                                     /* (sequence, KV head, row block); the hardware     */
                                     /* schedules them), 2 = balanced (equal ranges of   */
                                     /* 32-token units per CTA); auto takes balanced     */
                                     /* only when one K/V stream serves a whole CTA      */
#define ATLAS_OPT_ROWS_PER_CTA   5   /* query rows one CTA serves: 0 = auto (the fewest */
                                     /* of 4, 8, 16, 32, 64 holding q_len * G), else one */
                                     /* of those; fewer rows make more row blocks, each  */
                                     /* streaming the KV head's pages again              */
#define ATLAS_OPT_KERNEL         8   /* 0 = auto (the tensor-core kernel when head_dim  */
                                     /* is 128 and q_len * G >= 16, where QK^T and PV   */
                                     /* are real contractions), 1 = FP8 warp-MMA kernel, */
                                     /* 2 = tensor-core kernel (head_dim 128 only, else  */
                                     /* ATLAS_ERR_UNSUPPORTED); the tensor-core kernel   */
                                     /* runs blocks of 64 query rows in the grid         */
                                     /* partition (ATLAS_OPT_PARTITION and              */
                                     /* ATLAS_OPT_ROWS_PER_CTA do not apply to it)      */
#define ATLAS_OPT_WAIT_LIMIT_US  6   /* limit of every bounded wait inside the decode  */
                                     /* kernel, in microseconds: 0 = the default        */
                                     /* (200 ms), else 1 .. 10^7.  Counted in SM cycles */
                                     /* at 2 per ns: at least this long at any SM clock */
                                     /* up to 2 GHz, longer at a lower clock            */
#define ATLAS_OPT_TEST_SKIP_UNIT 7   /* TESTS ONLY: -1 = off (default); k >= 0 = the     */
                                     /* first K/V stream of CTA 0 never issues the copies */
                                     /* of its k-th unit (tensor-core kernel: of its k-th */
                                     /* 128-token tile), so the wait for them runs out:  */
                                     /* the call flags ATLAS_DEVERR_TIMEOUT, the output   */
                                     /* rows of the affected (sequence, KV head) are      */
                                     /* unspecified, every other one is computed, and no  */
                                     /* copy is left in flight.  Exercises the bounded-   */
                                     /* wait error path without any fault                 */

/*
 * Set a tuning option of later decode calls (see ATLAS_OPT_*).  Values out of
 * range return ATLAS_ERR_INVALID_ARG and change nothing.
 */
ATLAS_API atlas_status_t atlas_kv_pool_set_option(atlas_kv_pool_t* pool, int32_t option,
                                                  int32_t value);

/*
 * FP8 page append (quantise + scatter), the cache-fill step.
 * k_new / v_new: device [batch][n_new][num_kv_heads][head_dim] of dtype
 * (float32 or bf16), 16-byte aligned.  block_table: device int32
 * [batch][max_blocks_per_seq].  start_pos: device int32 [batch], position of
 * the first new token of each sequence.  Token t of sequence b is written to
 * position start_pos[b] + t with code E4M3(fp32(x) / fp32(scale[h])) using the
 * pool's k_scale / v_scale; the result is bit-exact with that definition.
 * Rows whose position is negative, past max_blocks_per_seq*page_size, or
 * whose page id is outside [0, num_pages) are skipped and flag
 * ATLAS_DEVERR_APPEND.  batch == 0 or n_new == 0 is a no-op.
 */
ATLAS_API atlas_status_t atlas_fp8_kv_append(const atlas_kv_pool_t* pool, const void* k_new,
                                   const void* v_new, int32_t dtype,
                                   const int32_t* block_table, int32_t max_blocks_per_seq,
                                   const int32_t* start_pos, int32_t batch, int32_t n_new,
                                   void* stream);

/*
 * Fused rotary embedding + FP8 quantise + paged append from the QKV
 * projection output of the new tokens (Atlas deep-dive, ainews.cool, "Kernel
 * fusion" paragraph: per-block steps fused into one kernel).  qkv: device
 * bf16 [batch][n_new][num_q_heads + 2 * num_kv_heads][head_dim] (per token:
 * the query heads, then the key heads, then the value heads), 16-byte
 * aligned.  cos_sin: device float32 [max_pos][head_dim], cos of the rotation
 * angles in columns 0 .. head_dim/2 - 1 and sin in the rest.  Token t of
 * sequence b has position start_pos[b] + t (device int32 [batch]).  Query and
 * key heads are rotated "rotate half" style (element i < head_dim/2 with
 * i + head_dim/2: out[i] = x[i] c - x[i+D/2] s, out[i+D/2] = x[i+D/2] c +
 * x[i] s) in float32 with every product and sum rounded separately; the
 * rotated queries are written to q_out (device bf16
 * [batch][n_new][num_q_heads][head_dim], round to nearest even), the rotated
 * keys and the values are quantised and written into the pool's pages exactly
 * as atlas_fp8_kv_append does.  Bit-exact with that definition.  A token whose
 * position is outside [0, max_pos) is skipped entirely (its q_out rows are
 * left unwritten); a position past the block table or a bad page id skips
 * that token's K and V rows; both flag ATLAS_DEVERR_APPEND.  batch == 0 or
 * n_new == 0 is a no-op.
 */
ATLAS_API atlas_status_t atlas_rope_fp8_kv_append(const atlas_kv_pool_t* pool, const void* qkv,
                                                  int32_t num_q_heads, const float* cos_sin,
                                                  int32_t max_pos, const int32_t* block_table,
                                                  int32_t max_blocks_per_seq,
                                                  const int32_t* start_pos, int32_t batch,
                                                  int32_t n_new, void* q_out, void* stream);

/*
 * Finer-grained FP8 scales (Atlas deep-dive, ainews.cool, "Quantisation"
 * paragraph: FP8 with per-group scale factors; here the finest group, one
 * token's row of one KV head).  The same append as atlas_fp8_kv_append, but
 * each new token's K row and V row of each KV head get their own dynamic scale
 * s = fp32(max |x|) / fp32(448) (IEEE division; 1.0 for an all-zero row) and
 * code = E4M3(fp32(x) / s); the scales are stored at [page][head][slot] of
 * k_tok_scale / v_tok_scale (device float32 [num_pages][num_kv_heads]
 * [page_size], caller-owned, 16-byte aligned), and v_scale_bound (device
 * float32 [num_kv_heads], caller-owned, zero before the first append of the
 * cache) is raised to the largest V scale appended per head.  The pool's
 * per-head scales are not used.  Bit-exact with that definition.
 */
ATLAS_API atlas_status_t atlas_fp8_kv_append_tokscale(
    const atlas_kv_pool_t* pool, const void* k_new, const void* v_new, int32_t dtype,
    const int32_t* block_table, int32_t max_blocks_per_seq, const int32_t* start_pos,
    int32_t batch, int32_t n_new, float* k_tok_scale, float* v_tok_scale, float* v_scale_bound,
    void* stream);

/*
 * Decode / verify over a cache filled by atlas_fp8_kv_append_tokscale: K is
 * dequantised with its per-token scales (applied to the scores), V with its
 * per-token scales (applied to the probabilities, relative to v_scale_bound
 * so that they stay in E4M3 range).  head_dim 128 only (the tensor-core
 * kernel; ATLAS_ERR_UNSUPPORTED otherwise).  Uses the pool's pages; other
 * arguments and errors as atlas_paged_gqa_decode.
 */
ATLAS_API atlas_status_t atlas_paged_gqa_decode_tokscale(
    const atlas_kv_pool_t* pool, const void* q, const float* k_tok_scale,
    const float* v_tok_scale, const float* v_scale_bound, const int32_t* block_table,
    int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t batch, int32_t num_q_heads,
    int32_t q_len, int32_t max_seq_len, float sm_scale, void* out, void* stream);

/*
 * Paged decode (q_len == 1) / MTP-verify (q_len > 1) grouped-query attention.
 * q: device bf16 [batch][q_len][num_q_heads][head_dim], 16-byte aligned.
 * k_pages / v_pages: the pool's page arrays (or arrays of identical shape).
 * k_scale / v_scale: device float32 [num_kv_heads].  block_table: device
 * int32 [batch][max_blocks_per_seq]; only the first ceil(seq_len/page_size)
 * entries of a row are read.  seq_lens: device int32 [batch].
 * max_seq_len: host upper bound of seq_lens (bounds the work of one CTA).
 * out: device bf16 [batch][q_len][num_q_heads][head_dim], 16-byte aligned.
 * A sequence with seq_len < q_len, seq_len > max_blocks_per_seq*page_size or
 * seq_len > max_seq_len gets zero output rows and flags ATLAS_DEVERR_SEQ_LEN;
 * a page id outside [0, num_pages) is skipped (its tokens do not take part)
 * and flags ATLAS_DEVERR_PAGE_ID.  batch == 0 is a no-op.  Uses the pool workspace.
 * Partition (ATLAS_OPT_PARTITION): each (sequence, KV head, row block)
 * segment is cut into splits of a fixed number of tokens, one CTA each, that
 * the hardware hands to SMs as they free up (the tensor-core kernel's CTAs
 * take these splits longest first, ranked in the kernel from seq_lens); or
 * the 32-token units of all segments are cut into equal ranges, one per CTA,
 * whatever the length mix.
 * A segment cut in several parts is merged by log-sum-exp by the CTA that
 * finishes it last.  A wait that runs out (200 ms) flags ATLAS_DEVERR_TIMEOUT.
 */
ATLAS_API atlas_status_t atlas_paged_gqa_decode(const atlas_kv_pool_t* pool, const void* q,
                                      const void* k_pages, const void* v_pages,
                                      const float* k_scale, const float* v_scale,
                                      const int32_t* block_table,
                                      int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                      int32_t batch, int32_t num_q_heads, int32_t q_len,
                                      int32_t max_seq_len, float sm_scale, void* out,
                                      void* stream);

/*
 * Ragged verify and chunked prefill over the paged cache: the same attention
 * as atlas_paged_gqa_decode, with a number of new rows per sequence (GB10
 * page: MTP verification at concurrency 1-128, where sequences verify
 * different numbers of drafts; a prefill chunk is the same with many rows).
 * cu_q_lens: device int32 [batch + 1], packed row offsets (cu_q_lens[0] = 0,
 * non-decreasing); sequence b owns rows cu_q_lens[b] .. cu_q_lens[b+1] - 1 of
 * q and out (device bf16 [cu_q_lens[batch]][num_q_heads][head_dim]), its
 * q_len_b = cu_q_lens[b+1] - cu_q_lens[b] may be 0 (nothing written).  New row
 * i of sequence b sees key positions t <= seq_lens[b] - q_len_b + i.
 * max_q_len: host upper bound of every q_len_b (<= the pool's max_q_len; it
 * sizes the row blocks).  The warp-MMA kernel runs the grid partition here.
 * Other arguments and errors as atlas_paged_gqa_decode.
 */
ATLAS_API atlas_status_t atlas_paged_gqa_decode_varlen(
    const atlas_kv_pool_t* pool, const void* q, const int32_t* cu_q_lens, const void* k_pages,
    const void* v_pages, const float* k_scale, const float* v_scale, const int32_t* block_table,
    int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t batch, int32_t num_q_heads,
    int32_t max_q_len, int32_t max_seq_len, float sm_scale, void* out, void* stream);

/*
 * One decode / verify step in one kernel: the FP8 append of the q_len new
 * tokens of every sequence (A0) fused with the attention (A1-A9).  Equivalent
 * to atlas_fp8_kv_append(pool, k_new, v_new, dtype, block_table,
 * max_blocks_per_seq, start_pos = seq_lens - q_len, batch, q_len) followed by
 * atlas_paged_gqa_decode on the pool's pages and scales: the pages end up
 * bit-identical and so does the output.  Every CTA whose split (or range)
 * holds a new token quantises and writes it, then reads it back with the rest.
 * k_new / v_new: device [batch][q_len][num_kv_heads][head_dim] of dtype, 16-byte
 * aligned.  A new token whose page id is outside [0, num_pages) is not written
 * and flags ATLAS_DEVERR_APPEND (and ATLAS_DEVERR_PAGE_ID for the decode).
 * Other arguments and errors as atlas_paged_gqa_decode.
 */
ATLAS_API atlas_status_t atlas_paged_gqa_append_decode(
    const atlas_kv_pool_t* pool, const void* k_new, const void* v_new, int32_t dtype,
    const void* q, const int32_t* block_table, int32_t max_blocks_per_seq,
    const int32_t* seq_lens, int32_t batch, int32_t num_q_heads, int32_t q_len,
    int32_t max_seq_len, float sm_scale, void* out, void* stream);

/*
 * The same decode / MTP-verify attention as atlas_paged_gqa_decode, for callers
 * that cannot allocate device memory for a workspace (code running inside a
 * host framework that owns every allocation and hands over only input and
 * output buffers, or a path that must not touch the allocator).  The pages
 * have no counterpart; this entry point exists for such callers only.
 *
 * No pool and no workspace: the geometry is passed directly, and the scratch
 * (split-KV partials, completion counters, error word) lives in one static
 * device array of 8 MiB per GPU, held from library load until process exit.
 * Nothing here allocates.  Arguments and layouts are those of
 * atlas_paged_gqa_decode plus num_kv_heads, head_dim, page_size and num_pages.
 * Every call shares the array: each call clears the counters and error word
 * on its stream before the launch, and calls that overlap on the GPU race.
 * When the split-KV partials of the automatic partition would not fit, the
 * call runs one CTA per segment (no partials); a call that would then need a
 * segment longer than 65536 tokens returns ATLAS_ERR_WORKSPACE.  The first
 * call on a device looks up the array's address with that device current;
 * make it before any stream capture.  Invalid sequences still get zero rows
 * and bad page ids are skipped, but no error word is reported.
 */
ATLAS_API atlas_status_t atlas_paged_gqa_decode_noalloc(
    const void* q, const void* k_pages, const void* v_pages, const float* k_scale,
    const float* v_scale, const int32_t* block_table, int32_t max_blocks_per_seq,
    const int32_t* seq_lens, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t page_size, int32_t num_pages, int32_t q_len, int32_t max_seq_len,
    float sm_scale, void* out, void* stream);

/*
 * The launch plan a decode call with these arguments would use.  With a CUDA
 * device present it queries the kernel's occupancy (no launch, no memory
 * traffic); without one it reports the plan for a 148-SM GPU.  Writes
 * min(n, ATLAS_PLAN_FIELDS) int32 fields to plan.
 */
ATLAS_API atlas_status_t atlas_paged_gqa_decode_plan(const atlas_kv_pool_t* pool, int32_t batch,
                                           int32_t num_q_heads, int32_t q_len,
                                           int32_t max_seq_len, int32_t* plan, int32_t n);

/*
 * Greedy acceptance of MTP draft tokens, the step after an MTP-verify decode
 * (GB10 page: MTP with K = 4 drafts; the speculative-decoding page,
 * blog.hotdry.top: draft -> verify -> accept).  logits: device
 * [batch][num_drafts + 1][vocab] of dtype (float32 or bf16), finite values;
 * row i scores the token after new position i of the verify step.  drafts:
 * device int32 [batch][num_drafts].  Writes, for every sequence:
 *   targets    device int32 [batch][num_drafts + 1]: first argmax of each row
 *              (ties to the lowest token id)
 *   n_accepted device int32 [batch]: leading drafts equal to their target
 *   next_token device int32 [batch]: targets[b][n_accepted[b]], the token
 *              emitted after the accepted drafts
 * One kernel; each logits row is read once.  Uses batch completion counters
 * of the pool's workspace (zero before and after; issue on the stream of the
 * pool's decode calls).  batch <= the pool's max_batch; batch == 0 is a
 * no-op.  Exact: integer results equal the definition bit for bit.
 */
ATLAS_API atlas_status_t atlas_mtp_greedy_accept(const atlas_kv_pool_t* pool, const void* logits,
                                                 int32_t dtype, int32_t batch,
                                                 int32_t num_drafts, int32_t vocab,
                                                 const int32_t* drafts, int32_t* targets,
                                                 int32_t* n_accepted, int32_t* next_token,
                                                 void* stream);

/*
 * Wait for the stream, read the pool's device error word into *code and
 * clear it (and, if it was set, the completion counters a call that stopped
 * early may have left).  Returns ATLAS_OK if it was zero,
 * ATLAS_ERR_DEVICE_CHECK if not.
 */
ATLAS_API atlas_status_t atlas_get_device_error(const atlas_kv_pool_t* pool, void* stream,
                                      int32_t* code);

/* Static description of a status code. */
ATLAS_API const char* atlas_status_string(atlas_status_t status);

/* Library version, e.g. "0.1.0". */
ATLAS_API const char* atlas_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATLAS_KV_H */
