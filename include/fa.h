/*
 * fa.h -- C ABI of libfa.so: exact IO-aware attention forward on B200 (sm_100a).
 *
 * The operation (definition, "FlashAttention-3 vs naive attention", cnblogs,
 * section 1.1; "FlashAttention" concept page, Definition):
 *
 *     O = softmax(Q K^T * scale + mask) V
 *
 * computed tile by tile with an online softmax (running row max m and sum l,
 * "gsyq.cn FA vs FIA" section 1), so the L x L score matrix never reaches
 * device memory.  Two modes:
 *   - fa_prefill: packed variable-length sequences ("flash-attention" skill
 *     page, section 3.4), optional causal mask (section 3.2), grouped kv heads
 *     (GQA/MQA appendix).
 *   - fa_decode_paged: one query token per request against a paged KV cache
 *     addressed by a block table (PagedAttention appendix), split along the
 *     context and merged by log-sum-exp (FlashDecoding / Split-KV appendix).
 *
 * Conventions shared by every entry point:
 *   - Every tensor pointer is a DEVICE pointer owned by the caller; the library
 *     keeps no pointer after returning.  Tensors are dense, row-major in the
 *     layout stated beside each argument, 16-byte aligned.
 *   - bf16 means IEEE bfloat16 (2 bytes); fp32 means IEEE binary32.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream); no call synchronises the host except fa_get_device_error.
 *   - Argument checks happen on the host before any launch; a failed check
 *     returns FA_ERR_INVALID_ARG or FA_ERR_UNSUPPORTED and launches nothing.
 *   - Values that only the device can see (cu_seqlens, seq_lens, block_table
 *     entries) are range-checked in the kernels: an out-of-range value never
 *     causes an out-of-bounds access; it sets a sticky device error word
 *     (FA_ERR_DEVICE_BOUNDS) and the affected rows are skipped or read as
 *     zero.  Every wait inside a kernel is bounded in time; on timeout the
 *     kernel sets FA_ERR_DEVICE_TIMEOUT and returns.  Read the word with
 *     fa_get_device_error.
 *   - head_dim d must be 64 or 128 on the bf16 paths; Hq % Hkv == 0.
 *   - scale <= 0 selects the default 1/sqrt(d) (skill page, section 3.2,
 *     softmax_scale=None).
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *fa_stream_t; /* identical to cudaStream_t */

/* Largest batch whose decode plan (the prefix sums of the per-request range
 * counts) each CTA of the decode's split kernel builds itself. */
#define FA_DECODE_PLAN_MAX_B 2048

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,    /* null pointer, bad shape, misalignment       */
    FA_ERR_UNSUPPORTED = 2,    /* valid but not implemented (e.g. d = 96)     */
    FA_ERR_CUDA = 3,           /* a CUDA runtime call or launch failed        */
    FA_ERR_DEVICE_BOUNDS = 4,  /* a kernel saw an out-of-range index          */
    FA_ERR_DEVICE_TIMEOUT = 5  /* a kernel wait ran past its time limit       */
} fa_status;

/*
 * Prefill: exact attention over B packed sequences.
 *
 *   q           bf16 [T, Hq, d]   query rows; token t of sequence b is row
 *                                 cu_seqlens[b] + i, i in [0, L_b)
 *   k, v        bf16 [T, Hkv, d]  key / value rows, same packing
 *   o           bf16 [T, Hq, d]   output (written)
 *   lse         fp32 [Hq, T]      natural-log log-sum-exp of each row's scaled
 *                                 scores (written), or NULL
 *   cu_seqlens  int32 [B+1]       device; cu_seqlens[0] = 0, nondecreasing,
 *                                 cu_seqlens[B] = T
 *   causal      nonzero: query i sees keys j <= i of its own sequence;
 *               zero: it sees all L_b keys of its own sequence
 *   scale       multiplier of Q K^T (<= 0: 1/sqrt(d))
 *   total_tokens  T (host copy of cu_seqlens[B]; sizes q/k/v/o)
 *   max_seqlen    optional hint (the pages' max_seqlen_q/k): an upper bound
 *                 on every L_b, known on the host, that sizes the device work
 *                 list of 256-row blocks.  <= 0 = not given: the library uses
 *                 min(T, 1048576), which always holds when T <= 1048576.  At
 *                 most 1048576 (FA_ERR_UNSUPPORTED above).  A hint smaller
 *                 than the longest sequence is an error the device reports:
 *                 the rows past ceil(max_seqlen / 256) * 256 are not computed
 *                 (their O and LSE are left as they were) and
 *                 FA_ERR_DEVICE_BOUNDS is set.
 * Query head h reads kv head h / (Hq / Hkv); Hq <= 65535.  A sequence with
 * L_b = 0 is skipped.  The grid is one CTA per SM, widened when a CTA would
 * have to list more than 192 work items (sequence, 256-row block, head).
 * Does not allocate.
 */
fa_status fa_prefill(const void *q, const void *k, const void *v, void *o, float *lse,
                     const int32_t *cu_seqlens, int B, int Hq, int Hkv, int d, int causal,
                     float scale, fa_stream_t stream, int total_tokens, int max_seqlen);

/*
 * Prefill with the mask variants of the "flash-attention" skill page,
 * section 3.3 (advanced features).  The first fifteen arguments are those of
 * fa_prefill; fa_prefill is this call with (-1, -1, 0, NULL, 0).
 *
 *   window_left,  sliding window (window_size = (left, right)): query i of a
 *   window_right  sequence sees key j only when
 *                 i - window_left <= j <= i + window_right; a negative value
 *                 means no limit on that side.  causal != 0 keeps j <= i as
 *                 well (so window_right does not matter then); (-1, 0)
 *                 without causal is the causal mask.
 *   softcap       > 0: every logit x = scale * <q_i, k_j> becomes
 *                 softcap * tanh(x / softcap) (Gemma-2 style capping);
 *                 0 = off.  Negative, NaN or infinite: FA_ERR_INVALID_ARG.
 *   alibi_slopes  fp32, device, or NULL.  Adds -slope * |i - j| to the
 *                 (capped) logit of query i and key j, with
 *                 slope = alibi_slopes[b * alibi_batch_stride + h] for
 *                 sequence b and query head h: stride 0 for one slope per
 *                 head ([Hq]), Hq for [B, Hq].  The array must hold every
 *                 index that formula reaches.
 *   alibi_batch_stride  >= 0 (FA_ERR_INVALID_ARG otherwise).
 * LSE is the log-sum-exp of the final logits (after cap and ALiBi) over the
 * visible keys.  Every row sees at least its own key, so none is empty.  A
 * window shorter than the sequence also cuts the work: each 128-row query
 * tile visits only the 128-key tiles its rows' windows reach.
 */
fa_status fa_prefill_ex(const void *q, const void *k, const void *v, void *o, float *lse,
                        const int32_t *cu_seqlens, int B, int Hq, int Hkv, int d, int causal,
                        float scale, fa_stream_t stream, int total_tokens, int max_seqlen,
                        int window_left, int window_right, float softcap,
                        const float *alibi_slopes, int alibi_batch_stride);

/*
 * FP8 prefill (the pages list FP8 among the data types of FA3/FA4): q, k, v
 * are OCP e4m3 bytes (4 exponent bits, bias 7, 3 mantissa bits) in the
 * layouts of fa_prefill, each with one fp32 descale factor; the operation
 * is fa_prefill's on the values descale * e4m3.  d must be 128; o is bf16
 * [T, Hq, d] and lse fp32 [Hq, T] (or NULL) as in fa_prefill.  Both
 * products run on the tensor cores in e4m3 with fp32 accumulation; the
 * softmax probabilities are rounded to e4m3 for the second product (relative
 * error up to 2^-4 each) and O is divided by the sum of those rounded values.
 * Descale factors must be positive and finite (FA_ERR_INVALID_ARG).
 * Does not allocate.
 */
fa_status fa_prefill_fp8(const void *q, const void *k, const void *v, void *o, float *lse,
                         const int32_t *cu_seqlens, int B, int Hq, int Hkv, int d, int causal,
                         float scale, float q_descale, float k_descale, float v_descale,
                         fa_stream_t stream, int total_tokens, int max_seqlen);

/*
 * Paged decode: one query token per request at the end of its context.
 *
 *   q            bf16 [B, Hq, d]
 *   k_pages,
 *   v_pages      bf16 [num_pages, page_size, Hkv, d]   the page pool
 *   block_table  int32 [B, max_blocks_per_seq]  device; entry i of row b is
 *                the pool page holding tokens [i*page_size, (i+1)*page_size)
 *                of request b.  Entries at i >= ceil(seq_lens[b]/page_size)
 *                are never read.
 *   seq_lens     int32 [B]  device; context length of each request,
 *                0 <= seq_lens[b] <= max_blocks_per_seq * page_size
 *   page_size    tokens per page (>= 1)
 *   num_splits   number of contiguous, near-equal page ranges each
 *                request's context is cut into; 0 = automatic: ranges of one
 *                fixed page count for all requests (see
 *                fa_decode_auto_splits).  The result does not depend on the
 *                partition beyond rounding.
 *   o            bf16 [B, Hq, d]  output (written)
 *   lse          fp32 [B, Hq]  natural-log log-sum-exp, or NULL
 *   workspace    device scratch of at least
 *                fa_decode_workspace_size(B, Hq, d, resolved num_splits)
 *                bytes, 256-byte aligned; NULL = the library allocates it
 *                stream-ordered (cudaMallocAsync/cudaFreeAsync on `stream`)
 * A request with seq_lens[b] = 0 yields O = 0 and LSE = -inf; num_pages may
 * be 0 when every context is empty (the pool is then never read).  Any
 * group size Hq / Hkv and any page_size >= 1 are taken: a page size that is
 * a multiple of 16 is gathered with TMA boxes of 16 tokens, any other token
 * by token with 16-byte copies.  Each K/V byte is read from device memory
 * once per kv head for groups of up to 64 query heads (once per 64 query
 * heads above that).  Kernels launched: the split kernel, then, when a
 * request can have more than one range, the LSE combine (a programmatic
 * dependent launch of the split kernel), and before them, for
 * B > FA_DECODE_PLAN_MAX_B with more than one range, a one-CTA plan kernel.
 */
fa_status fa_decode_paged(const void *q, const void *k_pages, const void *v_pages,
                          const int32_t *block_table, const int32_t *seq_lens, int page_size,
                          int num_splits, void *o, fa_stream_t stream, int B, int Hq, int Hkv,
                          int d, int max_blocks_per_seq, int num_pages, float scale, float *lse,
                          void *workspace, size_t workspace_bytes);

/*
 * Paged decode that allocates nothing (no counterpart in the pages; this is
 * a deployment convenience).  Same arguments and result as fa_decode_paged
 * without the workspace pair: the split scratch comes from a 64 MiB array
 * compiled into the library, held by every GPU that loads it until exit.
 *
 * For callers that cannot allocate device memory when they run a decode
 * step, e.g. a serving engine that has already reserved nearly all of HBM
 * for its KV-cache pool, or a step loop that must not block in or fail
 * inside an allocator.
 *
 *   - Returns FA_ERR_UNSUPPORTED, launching nothing, when
 *     fa_decode_workspace_size(B, Hq, d, resolved num_splits) exceeds
 *     64 MiB; use fewer splits or fa_decode_paged with your own workspace.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make
 *     that first call before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents
 *     (nothing in it needs to start at zero).  Calls that overlap on the GPU
 *     (different streams without ordering between them) race on it.
 */
fa_status fa_decode_paged_noalloc(const void *q, const void *k_pages, const void *v_pages,
                                  const int32_t *block_table, const int32_t *seq_lens,
                                  int page_size, int num_splits, void *o, fa_stream_t stream,
                                  int B, int Hq, int Hkv, int d, int max_blocks_per_seq,
                                  int num_pages, float scale, float *lse);

/*
 * Decode step that first appends the new token to the cache ("flash-attention"
 * skill page, section 3.5: flash_attn_with_kvcache with k_new, v_new,
 * cache_seqlens, block_table and on-the-fly rotary embedding).
 *
 *   q             bf16 [B, Hq, d]    the new token's queries (not modified)
 *   k_new, v_new  bf16 [B, Hkv, d]   its key and value
 *   k_pages,      bf16 [num_pages, page_size, Hkv, d]   the page pool,
 *   v_pages       MODIFIED: the new key and value are written at position
 *                 pos = cache_seqlens[b] of request b, i.e. page
 *                 block_table[b][pos / page_size], slot pos % page_size
 *   cache_seqlens int32 [B], device: tokens already cached per request
 *                 (not modified; the caller advances it)
 *   rotary_cos,   fp32 [rotary_max_pos, rotary_dim / 2], device, or both NULL
 *   rotary_sin    (no rotation).  With tables, q and k_new are rotated at pos:
 *                 pair i is (x_i, x_{i + rotary_dim/2}), or (x_{2i}, x_{2i+1})
 *                 when rotary_interleaved != 0, turned by the angle with
 *                 cosine cos[pos][i] and sine sin[pos][i]; dimensions at or
 *                 past rotary_dim are unchanged.  The rotation is computed in
 *                 fp64 and rounded once to bf16 (nearest, ties to even).
 *                 rotary_dim must be even, 2 <= rotary_dim <= d.
 *   workspace     >= fa_decode_append_workspace_size(B, Hq, d, resolved
 *                 num_splits) bytes, 256-byte aligned, or NULL (allocated
 *                 stream-ordered)
 * Every query then attends to the pos + 1 tokens of its request, exactly as
 * fa_decode_paged with seq_lens = cache_seqlens + 1; the other arguments and
 * limits are those of fa_decode_paged.  Requests must append to distinct
 * page slots.  A position outside the block table or the rotary table, or an
 * unused page there, records FA_ERR_DEVICE_BOUNDS; that request writes
 * nothing to the cache and yields O = 0, LSE = -inf.
 */
fa_status fa_decode_paged_append(const void *q, const void *k_new, const void *v_new,
                                 void *k_pages, void *v_pages, const int32_t *block_table,
                                 const int32_t *cache_seqlens, int page_size, int num_splits,
                                 void *o, fa_stream_t stream, int B, int Hq, int Hkv, int d,
                                 int max_blocks_per_seq, int num_pages, float scale, float *lse,
                                 const float *rotary_cos, const float *rotary_sin,
                                 int rotary_max_pos, int rotary_dim, int rotary_interleaved,
                                 void *workspace, size_t workspace_bytes);

/* Workspace of fa_decode_paged_append: the rotated queries (bf16
 * [B, Hq, d]), the new context lengths (int32 [B]) and the split workspace
 * of fa_decode_workspace_size, each rounded up to 256 bytes. */
size_t fa_decode_append_workspace_size(int B, int Hq, int d, int num_splits);

/* Bytes of workspace fa_decode_paged needs for this shape and split count
 * (partial outputs fp32 [B, Hq, S, d], partial LSEs fp32 [B, Hq, S] and
 * the per-request range counts int32 [B+1]); 0 when S <= 1. */
size_t fa_decode_workspace_size(int B, int Hq, int d, int num_splits);

/* The split count num_splits = 0 resolves to.  In that automatic mode every
 * page range spans the same number of pages c, chosen for whole rounds of
 * ranges per SM (counting every request at max_blocks_per_seq pages) with
 * little partial-output traffic, and at least 256 tokens; this returns
 * ceil(max_blocks_per_seq / c): the largest number of ranges any request can
 * have, which sizes the workspace.  num_sms <= 0 queries the current device. */
int fa_decode_auto_splits(int B, int Hq, int Hkv, int max_blocks_per_seq, int page_size,
                          int num_sms);

/*
 * fp32 debug paths: the same operations with fp32 q/k/v/o (layouts as
 * above), plain CUDA-core arithmetic, any d in [1, 256].  For checking
 * conventions at fp32 precision, not for speed.
 */
fa_status fa_prefill_f32(const float *q, const float *k, const float *v, float *o, float *lse,
                         const int32_t *cu_seqlens, int B, int Hq, int Hkv, int d, int causal,
                         float scale, fa_stream_t stream, int total_tokens, int max_seqlen);

fa_status fa_decode_paged_f32(const float *q, const float *k_pages, const float *v_pages,
                              const int32_t *block_table, const int32_t *seq_lens,
                              int page_size, float *o, fa_stream_t stream, int B, int Hq,
                              int Hkv, int d, int max_blocks_per_seq, int num_pages,
                              float scale, float *lse);

/*
 * Self-test hook (used by the tests, not by the attention path): evaluates
 * on the GPU, element by element, a scalar function the prefill kernel
 * computes its softmax weights with, so it can be compared with an exact
 * reference over its whole input range.
 *
 *   op  FA_MATH_EXP2_FMA:     2^x on the FMA pipe (range reduction plus the
 *                             cubic of exp2_poly.cuh); x < -126 gives 0
 *       FA_MATH_EXP2_MUFU:    2^x by ex2.approx.ftz (the MUFU unit)
 *       FA_MATH_SOFTCAP_LOG2: a * b-scaled tanh: b * tanh(x * a / (2 log2 e)),
 *                             i.e. the softcapped logit in log2 units with
 *                             a = 2 log2(e) scale / cap and b = cap log2(e)
 *   x, y  fp32 [n], device; y = f(x) (written)
 * Returns FA_ERR_INVALID_ARG for an unknown op or n < 0.
 */
enum { FA_MATH_EXP2_FMA = 0, FA_MATH_EXP2_MUFU = 1, FA_MATH_SOFTCAP_LOG2 = 2 };
fa_status fa_selftest_math(int op, const float *x, float *y, int n, float a, float b,
                           fa_stream_t stream);

/*
 * Self-test hook (used by the tests of the timeout path, not by the
 * attention path): sets, for the current device, which kernel makes one
 * warp of its first CTA wait on a barrier that nothing arrives at, and the
 * time limit of the kernels' abortable waits.
 *
 *   which          0 = none (normal operation), FA_STALL_PREFILL = the first
 *                  softmax warpgroup of the prefill kernels (its first wait
 *                  for S), FA_STALL_DECODE = the first consumer warp of the
 *                  decode split kernel (its first wait for a stage)
 *   wait_limit_ns  limit of the abortable waits; 0 = the default, 2 s
 * When the limit runs out the kernel records FA_ERR_DEVICE_TIMEOUT, its
 * other roles stop, it waits (up to 2 s, whatever wait_limit_ns says) for
 * its own copies and tensor-core work in flight, frees its tensor memory and
 * returns; the outputs of that call are unspecified.  Synchronous (writes
 * two device variables).  Call with (0, 0) to restore normal operation.
 */
enum { FA_STALL_PREFILL = 1, FA_STALL_DECODE = 2 };
fa_status fa_selftest_inject_stall(int which, unsigned long long wait_limit_ns);

/* Reads and clears the sticky device error word of the current device
 * (synchronises `stream` first).  *code receives FA_OK or the first
 * FA_ERR_DEVICE_* recorded.  Returns FA_ERR_CUDA if the read fails. */
fa_status fa_get_device_error(fa_stream_t stream, int *code);

/* Static description of a status code. */
const char *fa_get_error_string(fa_status status);

/* Library version, as MAJOR*10000 + MINOR*100 + PATCH. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
