/*
 * pgd.h -- C ABI of libpgd.so: paged GQA decode attention on B200 (sm_100a).
 *
 * Decode-phase attention over a paged KV cache: each running sequence has one
 * query token, which attends over that sequence's whole cached K/V history.
 * The history is read block by block through a block table; the query heads
 * of a GQA group share one KV head; every sequence in the batch has its own
 * context length; the work is split along the KV length and the splits are
 * merged by log-sum-exp.
 *
 * Sources (page title and section):
 *   "attention kernels" (froggydisk, LLM serving / decoding):
 *     section "standard attention"      -- S = Q K^T, P = softmax(S), O = P V
 *     section "FlashAttention"          -- online softmax over K blocks is exact
 *     section "prefill and decode attention" -- decode reads each KV head once
 *        for all query heads of its group; the work is split along the KV
 *        length and the splits are merged like the online softmax
 *     section "paged KV and kernels"    -- block table; variable-length batch
 *        in one launch; FP8 KV read directly
 *   "Optimization 1: batching and attention" (beengineer500):
 *     section 2.4 -- num_attention_heads / num_key_value_heads; 32/8 = 4 heads
 *        share one KV head
 *     section 3.4 -- PagedAttention: fixed-size blocks, block table from
 *        logical to physical block, blocks need not be contiguous
 *
 * Conventions for every entry point:
 *   - Device pointers are caller-owned device memory; nothing is freed or
 *     kept past the call except the library's own workspace (see below).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call only enqueues work on `stream`; none synchronises
 *     with the host, so results are ready once the stream has reached them.
 *   - Host-side argument checks run before any launch and return a status;
 *     on error nothing is enqueued.
 *   - Faults the device detects (a block id outside [0, num_blocks), a
 *     context length outside [0, max_blocks_per_seq * block_size], a slot
 *     outside the pool, a pipeline wait that ran out of time) never trap:
 *     the kernel records a flag, keeps every access in bounds and returns;
 *     pgd_get_device_error() reports and clears the flags.  Outputs of a call
 *     that raised a flag are undefined.
 *
 * KV cache layout ("HND"): k_cache and v_cache are
 *     [num_blocks][num_kv_heads][block_size][head_dim]
 * elements of the cache type (bf16, or FP8 E4M3 bytes), so one (block, KV
 * head) tile of block_size x head_dim is contiguous.  Token t of sequence s
 * lives in physical block block_table[s][t / block_size] at row
 * t % block_size.  Query head i reads KV head i / g, g = num_q_heads /
 * num_kv_heads.
 */
#ifndef PGD_H_
#define PGD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PGD_OK = 0,
    PGD_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer   */
    PGD_ERR_UNSUPPORTED = 2,   /* shape outside the compiled variants          */
    PGD_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed            */
    PGD_ERR_DEVICE_BOUNDS = 4, /* device flagged an out-of-range index         */
    PGD_ERR_TIMEOUT = 5,       /* device flagged a pipeline wait that timed out */
    PGD_ERR_WORKSPACE = 6      /* caller workspace too small                   */
} pgd_status;

typedef enum {
    PGD_KV_BF16 = 0,           /* bf16 K/V, 2 bytes per element                 */
    PGD_KV_FP8_E4M3 = 1        /* FP8 E4M3 K/V bytes times a per-KV-head scale  */
} pgd_kv_dtype;

/* Human-readable name of a status code (static string). */
const char *pgd_status_string(pgd_status status);

/* Library version, "major.minor.patch" (static string). */
const char *pgd_version(void);

/* ------------------------------------------------------------------------ */
/* KV append                                                                */
/* ------------------------------------------------------------------------ */
/*
 * pgd_kv_append -- write the K and V rows of new tokens into their cache
 * slots ("batching and attention" 3.4: a token's KV lives in a slot of a
 * fixed-size physical block).
 *
 *   k_new, v_new   device, [num_tokens][num_kv_heads][head_dim] elements of
 *                  the cache type (bf16, or E4M3 bytes), 16-byte aligned.
 *   slot_mapping   device int64 [num_tokens]; token t goes to physical block
 *                  slot / block_size, row slot % block_size.  A slot < 0 is a
 *                  padding token and is skipped; a slot >= num_blocks *
 *                  block_size is skipped and flags PGD_ERR_DEVICE_BOUNDS.
 *   k_cache, v_cache  device, HND layout above, 16-byte aligned; rows that no
 *                  token maps to are left untouched.
 *   num_tokens >= 0 (0 enqueues nothing); head_dim in {128, 256};
 *   block_size in {16, 32, 64}; num_kv_heads in 1 .. 65536 (more is
 *   PGD_ERR_UNSUPPORTED).
 * The copy is bit-exact.  Two tokens mapped to the same slot race (the
 * result is one of them).
 */
pgd_status pgd_kv_append(const void *k_new, const void *v_new,
                         const int64_t *slot_mapping, int32_t num_tokens,
                         void *k_cache, void *v_cache,
                         int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                         int32_t num_blocks, pgd_kv_dtype kv_dtype, void *stream);

/*
 * pgd_kv_append_quant -- the append of pgd_kv_append into an FP8 E4M3 cache
 * from bf16 rows ("attention kernels", sections "paged KV and kernels" and
 * "what to check": FP8 KV caches, read directly by the kernel).  Element x of
 * KV head h is stored as the E4M3 value nearest to x / scale[h] (the division
 * in fp32, IEEE round to nearest; the conversion rounds to nearest with ties
 * to even and saturates magnitudes above 448 to +-448; NaN stays NaN), so
 * that e4m3 * scale[h] approximates x.
 *
 *   k_new, v_new      device bf16 [num_tokens][num_kv_heads][head_dim],
 *                     16-byte aligned
 *   slot_mapping      device int64 [num_tokens], as pgd_kv_append
 *   k_cache, v_cache  device E4M3 bytes, HND layout, 8-byte aligned
 *   k_scale, v_scale  device fp32 [num_kv_heads] (the scales the decode uses)
 *   head_dim in {128, 256}; block_size in {16, 32, 64}; num_kv_heads in
 *   1 .. 65536.
 * Bit-exact with that definition.
 */
pgd_status pgd_kv_append_quant(const void *k_new, const void *v_new,
                               const int64_t *slot_mapping, int32_t num_tokens,
                               void *k_cache, void *v_cache,
                               const float *k_scale, const float *v_scale,
                               int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                               int32_t num_blocks, void *stream);

/* ------------------------------------------------------------------------ */
/* Paged decode attention                                                   */
/* ------------------------------------------------------------------------ */
/*
 * pgd_decode_workspace_bytes -- bytes of device workspace that
 * pgd_paged_decode_attention needs on the current device with an automatic
 * grid (the split partial outputs and their log-sum-exps; no zeroing
 * needed).  num_seqs is accepted for interface stability; the size depends
 * on the group size, head_dim and the device's SM count.  Returns 0 for
 * invalid sizes.
 */
size_t pgd_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads,
                                  int32_t num_kv_heads, int32_t head_dim);

/*
 * pgd_paged_decode_attention -- one decode step of attention for a batch.
 *
 * For sequence s and query head i (KV head h = i / g), with n = context_lens[s]:
 *   x_t   = scale * sum_d q[s][i][d] * K_t[d]            t = 0..n-1
 *   out   = sum_t exp(x_t - M) V_t / sum_t exp(x_t - M),  M = max_t x_t
 *   lse   = M + ln sum_t exp(x_t - M)
 * where K_t, V_t are row t % block_size of physical block
 * block_table[s][t / block_size], KV head h ("attention kernels", sections
 * "standard attention" and "paged KV and kernels").  For FP8 E4M3 caches
 * K_t = e4m3(byte) * k_scale[h] and V_t = e4m3(byte) * v_scale[h].
 * n = 0 gives out = 0 and lse = -inf.
 *
 * The work of the whole batch is divided evenly over a grid sized to the
 * device: each CTA streams an equal share of the (sequence, KV head, block)
 * tiles through a TMA shared-memory pipeline, reads each K/V tile once for
 * all g query heads of its group, and keeps an online softmax; a sequence
 * whose tiles fall into several CTAs is merged by log-sum-exp by the CTA that
 * finishes its last share ("prefill and decode attention").  The result does
 * not depend on where the blocks sit in the pool, and repeated calls with the
 * same inputs and grid give the same bits (the splits are merged in a fixed
 * order).
 *
 *   q             device bf16 [num_seqs][num_q_heads][head_dim], 16-byte aligned
 *   k_cache, v_cache  device, HND layout, 16-byte aligned, num_blocks blocks
 *   block_table   device int32 [num_seqs][max_blocks_per_seq]; entries past
 *                 ceil(context_lens[s] / block_size) are never read
 *   context_lens  device int32 [num_seqs], each in [0, max_blocks_per_seq *
 *                 block_size]
 *   max_context_len  host hint >= every context length (0 = unknown); only
 *                 used to size the grid for small batches
 *   num_q_heads % num_kv_heads == 0, g = num_q_heads / num_kv_heads in
 *                 1 .. 16; head_dim in {128, 256} (256 with bf16 only);
 *                 block_size in {16, 32, 64}
 *   scale         softmax scale applied to q.k (e.g. 1/sqrt(head_dim))
 *   kv_dtype      PGD_KV_BF16 or PGD_KV_FP8_E4M3
 *   k_scale, v_scale  device fp32 [num_kv_heads] for FP8 (NULL for bf16)
 *   out           device bf16 [num_seqs][num_q_heads][head_dim] (RNE from fp32),
 *                 16-byte aligned
 *   lse_out       optional device fp32 [num_seqs][num_q_heads] (natural log),
 *                 NULL to skip
 *   workspace, workspace_bytes  device scratch for the split partials, at
 *                 least pgd_decode_workspace_bytes(...) bytes (any contents);
 *                 NULL/0 selects a library-owned buffer (grown on demand with
 *                 cudaMalloc, kept until pgd_shutdown()).  The library also
 *                 keeps one int32 arrival counter per (sequence, KV head) in
 *                 its own zeroed device buffer (grown the same way).  Calls
 *                 that share a workspace, or run on one device at the same
 *                 time, must not overlap on the GPU.
 *   num_ctas      0 = automatic grid (pgd_decode_grid tells which); > 0
 *                 forces that many CTAs (used to test split-count
 *                 invariance)
 *   stream        cudaStream_t as void*
 */
pgd_status pgd_paged_decode_attention(
    const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_table, int32_t max_blocks_per_seq,
    const int32_t *context_lens, int32_t num_seqs, int32_t max_context_len,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t num_blocks, float scale, pgd_kv_dtype kv_dtype,
    const float *k_scale, const float *v_scale,
    void *out, float *lse_out,
    void *workspace, size_t workspace_bytes, int32_t num_ctas, void *stream);

/*
 * pgd_decode_step -- one whole decode step in one launch: the KV append of
 * each sequence's newest token ("batching and attention" 3.4: the new K/V
 * row goes to its slot in the sequence's last block) fused with the decode
 * attention of pgd_paged_decode_attention.  The result equals
 * pgd_kv_append(k_new, v_new, slots) followed by pgd_paged_decode_attention,
 * with slots[s] = block_table[s][(n-1)/block_size] * block_size +
 * (n-1) % block_size, n = context_lens[s] (the count already includes the new
 * token; sequences with n = 0 append nothing).
 *
 *   k_new, v_new  device [num_seqs][num_kv_heads][head_dim] in the cache type
 *                 (bf16 or E4M3 bytes), 16-byte aligned
 *   k_cache, v_cache  written at those slots, read everywhere else
 *   all other arguments as pgd_paged_decode_attention.
 * The CTA that reads a sequence's last tile for one KV head also writes that
 * head's new row into it, before reading it, so no other launch is needed.
 */
pgd_status pgd_decode_step(
    const void *q, const void *k_new, const void *v_new, void *k_cache, void *v_cache,
    const int32_t *block_table, int32_t max_blocks_per_seq,
    const int32_t *context_lens, int32_t num_seqs, int32_t max_context_len,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t num_blocks, float scale, pgd_kv_dtype kv_dtype,
    const float *k_scale, const float *v_scale,
    void *out, float *lse_out,
    void *workspace, size_t workspace_bytes, int32_t num_ctas, void *stream);

/*
 * pgd_paged_decode_attention_ex -- pgd_paged_decode_attention generalised to
 * q_len query tokens per sequence and an optional sliding window.
 *
 * The q_len newest tokens of sequence s occupy positions n - q_len .. n - 1
 * (n = context_lens[s] counts them, their K/V already in the cache).  Query
 * token j (0 <= j < q_len) sees positions t < hi = n - q_len + 1 + j (causal
 * among the new tokens, as in the verification step of speculative decoding
 * in the inference lecture's section on it), and with window > 0 only
 * t >= hi - window (sliding-window attention, the co-design page's section on
 * reducing the attended range).  A row that sees no position gets out = 0 and
 * lse = -inf; the formulas are otherwise those of
 * pgd_paged_decode_attention over the visible positions.
 *
 *   q        device bf16 [num_seqs][q_len][num_q_heads][head_dim]
 *   out      device bf16 [num_seqs][q_len][num_q_heads][head_dim]
 *   lse_out  optional fp32 [num_seqs][q_len][num_q_heads]
 *   q_len    >= 1 with g * q_len <= 32 (g = num_q_heads / num_kv_heads): every
 *            query row of a KV head rides on one pass over its K/V tiles
 *            (up to 16 rows all four consumer warps hold every row; 17 to 32
 *            rows are split into two groups of 16, each over all tokens)
 *   window   0 = the whole causal range; > 0 = the last `window` positions
 *   workspace  at least pgd_decode_workspace_bytes(num_seqs,
 *            num_q_heads * q_len, num_kv_heads, head_dim) bytes, or NULL/0
 *   all other arguments and errors as pgd_paged_decode_attention; q_len = 1,
 *   window = 0 gives exactly that call.  g * q_len > 32 returns
 *   PGD_ERR_UNSUPPORTED.  Blocks that lie wholly before a window are not read.
 */
pgd_status pgd_paged_decode_attention_ex(
    const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_table, int32_t max_blocks_per_seq,
    const int32_t *context_lens, int32_t num_seqs, int32_t max_context_len,
    int32_t q_len, int32_t window,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t num_blocks, float scale, pgd_kv_dtype kv_dtype,
    const float *k_scale, const float *v_scale,
    void *out, float *lse_out,
    void *workspace, size_t workspace_bytes, int32_t num_ctas, void *stream);

/* ------------------------------------------------------------------------ */
/* Consumer math of the decode kernels                                      */
/* ------------------------------------------------------------------------ */
/*
 * The decode kernels form q.k and p.V on the tensor cores by default: a small
 * mma.sync per 16 tokens with the group's query rows on the narrow side.
 * PGD_MATH_CUDA_CORE selects a variant that does the same arithmetic with
 * FP32 FMAs and warp-shuffle reductions (the form the decode kernels of the
 * "attention kernels" page describe), kept so that the two can be measured
 * against each other on this bandwidth-bound path.  It covers bf16 caches
 * with head_dim 128 and at most 8 query rows per KV head (g * q_len <= 8);
 * while it is selected, other shapes return PGD_ERR_UNSUPPORTED.  Results of
 * the two agree within the stated tolerances, not bit for bit.
 *
 * pgd_set_decode_math -- process-wide setting for every decode entry point
 * that follows (host only; PGD_ERR_INVALID_ARG for an unknown value).
 * pgd_get_decode_math -- the current setting.
 */
typedef enum {
    PGD_MATH_TENSOR_CORE = 0,
    PGD_MATH_CUDA_CORE = 1
} pgd_decode_math;

pgd_status pgd_set_decode_math(pgd_decode_math math);
pgd_decode_math pgd_get_decode_math(void);

/* ------------------------------------------------------------------------ */
/* Test hook for the timeout path                                           */
/* ------------------------------------------------------------------------ */
/*
 * Every wait inside the decode kernels (a K/V stage landing, a segment
 * descriptor, a free ring slot, an appended row) is bounded: after the limit
 * the kernel raises the timeout flag (8), its warps leave together, the
 * producer still waits for every copy it issued (with its own fixed limit of
 * 1 s) so nothing lands after the CTA exits, and pgd_get_device_error()
 * returns PGD_ERR_TIMEOUT and re-zeroes the arrival counters, so the next
 * call starts clean.  No correct input makes a wait run out, so this hook
 * exists to test that path: a limit of a few ns makes the waits give up.
 *
 * pgd_debug_set_wait_limit_ns -- process-wide limit of those waits for the
 * decode launches that follow, in ns; 0 restores the default (1 s).  Outputs
 * of a launch that timed out are undefined.  Not for production use.
 * pgd_debug_get_wait_limit_ns -- the current limit.
 */
pgd_status pgd_debug_set_wait_limit_ns(uint64_t limit_ns);
uint64_t pgd_debug_get_wait_limit_ns(void);

/*
 * pgd_decode_grid -- host function (no CUDA call): the CTA count of the
 * automatic grid (num_ctas = 0) of the decode entry points on a device with
 * `sms` multiprocessors that hold `ctas_per_sm` decode CTAs each (on a B200:
 * 148 SMs, 2 CTAs at head_dim 128, 1 at 256).  The batch's work counts each
 * (sequence, KV head) unit as its blocks plus a fixed cost (48 KB of K/V
 * streaming time for bf16 caches, 36 KB for FP8), every unit taken at
 * max_context_len (or max_blocks_per_seq * block_size when it is 0):
 *   - grid = one wave (sms * ctas_per_sm), or fewer so that every CTA gets
 *     at least four 64-token stages of that work (the cap);
 *   - with fewer units than that, units of equal length should split into
 *     whole pieces, one per CTA: a batch below the wave takes the multiple of
 *     the unit count nearest the cap, and a full wave is rounded down to a
 *     multiple of the unit count when that drops at most 1/8 of it.
 * Other arguments as pgd_paged_decode_attention; fp8 = 1 for an FP8 E4M3
 * cache.  Returns the CTA count, or 0 for invalid arguments.
 */
int64_t pgd_decode_grid(int32_t sms, int32_t ctas_per_sm, int32_t num_seqs,
                        int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                        int32_t max_blocks_per_seq, int32_t max_context_len, int32_t fp8);

/* ------------------------------------------------------------------------ */
/* KV parallelism: one sequence's KV split along its length over GPUs       */
/* ------------------------------------------------------------------------ */
/*
 * Models with few KV heads run out of tensor parallelism at the KV head
 * count; attention then shards each sequence's KV along its length over the
 * GPUs (KVP, the co-design page's "Principle 4").  Each GPU decodes its
 * slice into an unrounded split result (o, lse), the GPUs exchange those
 * (an all-gather of num_seqs * num_q_heads * (head_dim + 1) fp32 per GPU),
 * and pgd_merge_partials combines them exactly as the splits inside one GPU
 * are combined ("attention kernels", "prefill and decode attention").
 *
 * pgd_kvp_plan -- host function (no CUDA call): the slice of every sequence
 * that `rank` holds.  A sequence with nb = ceil(n / block_size) blocks is cut
 * at block boundaries into world_size contiguous runs; rank r holds logical
 * blocks [floor(nb * r / W), floor(nb * (r + 1) / W)), i.e. tokens from
 * block_start[s] * block_size, slice_len[s] of them (0 when the run is
 * empty).  The rank's block table lists those blocks in order, so its slice
 * decodes as a sequence of slice_len[s] tokens.
 *   context_lens  host int32 [num_seqs], each >= 0
 *   block_start, slice_len  host int32 [num_seqs], written
 *   world_size >= 1, 0 <= rank < world_size
 */
pgd_status pgd_kvp_plan(const int32_t *context_lens, int32_t num_seqs, int32_t block_size,
                        int32_t world_size, int32_t rank, int32_t *block_start,
                        int32_t *slice_len);

/*
 * pgd_paged_decode_partial -- pgd_paged_decode_attention for one KV slice,
 * with the result left unrounded for a later merge: o_part gets the fp32
 * softmax-weighted sum over the slice's tokens and lse_part its natural-log
 * log-sum-exp (required).  A sequence with an empty slice gets o = 0 and
 * lse = -inf, which carries no weight in the merge.
 *
 *   o_part    device fp32 [num_seqs][num_q_heads][head_dim], 16-byte aligned
 *   lse_part  device fp32 [num_seqs][num_q_heads]
 *   all other arguments, limits and errors as pgd_paged_decode_attention
 *   (context_lens and block_table describe the slice).
 * The outputs of W slices, stacked as [W][num_seqs * num_q_heads][head_dim]
 * and [W][num_seqs * num_q_heads], are pgd_merge_partials' inputs.
 */
pgd_status pgd_paged_decode_partial(
    const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_table, int32_t max_blocks_per_seq,
    const int32_t *context_lens, int32_t num_seqs, int32_t max_context_len,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t num_blocks, float scale, pgd_kv_dtype kv_dtype,
    const float *k_scale, const float *v_scale,
    float *o_part, float *lse_part,
    void *workspace, size_t workspace_bytes, int32_t num_ctas, void *stream);

/*
 * pgd_paged_decode_attention_noalloc -- the same decode step as
 * pgd_paged_decode_attention, for callers that must not have the library
 * allocate device memory: a serving engine that has reserved nearly all HBM
 * for its KV-cache pool (a cudaMalloc at decode time can fail), a host that
 * routes and accounts every device byte through its own allocator, or a
 * decode loop that cannot absorb the device-wide synchronisation of a
 * cudaFree when a library buffer grows.  There is no counterpart on the
 * pages; this is an interface choice of the library.
 *
 * Arguments are those of pgd_paged_decode_attention without the workspace:
 * the caller still provides every input and output.  The split partials and
 * the arrival counters live in one static device array of 8 MiB per device,
 * held until the process exits.  With CUDA's default lazy module loading the
 * array is committed on a device at the first call of this library there
 * (any entry point), not when the library is loaded: make one call on each
 * device before reserving the KV-cache pool, so that the 8 MiB are already
 * taken.  The call allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library routine.
 *   - Limits: num_seqs * num_kv_heads <= 65536, and the split partials of the
 *     grid must fit in the rest of the array; an automatic grid is reduced to
 *     fit, an explicit num_ctas that does not fit is rejected.  Requests past
 *     a limit return PGD_ERR_WORKSPACE and enqueue nothing.
 *   - Set-up: the first call on each device (with that device current)
 *     resolves the array's device address with cudaGetSymbolAddress; make
 *     that first call before any stream capture.
 *   - Every call clears the counters it uses (a cudaMemsetAsync on `stream`)
 *     and then reuses the array, which keeps the previous call's contents.
 *     Calls on one device that overlap on the GPU (other streams, other host
 *     threads) share the array and race: serialise them.
 */
pgd_status pgd_paged_decode_attention_noalloc(
    const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_table, int32_t max_blocks_per_seq,
    const int32_t *context_lens, int32_t num_seqs, int32_t max_context_len,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t num_blocks, float scale, pgd_kv_dtype kv_dtype,
    const float *k_scale, const float *v_scale,
    void *out, float *lse_out, int32_t num_ctas, void *stream);

/*
 * pgd_merge_partials -- log-sum-exp merge of split results ("attention
 * kernels", section "prefill and decode attention": splits along the KV
 * length are merged the same way the online softmax merges blocks).  For
 * each row r:  M = max_p lse_part[p][r];  w_p = exp(lse_part[p][r] - M);
 * out[r] = sum_p w_p o_part[p][r] / sum_p w_p;  lse[r] = M + ln sum_p w_p.
 * Splits with lse = -inf carry no weight; a row whose splits are all -inf
 * gives out = 0, lse = -inf.  Used to merge per-GPU splits of one sequence.
 *
 *   o_part    device fp32 [num_parts][rows][head_dim], 16-byte aligned
 *   lse_part  device fp32 [num_parts][rows] (natural log)
 *   out       device bf16 [rows][head_dim], 8-byte aligned
 *   lse_out   optional device fp32 [rows], NULL to skip
 *   num_parts >= 1, rows >= 0, head_dim in {128, 256}
 */
pgd_status pgd_merge_partials(const float *o_part, const float *lse_part,
                              int32_t num_parts, int32_t rows, int32_t head_dim,
                              void *out, float *lse_out, void *stream);

/*
 * pgd_get_device_error -- wait for `stream`, then read and clear the device
 * flags raised by earlier calls on this device.  Returns PGD_OK when none
 * was raised, PGD_ERR_DEVICE_BOUNDS or PGD_ERR_TIMEOUT otherwise (and
 * *flags, if non-NULL, receives the raw bit set: 1 block id, 2 context
 * length, 4 slot, 8 wait timeout).
 */
pgd_status pgd_get_device_error(void *stream, uint32_t *flags);

/* Free library-owned workspaces (call with no work in flight). */
pgd_status pgd_shutdown(void);

/* ------------------------------------------------------------------------ */
/* Short forms with the argument lists of the problem statement.            */
/* ------------------------------------------------------------------------ */
/* kv_append for bf16 caches: pgd_kv_append with PGD_KV_BF16. */
pgd_status kv_append(const void *k_new, const void *v_new, const int64_t *slot_mapping,
                     int32_t num_tokens, void *k_cache, void *v_cache,
                     int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                     int32_t num_blocks, void *stream);

/* paged_decode_attention for bf16 caches, no lse output, library workspace,
 * automatic grid: pgd_paged_decode_attention with those choices. */
pgd_status paged_decode_attention(const void *q, const void *k_cache, const void *v_cache,
                                  const int32_t *block_table, int32_t max_blocks_per_seq,
                                  const int32_t *context_lens, int32_t num_seqs,
                                  int32_t num_q_heads, int32_t num_kv_heads,
                                  int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                  float scale, void *out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PGD_H_ */
