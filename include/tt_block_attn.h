/*
 * tt_block_attn.h -- C ABI of the TwoTower layer-aligned block attention on
 * NVIDIA B200 (sm_100a).
 *
 * The operation (paperfeed.app review of arXiv 2606.26493, "Nemotron-Labs-
 * TwoTower", section "The idea: freeze the reader, train the writer"): at
 * every attention layer i of the denoiser tower, the S noisy tokens of the
 * current block b form the queries Q_b^(i); the keys and values are the
 * frozen context tower's layer-i KV cache over every committed token,
 * followed by the denoiser's own KV for the block.  The cache is fully
 * visible (only the context tower itself is causal), attention inside the
 * block is bidirectional, still-masked positions included, and one
 * softmax runs over the concatenation.  The page's equation was lost in
 * extraction; the single joint softmax is the reading of its prose.
 *
 * For sequence n, query head j (KV head h = j / g, g = Hq / Hkv) and block
 * row t:
 *     keys  = { k_ctx[n,h,l] : 0 <= l < L_n }  ++  { k_blk[n,u,h] : 0 <= u < S }
 *     s_k   = scale * <q[n,t,j], k>
 *     out   = sum_k exp(s_k - m) v_k / sum_k exp(s_k - m),  m = max_k s_k
 *     lse   = m + ln sum_k exp(s_k - m)
 *
 * The block-causal entry point is the training / prefill form (same review,
 * section "Training and sampling": block b conditions on the frozen caches
 * c_{<b} and on itself): block b of a length-N sequence attends to context
 * positions [0, S*b) and to its own block positions [S*b, S*b+S).
 *
 * Besides the two attention entry points, the library carries the steps next to
 * them in a denoising loop: the block-causal backward (gradients for training),
 * the committed-block cache update and the confidence-unmasking step.
 *
 * Conventions shared by every entry point
 *   - Tensors are dense, row-major, device memory owned by the caller.
 *     q, k_*, v_* (and the backward's dout) are bf16; out, lse and gradients
 *     are fp32; ctx_lens is int32.  Every tensor pointer must be 16-byte
 *     aligned (the unmasking step's int / float arrays: 4-byte).
 *   - Calls are asynchronous and ordered on `stream`; none synchronises the
 *     host except tt_block_attn_check and tt_block_attn_profile_read.
 *   - A plan may be used by one stream at a time (it owns scratch memory).
 *   - Errors the host can see are returned synchronously.  Errors only the
 *     device can see (ctx_lens out of range, a pipeline wait that timed out)
 *     set the plan's device error word; the call's output is then
 *     unspecified and tt_block_attn_check reports the error.  No kernel traps.
 *   - Thread safety: distinct plans may be used from distinct threads.
 */
#ifndef TT_BLOCK_ATTN_H
#define TT_BLOCK_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TT_API __attribute__((visibility("default")))
#else
#define TT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                     /* same type as cudaStream_t */
typedef struct CUstream_st* tt_stream_t;

typedef enum {
  TT_OK = 0,
  TT_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad descriptor or size     */
  TT_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. head_dim 96)          */
  TT_ERR_CUDA = 3,          /* a CUDA runtime call or a kernel launch failed         */
  TT_ERR_DEVICE_ARG = 4,    /* seen on the device: a ctx_lens value out of range     */
  TT_ERR_TIMEOUT = 5        /* seen on the device: a pipeline wait ran out its limit */
} tt_status_t;

typedef enum {
  TT_KERNEL_AUTO = 0,       /* the tcgen05 kernel                                    */
  TT_KERNEL_TCGEN05 = 1,    /* warp-specialised TMA + tcgen05.mma + TMEM kernel      */
  TT_KERNEL_MMA_SYNC = 2    /* warp-level mma.sync baseline kernel                   */
} tt_kernel_t;

#define TT_PLAN_HOST_IO 1   /* flags: allocate device staging for tt_block_attn_host */
#define TT_PLAN_OUT_BF16 2  /* flags: `out` of the decode, paged, host and block-causal calls is
                               bf16 (round to nearest even) instead of fp32; lse stays fp32 */

typedef struct {
  int batch;          /* B >= 0 (B = 0 makes every call a no-op)                    */
  int num_q_heads;    /* Hq >= 1                                                     */
  int num_kv_heads;   /* Hkv >= 1, Hq % Hkv == 0; query head j reads KV head j/(Hq/Hkv) */
  int head_dim;       /* D: 64 or 128                                                */
  int block_size;     /* S >= 1 with S * (Hq / Hkv) <= 256                           */
  int ctx_capacity;   /* decode: Lcap >= 0, the token stride of k_ctx / v_ctx        */
  int seq_len;        /* block-causal: N >= 0, N % S == 0 (0: decode-only plan)      */
  float scale;        /* softmax scale; 0 selects 1/sqrt(head_dim)                   */
  int kernel;         /* tt_kernel_t                                                 */
  int num_ctas;       /* persistent grid size; 0 selects the device's SM count       */
  int flags;          /* TT_PLAN_HOST_IO | TT_PLAN_OUT_BF16, or 0                    */
  int wait_timeout_us;/* limit of every in-kernel wait; 0 selects 1000000 (1 s)      */
} tt_block_attn_desc;

typedef struct tt_plan_s* tt_plan_t;

typedef struct {
  int kernel;              /* tt_kernel_t actually used                               */
  int num_ctas;            /* work ranges (persistent CTAs)                           */
  int key_tile;            /* keys per pipeline tile                                  */
  int rows_per_unit;       /* S * g, the packed query rows of one (sequence, KV head) */
  size_t workspace_bytes;  /* device scratch owned by the plan                        */
  int sm_count;
  int variant;             /* tcgen05 kernel form: 0 default, 2 transposed PV, 3 2-SM pairs */
  int fused_combine;       /* non-zero: decode calls run the split combine in the attention
                              kernel's tail (one launch per call)                          */
} tt_plan_info;

/* Create a plan: validates the descriptor, picks the kernel and the work split
 * for `device`, and allocates every piece of device scratch the calls need
 * (split partials, per-range records, the error word, optional host-IO
 * staging).  The calls themselves never allocate.  Returns TT_ERR_INVALID_ARG
 * for a malformed descriptor, TT_ERR_UNSUPPORTED for head_dim other than
 * 64/128 or S*g > 256, TT_ERR_CUDA if allocation fails.  *out_plan is set only
 * on TT_OK; release it with tt_block_attn_plan_destroy. */
TT_API tt_status_t tt_block_attn_plan(const tt_block_attn_desc* desc, int device, tt_plan_t* out_plan);

TT_API void tt_block_attn_plan_destroy(tt_plan_t plan);

TT_API tt_status_t tt_block_attn_plan_get_info(tt_plan_t plan, tt_plan_info* info);

/* Decode-time block attention (one denoising step of one attention layer).
 *   q        [B, S, Hq, D]    bf16  queries of the block's S noisy tokens
 *   k_ctx    [B, Hkv, Lcap, D] bf16 context-tower layer-i keys (rows >= L_n unread)
 *   v_ctx    [B, Hkv, Lcap, D] bf16 context-tower layer-i values
 *   k_blk    [B, S, Hkv, D]   bf16  the denoiser's own block keys
 *   v_blk    [B, S, Hkv, D]   bf16  the denoiser's own block values
 *   ctx_lens [B]              int32 committed context length L_n, 0 <= L_n <= Lcap
 *   out      [B, S, Hq, D]    fp32  attention output (bf16 on a TT_PLAN_OUT_BF16 plan)
 *   lse      [B, Hq, S]       fp32  natural-log log-sum-exp per row; may be NULL
 * Context rows at or beyond L_n are never used, whatever they hold.  Out-of-range
 * ctx_lens values are clamped on the device and flagged TT_ERR_DEVICE_ARG.
 * Launches, all on `stream`: the attention kernel, then (when units were cut over
 * several work ranges) the split combine kernel, launched as its programmatic
 * dependent.  Plans whose units all get at least two ranges, each of at most 32 key
 * tiles at the plan's context capacity, launch the attention kernel cooperatively
 * and combine in its tail instead: one launch per call (tt_plan_info.fused_combine).
 * The attention kernel is itself a programmatic dependent of the kernel before it on
 * `stream`: its setup may overlap that kernel's tail, and it touches no global memory
 * before that kernel has completed, so stream order holds as for a plain launch. */
TT_API tt_status_t tt_block_attn(tt_plan_t plan, const void* q, const void* k_ctx, const void* v_ctx,
                          const void* k_blk, const void* v_blk, const int32_t* ctx_lens,
                          float* out, float* lse, tt_stream_t stream);

/* Decode over a PAGED context cache: the serving form, where the context tower's
 * layer-i cache of every sequence lives in fixed-size pages drawn from one shared pool.
 * The context tower alone holds sequence-length-dependent state, one prefix cache as in
 * AR serving (paperfeed review of arXiv 2606.26493, "What this changes, and what to be
 * skeptical of"), and committed blocks are ingested one after another ("Training and
 * sampling"); with contexts of widely different lengths a contiguous Lcap slab per
 * sequence would waste memory.  Same attention as tt_block_attn; only the addressing of
 * the context keys and values differs.
 *   k_pages    [num_pages, Hkv, page_size, D] bf16  key pool (device)
 *   v_pages    [num_pages, Hkv, page_size, D] bf16  value pool (device)
 *   page_table [B, pages_per_seq]             int32 pool page of each sequence's
 *              logical page: position l of sequence n is row l % page_size of page
 *              page_table[n][l / page_size] (device, read-only)
 *   q, k_blk, v_blk, ctx_lens, out, lse       as tt_block_attn, with
 *              0 <= ctx_lens[n] <= pages_per_seq * page_size
 * page_size is a power of two in [16, 65536]; the plan's ctx_capacity is not used.
 * Only the entries page_table[n][0 .. ceil(L_n / page_size)) are read; every one of
 * them must lie in [0, num_pages): a page outside the pool reads as zeros and is
 * flagged TT_ERR_DEVICE_ARG (as are out-of-range ctx_lens, which are clamped).
 * pages_per_seq == 0 means no context (k_pages / v_pages / page_table may be NULL).
 * Runs the default tcgen05 kernel (whatever TT_TCGEN05_VARIANT selects for
 * tt_block_attn) or the mma.sync kernel, as the plan chose, over the plan's work
 * ranges.  A plan made for the 2-SM form has one range per SM pair, so its paged
 * calls leave half the SMs idle: make paged plans without that form.  The caller
 * owns all buffers, nothing is allocated.  TT_ERR_INVALID_ARG for a bad page_size, negative
 * counts, a NULL pointer that is needed or a misaligned one (16 bytes for the bf16
 * and fp32 tensors, 4 for the int32 arrays); TT_ERR_UNSUPPORTED when a pool or a
 * logical capacity holds 2^31 rows or more. */
TT_API tt_status_t tt_block_attn_paged(tt_plan_t plan, const void* q, const void* k_pages,
                                const void* v_pages, const int32_t* page_table, int32_t num_pages,
                                int32_t page_size, int32_t pages_per_seq, const void* k_blk,
                                const void* v_blk, const int32_t* ctx_lens, float* out, float* lse,
                                tt_stream_t stream);

/* Block-causal training / prefill form over whole sequences of length N = seq_len.
 *   q      [B, N, Hq, D]  bf16      out [B, N, Hq, D] fp32 (bf16 on a TT_PLAN_OUT_BF16 plan)
 *   k_ctx  [B, Hkv, N, D] bf16 (context tower over the clean sequence), v_ctx likewise
 *   k_blk  [B, N, Hkv, D] bf16 (denoiser over the noisy sequence),     v_blk likewise
 *   lse    [B, Hq, N] fp32 natural log, may be NULL
 * Block b = positions [S*b, S*b+S) attends to k_ctx positions [0, S*b) and to its
 * own k_blk positions, bidirectionally.  Requires a plan with seq_len > 0.
 * Work split: the B*Hkv*(N/S) units (one per block and KV head) are laid end to end
 * in key tiles and cut into the plan's ranges.  On the default tcgen05 kernel the
 * boundaries weigh each unit as its key tiles plus a fixed cost of 8 tiles (its Q
 * load and pipeline restart, and its output epilogue), so that ranges of many short
 * early blocks take no longer than ranges of a few long late ones; the other kernels
 * split the tiles evenly.  tt_debug_causal_split shows the boundaries. */
TT_API tt_status_t tt_block_attn_block_causal(tt_plan_t plan, const void* q, const void* k_ctx,
                                       const void* v_ctx, const void* k_blk, const void* v_blk,
                                       float* out, float* lse, tt_stream_t stream);

/* Decode from HOST buffers (same layouts as tt_block_attn, same shapes as the plan):
 * copies the inputs into plan-owned device staging (the plan needs TT_PLAN_HOST_IO),
 * runs tt_block_attn, and copies out (and lse, when non-NULL) back, all ordered on
 * `stream`.  One cudaMemcpyAsync per buffer.  Host buffers should be page-locked
 * for the copies to be asynchronous and must stay valid until the stream has
 * been synchronised; the call itself does not synchronise. */
TT_API tt_status_t tt_block_attn_host(tt_plan_t plan, const void* q, const void* k_ctx, const void* v_ctx,
                               const void* k_blk, const void* v_blk, const int32_t* ctx_lens,
                               float* out, float* lse, tt_stream_t stream);

/* Decode without any device allocation, for callers that cannot call cudaMalloc
 * (engines and plugins that own all device memory and forbid further allocations,
 * or serving loops that must never stall on an allocation).  The paper has no
 * counterpart: this is a deployment variant of tt_block_attn.
 *   desc      shape as for tt_block_attn_plan; seq_len and flags must be 0.
 *             num_ctas = 0 picks the work split automatically; an explicit
 *             num_ctas whose scratch exceeds the limit below is rejected with
 *             TT_ERR_INVALID_ARG (tt_last_error_detail states the sizes).
 *   q .. lse  exactly as for tt_block_attn (device memory, same layouts).
 *   status    optional device uint32: zeroed, then receives the device error
 *             bits (1 = ctx_lens out of range, 2 = a wait timed out); NULL
 *             discards them.
 * Scratch: one file-scope device array of 40 MiB that every GPU loading this
 * library keeps until the process exits (one range per SM of a 148-SM GPU at
 * S*g = 256 rows and head_dim 128; an automatic split shrinks its range count
 * to fit).  The first call on a device (with
 * that device current) resolves the array's device address; make that first
 * call before any stream capture.  Every call shares the array and leaves its
 * contents behind, so calls that overlap on the GPU (different streams, or
 * different host threads on one device) race: order them.  The call allocates
 * nothing and does not synchronise. */
TT_API tt_status_t tt_block_attn_noalloc(const tt_block_attn_desc* desc, const void* q, const void* k_ctx,
                                         const void* v_ctx, const void* k_blk, const void* v_blk,
                                         const int32_t* ctx_lens, float* out, float* lse, uint32_t* status,
                                         tt_stream_t stream);

/* Block-causal backward pass (paperfeed.app review of arXiv 2606.26493, section
 * "Training and sampling": the loss of block b is conditioned on the noisy block and
 * the frozen caches c_{<b}; the context tower runs without gradients).  Gradients of
 * sum(dout * out) with respect to the denoiser's queries and its own block keys and
 * values; the context cache gets none.  For the rows r of block b and the keys k of
 * its key set (context positions < S*b, then its own S positions):
 *   p = exp(scale q.k - lse),  ds = p (dout.v - dout.out),
 *   dq = scale sum_k ds k,  dk_blk[k] = scale sum_r ds q_r,  dv_blk[k] = sum_r p dout_r
 * (block keys only; summed over the g query heads of each KV head).
 *   q, k_ctx, v_ctx, k_blk, v_blk   the forward's inputs, layouts of tt_block_attn_block_causal
 *   out  [B, N, Hq, D] fp32, lse [B, Hq, N] fp32   the forward's outputs (lse required);
 *                                  a TT_PLAN_OUT_BF16 plan is rejected (TT_ERR_UNSUPPORTED)
 *   dout [B, N, Hq, D] bf16        dL/dout (a bf16 operand of the tensor cores, like q, k, v)
 *   dq   [B, N, Hq, D] fp32        written
 *   dk_blk, dv_blk [B, N, Hkv, D] fp32   cleared, then written
 * The plan must be a block-causal plan (seq_len > 0).  Asynchronous on `stream`. */
TT_API tt_status_t tt_block_attn_block_causal_backward(tt_plan_t plan, const void* q, const void* k_ctx,
                                                       const void* v_ctx, const void* k_blk, const void* v_blk,
                                                       const float* out, const float* lse, const void* dout,
                                                       float* dq, float* dk_blk, float* dv_blk,
                                                       tt_stream_t stream);

/* Confidence-unmasking step of block sampling (paperfeed.app review of arXiv
 * 2606.26493, section "Training and sampling": every masked position is predicted in
 * parallel, each prediction with confidence above gamma = 0.8 is committed, the rest
 * stay masked for the next step).  For each position (n, s) masked on entry:
 *   argmax[n, s] = the first index of the largest logit,
 *   p_max[n, s]  = its softmax probability (fp32);
 * positions not masked on entry get p_max = 0, argmax = -1 and are not changed.
 * Then, per sequence, every masked position with p_max > gamma commits
 * (tokens[n, s] = argmax[n, s], masked[n, s] = 0); when none does and min_one is
 * non-zero, the masked position with the largest p_max (the first among equals)
 * commits instead.  n_committed[n] (may be NULL) receives the count.
 *   logits [B, S, V] bf16 (16-byte aligned); tokens [B, S] int32 and masked [B, S]
 *   uint8 updated in place; p_max [B, S] fp32 and argmax [B, S] int32 written.
 * Uses the current device; asynchronous on `stream`; 1 <= S <= 1024. */
TT_API tt_status_t tt_confidence_unmask(const void* logits, int batch, int block, int vocab, float gamma,
                                        int min_one, int32_t* tokens, uint8_t* masked, float* p_max,
                                        int32_t* argmax, int32_t* n_committed, tt_stream_t stream);

/* Committed-block cache update (paperfeed.app review of arXiv 2606.26493, section
 * "The idea: freeze the reader, train the writer": a committed block is ingested by
 * the frozen context tower, which extends its per-layer caches).  For every sequence n:
 *   k_ctx[n, h, L_n + t, :] = k_new[n, t, h, :],  v_ctx likewise,  t < S, h < Hkv,
 * with L_n = ctx_lens[n] read on the device, and then, when `advance` is non-zero,
 * ctx_lens[n] = L_n + S.
 *   k_new, v_new [B, S, Hkv, D] bf16  the context tower's layer-i K/V of the S committed
 *                                     positions (computed by the caller)
 *   k_ctx, v_ctx [B, Hkv, Lcap, D] bf16, updated in place; other rows are not touched
 *   ctx_lens     [B] int32 on the device, read (and advanced) in place
 * Uses the plan's B, S, Hkv, D and Lcap (ctx_capacity); asynchronous on `stream`.
 * A sequence with L_n < 0 or L_n + S > Lcap is left untouched (rows and length) and
 * raises TT_ERR_DEVICE_ARG at the next tt_block_attn_check.  Host-detectable errors
 * (null or misaligned pointers, Lcap < S) return TT_ERR_INVALID_ARG. */
TT_API tt_status_t tt_kv_append(tt_plan_t plan, const void* k_new, const void* v_new, void* k_ctx, void* v_ctx,
                                int32_t* ctx_lens, int advance, tt_stream_t stream);

/* Synchronise `stream`, then read and clear the plan's device error word.
 * Returns TT_OK, TT_ERR_DEVICE_ARG or TT_ERR_TIMEOUT (or TT_ERR_CUDA if the
 * synchronisation itself failed). */
TT_API tt_status_t tt_block_attn_check(tt_plan_t plan, tt_stream_t stream);

/* Per-kernel timing hook.  While enabled, every kernel the plan launches is
 * bracketed by two CUDA events recorded on the launching stream (up to 4096
 * launches are kept).  tt_block_attn_profile_read synchronises on the recorded
 * events and returns, for kernel id 0 (attention), 1 (split combine) or 2
 * (block-causal backward), the number of launches and their summed duration in
 * milliseconds.  In a stream being captured into a CUDA graph the events are
 * recorded as graph nodes, so the graph's replays are timed.  Calling
 * tt_block_attn_profile again clears the record. */
TT_API tt_status_t tt_block_attn_profile(tt_plan_t plan, int enable);
TT_API tt_status_t tt_block_attn_profile_read(tt_plan_t plan, int kernel_id, int* launches, double* total_ms);

/* Failure-path self test: launches one CTA that waits on a shared-memory
 * barrier nothing arrives at, using the same bounded wait as the attention
 * kernels, with a limit of `timeout_us`.  Expected result: TT_ERR_TIMEOUT, with
 * the device context still usable afterwards. */
TT_API tt_status_t tt_selftest_wait_timeout(int device, int timeout_us, tt_stream_t stream);

/* Numerics self test: evaluates on the device the library's FMA-pipe exp2 (range
 * reduction plus a fitted degree-3 polynomial, maximum relative error 7.5e-5 for
 * arguments in [-125, 127]) on the n host values x and writes the n results to y
 * (host).  The softmax of the default tcgen05 attention kernel computes one weight
 * pair in eight with this routine, the unmasking scan one pair in four, and the rest
 * with the hardware exp2 (ex2.approx).
 * Synchronous; allocates its own buffers. */
TT_API tt_status_t tt_selftest_exp2(int device, const float* x, float* y, int n);

/* Host-only view of the work split (no GPU needed): for `num_units` units with
 * tiles_per_unit[u] tiles each over `num_ctas` ranges, writes for every range c
 * its first global tile (range_start[c], num_ctas+1 entries) and, per unit, the
 * first and last range that touch it (unit_first[u], unit_last[u]).  The same
 * code decides the split inside the kernels. */
TT_API tt_status_t tt_debug_work_split(int num_units, const int* tiles_per_unit, int num_ctas,
                                long long* range_start, int* unit_first, int* unit_last);

/* Host-only view of the block-causal work split of the default tcgen05 kernel (no
 * GPU needed): for B = batch sequences of seq_len positions in blocks of
 * block_size, Hkv = num_kv_heads and key_tile keys per tile, writes the first
 * global tile of each of the num_ctas ranges and the total T (range_start, host,
 * num_ctas + 1 entries; ranges beyond min(num_ctas, T) start at T).  unit_cost is
 * the fixed cost of a unit in key tiles: -1 takes the plan's default (8), 0 gives
 * the even split of tt_debug_work_split.  The plan builds its table with the same
 * code.  TT_ERR_INVALID_ARG for non-positive sizes, seq_len not a multiple of
 * block_size or a NULL range_start; TT_ERR_UNSUPPORTED when one (n, h) has 2^31
 * tiles or more. */
TT_API tt_status_t tt_debug_causal_split(int batch, int num_kv_heads, int seq_len, int block_size,
                                         int key_tile, int num_ctas, int unit_cost, long long* range_start);

TT_API const char* tt_status_string(tt_status_t status);

/* Detail of the last host-side error on the calling thread ("" if none). */
TT_API const char* tt_last_error_detail(void);

#ifdef __cplusplus
}
#endif

#endif /* TT_BLOCK_ATTN_H */
