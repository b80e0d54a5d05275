/*
 * da.h -- C ABI of libda.so: split-KV decode attention over a paged,
 * variable-length KV cache, load-balanced by an on-device tile planner
 * ("Dynamic Attention"), for NVIDIA B200 (sm_100a).
 *
 * Source of the operation: "Tencent HPC lands in SGLang, challenging default
 * inference kernels", section "Why Tencent HPC matters for online model
 * serving": in a continuous batch one request may hold a 16,000-token context
 * while another has just started with 1,000, so a static attention schedule
 * leaves one block with far more work than another; the KV-cache work is cut
 * into smaller uniform tiles and a scheduler hands the tiles to CTAs according
 * to the current workload, rebuilding that mapping as request lengths change
 * during decoding.  The same section names the baseline: a static split-k
 * policy, which either idles units or launches empty chunks for short
 * requests.  The article gives no API; the calls below are this library's.
 *
 * One decode step is three asynchronous calls on one stream:
 *   da_plan              (or da_static_plan)  seq_lens -> work list in `ws`
 *   da_decode_attention  work list -> out/lse (single-segment requests) and
 *                        per-segment partials (requests split over CTAs)
 *   da_combine           partials -> out/lse by log-sum-exp merge
 * or one call, da_decode_step, which enqueues the same three launches.
 * (With merge_in_decode = 1 in the descriptor the decode kernel merges split
 * requests itself and da_combine enqueues nothing.)  Before the step, the new
 * token's K/V rows go into their pages with da_append_kv, or with
 * da_plan_append, which also builds the dynamic plan in the same launch and
 * then stands in for da_plan.  da_decode_step_host runs a whole step from host
 * buffers in one call.
 * The host never reads seq_lens: every launch's grid is fixed by the problem
 * and the plan descriptor, so requests can join, grow, finish or be cancelled
 * between steps without a host round trip, and the three calls can be
 * captured in a CUDA graph.
 *
 * Conventions for every call:
 *   - Return 0 (DA_OK) or a negative DA_ERR_* code.  Host-side argument
 *     checks happen before anything is enqueued; a call that returns an error
 *     has enqueued nothing.  DA_ERR_CUDA means a CUDA runtime call failed; its
 *     cudaError_t value is available from da_last_cuda_error() (per thread).
 *   - "dev" pointers are device memory (or managed memory) on the current
 *     device; "host" pointers are ordinary host memory.  The caller allocates
 *     and owns every buffer; the library allocates, frees and synchronises
 *     nothing, except da_read_status, which synchronises its stream.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is asynchronous; buffers must stay alive until it ends.
 *   - Data errors found on the device (a length out of range, a page id out
 *     of range, a wait that timed out) are not faults: the kernels skip the
 *     bad work, record a DA_DEV_* code and the first offending index in the
 *     workspace header, and keep going.  da_read_status reads them back.
 */
#ifndef DA_H
#define DA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DA_API __attribute__((visibility("default")))
#else
#define DA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes ------------------------------------------------------------------- */
#define DA_OK 0
#define DA_ERR_INVALID_ARG (-1) /* null pointer, negative size, inconsistent shapes */
#define DA_ERR_UNSUPPORTED (-2) /* valid but not built: head_dim, group size, page size, tile size */
#define DA_ERR_CUDA (-3)        /* a CUDA runtime call failed; see da_last_cuda_error() */
#define DA_ERR_WORKSPACE (-4)   /* workspace smaller than da_workspace_size() asks for */

/* ---- device status codes (workspace header, read with da_read_status) --------------- */
#define DA_DEV_OK 0
#define DA_DEV_BAD_SEQLEN 1 /* seq_lens[b] < 0 or > max_pages_per_req*page_size; request b treated as empty */
#define DA_DEV_BAD_PAGE 2   /* a block-table entry outside [0, num_pages); that chunk is skipped */
#define DA_DEV_TIMEOUT 3    /* a pipeline wait gave up after its time limit; results are incomplete */
#define DA_DEV_BAD_PLAN 4   /* the workspace holds no plan matching this descriptor */
#define DA_DEV_BAD_BALANCE 5 /* desc->balance is not a table for this descriptor (da_balance_set); the
                                step ran with the even split instead */

/* ---- plan kinds ---------------------------------------------------------------------- */
#define DA_PLAN_DYNAMIC 0 /* load-balanced: U tiles over C CTAs per KV head, contiguous ranges */
#define DA_PLAN_STATIC 1  /* comparator: S equal splits per request, B*S CTAs per KV head */

/* ---- output formats (da_plan_desc.out_format) ----------------------------------------- */
#define DA_OUT_BF16 0 /* out is bf16; single-segment requests are written by the decode kernel */
#define DA_OUT_F32 1  /* out is fp32; every request's result goes through the partials and da_combine */

/*
 * The problem: one decode step of a continuous batch.
 *
 *   q            bf16 [batch][num_q_heads][head_dim]            (one query token per request)
 *   k/v cache    bf16 [num_pages][num_kv_heads][page_size][head_dim]
 *                token t of request b lives in page block_table[b][t / page_size],
 *                slot t % page_size; each (page, KV head) is one contiguous
 *                page_size*head_dim*2-byte block.  Slots past a request's length
 *                may hold anything (they are never used).
 *   block_table  int32 [batch][max_pages_per_req]; only the first
 *                ceil(seq_lens[b]/page_size) entries of row b are read, and several
 *                requests may name the same page (shared prefixes).
 *   seq_lens     int32 [batch], the number of cached tokens of each request,
 *                0 for a finished or cancelled slot.
 *   out          bf16 [batch][num_q_heads][head_dim] (fp32 with out_format DA_OUT_F32);
 *                lse fp32 [batch][num_q_heads]
 *
 * Query head h reads KV head h / (num_q_heads / num_kv_heads) (consecutive
 * grouping).  out = softmax(scale * q . K^T) . V over the request's tokens and
 * lse = ln sum_t exp(scale * q . k_t) (natural log of the scaled scores); an
 * empty request gives out = 0, lse = -inf.
 *
 * Multi-query decode (q_len > 1: several new tokens per request, e.g. draft
 * tokens of speculative decoding): the q_len queries are the last q_len tokens
 * already in the cache; query i of request b sits at position
 * seq_lens[b] - q_len + i and attends causally to tokens [0, seq_lens[b] - q_len + i]
 * (none when that range is empty).  Then q, out are [batch][q_len][num_q_heads][head_dim]
 * and lse is [batch][q_len][num_q_heads]; the K/V of each request are read once for
 * all its queries.
 *
 * Supported: head_dim 64 or 128; G = num_q_heads / num_kv_heads with
 * G * q_len <= 16; page_size a positive multiple of
 * 16; num_pages * num_kv_heads * page_size below 2^31.
 */
typedef struct da_problem {
  int32_t batch;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t page_size;
  int32_t max_pages_per_req;
  int32_t num_pages;
  float scale;
  int32_t q_len; /* queries per request; 0 or 1 = plain single-token decode */
} da_problem;

/*
 * Host-side description of a plan, filled by da_plan_desc_init from host
 * arguments only.  Pass the same descriptor to every call of a step.
 */
typedef struct da_plan_desc {
  int32_t kind;            /* DA_PLAN_DYNAMIC or DA_PLAN_STATIC */
  int32_t batch;           /* B, copied from the problem */
  int32_t tile_tokens;     /* T: tokens per tile (the planner's unit of work) */
  int32_t num_ctas;        /* grid width per KV head: C (dynamic) or B*S (static) */
  int32_t splits;          /* S for a static plan, 0 for a dynamic one */
  int32_t max_segments;    /* capacity of the segment list: C+B-1 (dynamic) or B*S (static) */
  int32_t num_kv_heads;    /* Hkv, copied from the problem */
  int32_t merge_in_decode; /* 0 (default): split requests are merged by da_combine's kernel;
                              1: by the decode kernel's last CTA for each of them (no extra launch;
                              faster for batches of many long requests, slower when one request
                              is split over many CTAs).  The last CTA is found by per-request
                              counts in the workspace that only the plan resets, so with 1 every
                              decode launch needs its own plan launch before it (two decodes
                              from one plan leave split requests unmerged); with 0 a plan may
                              serve several decode launches over the same seq_lens */
  int32_t out_format;      /* DA_OUT_BF16 (default) or DA_OUT_F32: `out` holds fp32 values, for a
                              caller that merges this step's result with others (one slice of a
                              request's cache per GPU) and wants no bf16 rounding before that
                              merge.  Every segment's result then goes to the partials and
                              da_combine writes `out` for every request (also those with one
                              segment); merge_in_decode must be 0 */
  int32_t start_cost;      /* dynamic plans: units charged, besides its tiles, to the CTA that starts
                              a request (the fixed cost of a segment: loading the request's query,
                              merging and writing its result).  The plan spreads tiles plus these
                              start units evenly, so a CTA that starts many short requests gets
                              fewer tiles.  Default 2 (measured on B200 at 64-token tiles); 0 is the
                              tiles-only plan.  Must be 0 for a static plan. */
  const int32_t* balance;  /* dynamic plans: dev, a table written by da_balance_set (per-CTA weights
                              and which CTA of the plan each block of the decode grid runs), or
                              NULL (default): every CTA gets an even share.  See da_balance_set. */
  int64_t* block_times;    /* dev int64 [num_kv_heads][num_ctas][2], or NULL (default): every decode
                              launch writes, for block (x, g) of its grid, the %globaltimer (ns) at
                              its start and at its end, input to da_balance_from_times */
} da_plan_desc;

/*
 * da_plan_desc_init -- validate a problem and fix the plan geometry (and set
 * merge_in_decode = 0, out_format = DA_OUT_BF16, start_cost = 2 for a dynamic
 * plan, 0 for a static one; change those fields afterwards if wanted).
 *   kind         DA_PLAN_DYNAMIC or DA_PLAN_STATIC.
 *   tile_tokens  T > 0, a multiple of 16; 0 = default (64).
 *   width        dynamic: C, CTAs per KV head; 0 = default
 *                  max(1, floor(num_SMs * 2 / num_kv_heads)) on the current device.
 *                static: S, splits per request; 0 = default
 *                  clamp(ceil(num_SMs * 2 / (batch * num_kv_heads)), 1, 64).
 *   desc         host, out.
 * Tile size and C change only how work is spread; the result is the same up
 * to fp32 rounding.  Queries the current device only when a default is asked.
 * Errors: DA_ERR_INVALID_ARG for a bad problem or kind, DA_ERR_UNSUPPORTED for
 * a shape the kernels are not built for, DA_ERR_CUDA if a default needs a device
 * query that fails.  Source: "Tencent HPC lands in SGLang, challenging default
 * inference kernels", section "Why Tencent HPC matters for online model serving"
 * (the KV-cache work is cut into uniform tiles that a scheduler hands to CTAs):
 * T is the tile, C the number of CTAs per KV head that share the tiles.
 */
DA_API int da_plan_desc_init(const da_problem* prob, int32_t kind, int32_t tile_tokens, int32_t width,
                             da_plan_desc* desc);

/*
 * da_workspace_size -- bytes the caller must allocate on the device:
 *   ws_bytes           the plan (int32 header and work list), 16-byte aligned
 *   partial_o_bytes    fp32 [max_segments][q_len][num_q_heads][head_dim]
 *   partial_lse_bytes  fp32 [max_segments][q_len][num_q_heads]
 * Any output pointer may be NULL.  Host only; enqueues nothing.  Errors as for
 * da_plan_desc_init (a descriptor that does not match the problem is
 * DA_ERR_INVALID_ARG).  Source: as for da_plan below (the work list) and
 * da_combine (the split partials).
 */
DA_API int da_workspace_size(const da_problem* prob, const da_plan_desc* desc, size_t* ws_bytes,
                             size_t* partial_o_bytes, size_t* partial_lse_bytes);

/*
 * da_plan_workspace_size -- the same three sizes for a dynamic plan of tile
 * size tile_tokens and num_ctas CTAs per KV head (0 = the defaults of
 * da_plan_desc_init), without building a descriptor first: it is
 * da_plan_desc_init(prob, DA_PLAN_DYNAMIC, tile_tokens, num_ctas) followed by
 * da_workspace_size.  Host only; any output pointer may be NULL; errors as for
 * those two calls.  The descriptor exists because every call of a step must
 * agree on the plan geometry (T, C, the segment capacity C + B - 1, the plan
 * kind); this call is for callers that size buffers before they build one.
 * Source: as for da_plan.
 */
DA_API int da_plan_workspace_size(const da_problem* prob, int32_t tile_tokens, int32_t num_ctas, size_t* ws_bytes,
                                  size_t* partial_o_bytes, size_t* partial_lse_bytes);

/*
 * da_workspace_offsets -- word (int32) offsets of the arrays inside `ws`, for
 * callers that inspect a plan (tests, tools):
 *   off[0] header (16 words: units U, segments S, C, T, status, bad index,
 *          kind, B, max_segments, splits, 6 spare)
 *   off[1] segments, int32x4 [max_segments] = {request, cta, tile_begin, tile_end}
 *          (tiles relative to the request; tile_begin == tile_end is an empty
 *          static split)
 *   off[2] req_tile_prefix [B+1]   off[3] req_seg_begin [B+1]
 *   off[4] cta_seg_begin [num_ctas+1]
 *   off[5] req_done [B][num_kv_heads]: segments finished this step (reset by the planner)
 *   off[6] total words
 * Segments of request b are [req_seg_begin[b], req_seg_begin[b+1]); segments
 * of CTA c are [cta_seg_begin[c], cta_seg_begin[c+1]); both in tile order.
 */
DA_API int da_workspace_offsets(const da_plan_desc* desc, int64_t off[7]);

/*
 * da_plan -- dynamic (load-balanced) plan, one 1-CTA kernel.
 *   seq_lens  dev int32 [batch].
 *   ws        dev, >= ws_bytes, 16-byte aligned; overwritten (header status reset).
 * n_b = ceil(L_b / T) tiles per request, U = sum n_b; KV head by KV head, CTA c
 * gets the contiguous global tile range [floor(c*U/C), floor((c+1)*U/C)), cut
 * at request boundaries into segments.  Requests with a bad length get 0
 * tiles and DA_DEV_BAD_SEQLEN (first bad index = the lowest such b).
 * The host never reads seq_lens: the plan is rebuilt on the device every step.
 * Errors: DA_ERR_INVALID_ARG (null or unaligned pointer, a static descriptor),
 * DA_ERR_WORKSPACE (ws_bytes too small), DA_ERR_CUDA (launch refused).
 * Source: "Tencent HPC lands in SGLang, challenging default inference kernels",
 * section "Why Tencent HPC matters for online model serving": the KV-cache work
 * is cut into smaller uniform tiles and assigned by the current workload, and
 * the mapping is rebuilt as request lengths change during decoding.
 */
DA_API int da_plan(const da_problem* prob, const da_plan_desc* desc, const int32_t* seq_lens, void* ws,
                   size_t ws_bytes, void* stream);

/*
 * Balancing the plan against the speed of the SMs.
 *
 * The decode kernel streams K/V at the HBM roof while every CTA runs, but with
 * an even split the CTAs do not end together: some SMs stream a few percent
 * slower than others (on B200 the same SMs in every workload, within a process
 * and on other boxes), and the last ones end up to 9 % after the median, with
 * HBM partly idle meanwhile.  A balance table gives each CTA of the dynamic plan a
 * weight, and places the CTAs on the blocks of the decode grid so that the
 * blocks running one CTA (one per KV head) sit on SMs of like speed:
 *   - CTA c's range of units is [first(c), first(c+1)) with
 *     first(c) = c + floor((U - C) * W_c / W), W_c = sum_{k<c} w_k, W = sum w
 *     (one unit each, the rest in proportion; equal weights give the even
 *     split floor(c*U/C) exactly; with U < C the weights are not used);
 *   - block (x, g) of the decode grid runs CTA perm[g][x] of the plan.
 * The table changes who computes which tiles, never what is computed; for a
 * given table, plan and results are deterministic.  A table is measured with
 * desc->block_times over a few steps and da_balance_from_times.
 * Source of the scheme it refines: "Tencent HPC lands in SGLang, challenging
 * default inference kernels", section "Why Tencent HPC matters for online model
 * serving" (tiles handed to CTAs by the current workload); the weighting is this
 * implementation's addition.
 */

/* Words (int32) of a balance table: 4 + num_ctas + num_kv_heads * num_ctas.  Host only.
   Errors: DA_ERR_INVALID_ARG (null pointer, not a dynamic descriptor), DA_ERR_UNSUPPORTED
   (num_ctas above 2048, the planner's limit for weighted ranges). */
DA_API int da_balance_words(const da_plan_desc* desc, size_t* words);

/*
 * da_balance_set -- check a balance table on the host and copy it to the device.
 *   weights  host int32 [num_ctas], each in [1, 65536]
 *   perm     host int32 [num_kv_heads][num_ctas], each row a permutation of
 *            0 .. num_ctas-1 (row g, entry x: the CTA of the plan that block
 *            (x, g) of the decode grid runs)
 *   table    dev, da_balance_words(desc) int32 words, 4-byte aligned; then set
 *            desc->balance = table
 * Enqueues host-to-device copies on `stream`.  Pageable host arrays may be reused
 * when the call returns; page-locked ones must stay unchanged until the copies
 * have run.  Errors: DA_ERR_INVALID_ARG (null pointer, a weight out of
 * range, a row that is not a permutation), DA_ERR_UNSUPPORTED as for
 * da_balance_words, DA_ERR_CUDA (a copy refused).  A table whose header does not
 * match the descriptor it is used with is ignored by the planner, which records
 * DA_DEV_BAD_BALANCE.
 */
DA_API int da_balance_set(const da_plan_desc* desc, const int32_t* weights, const int32_t* perm, int32_t* table,
                          void* stream);

/*
 * da_balance_from_times -- a balance table from measured block times.  Host only.
 *   times      host int64 [num_kv_heads][num_ctas][2]: start and end (ns) of every
 *              block, as written to desc->block_times (e.g. per-block medians over
 *              a few steps), measured with the table (prev_weights, prev_perm)
 *              in use, NULL for the even split and the identity placement
 *   weights, perm  host out, as for da_balance_set
 * Each block's speed is its CTA's share of the work (its weight) over its time.
 * In every KV head's row the blocks are ranked by speed and block x takes CTA
 * rank(x), so that CTA c runs on the c-th slowest block of every row; its weight
 * is the mean speed of those blocks (relative, scaled to 4096 on average).  A block
 * without a usable time counts at its row's median speed.  Errors:
 * DA_ERR_INVALID_ARG (null pointer, a previous table that fails the checks of
 * da_balance_set), DA_ERR_UNSUPPORTED as for da_balance_words.
 */
DA_API int da_balance_from_times(const da_plan_desc* desc, const int64_t* times, const int32_t* prev_weights,
                                 const int32_t* prev_perm, int32_t* weights, int32_t* perm);

/*
 * da_static_plan -- static split-k plan (the comparator), same work-list format.
 * With maxT = ceil(max_b L_b / T) and chunk = ceil(maxT / S) tiles, split s of
 * request b is CTA b*S+s and covers tiles [min(s*chunk, n_b), min((s+1)*chunk, n_b)),
 * empty when s*chunk >= n_b (the CTA is launched and finds nothing to do).
 * Errors as for da_plan (a dynamic descriptor is DA_ERR_INVALID_ARG).
 * Source: "Tencent HPC lands in SGLang, challenging default inference kernels",
 * section "Why Tencent HPC matters for online model serving": the library's own
 * static split-k baseline, a fixed split policy that either leaves units idle or
 * launches empty chunks for short requests.
 */
DA_API int da_static_plan(const da_problem* prob, const da_plan_desc* desc, const int32_t* seq_lens, void* ws,
                          size_t ws_bytes, void* stream);

/*
 * da_decode_attention -- the split-KV decode kernel, grid (num_ctas, num_kv_heads).
 *   q, k_cache, v_cache, block_table, seq_lens: dev, layouts as in da_problem;
 *     k_cache and v_cache must be 16-byte aligned.
 *   ws: dev, a plan made by da_plan / da_static_plan with the same descriptor
 *     and the same seq_lens contents.
 *   partial_o, partial_lse: dev scratch, sizes from da_workspace_size.
 *   out, lse: dev outputs.  Requests with one segment are written directly
 *     (with out_format DA_OUT_F32 they too go through the partials and da_combine);
 *     the others by da_combine, or, with merge_in_decode = 1, by the decode
 *     kernel: the last CTA to finish a segment of a split request (counters in
 *     `ws`, release/acquire fences, partials read back from L2) merges it, and
 *     requests with no segment are written as 0 / -inf.
 * Each CTA streams its tiles' K and V rows (bf16, TMA, multi-stage shared
 * memory ring) and keeps, per query head of its KV group, the running max,
 * running sum and fp32 accumulator of the online softmax.
 * Errors: DA_ERR_INVALID_ARG (null pointer; k_cache, v_cache, partial_o or ws
 * not 16-byte aligned, q not 4-byte or out not 8-byte aligned; a descriptor
 * that does not match the problem), DA_ERR_UNSUPPORTED (shape), DA_ERR_CUDA
 * (tensor-map encoding or launch refused).  Data errors go to the status word
 * in `ws` (DA_DEV_BAD_PAGE, DA_DEV_TIMEOUT, DA_DEV_BAD_PLAN when `ws` holds no
 * plan for this descriptor).
 * Source: "Tencent HPC lands in SGLang, challenging default inference kernels",
 * section "Why Tencent HPC matters for online model serving": decode attention
 * over each request's cached history, whose work is uneven because one request
 * may hold a far longer context than another, and a longer history means more
 * cached data to read; the CTAs take the uniform tiles the plan gives them.
 */
DA_API int da_decode_attention(const da_problem* prob, const da_plan_desc* desc, const void* q,
                               const void* k_cache, const void* v_cache, const int32_t* block_table,
                               const int32_t* seq_lens, const void* ws, float* partial_o, float* partial_lse,
                               void* out, float* lse, void* stream);

/*
 * da_decode_attention_fp8 -- the same step over an FP8 KV cache.
 *   k_cache, v_cache  dev, FP8 E4M3 codes (OCP "E4M3FN", one byte each),
 *                     [num_pages][num_kv_heads][page_size][head_dim]; head_dim must be 128.
 *   k_scale, v_scale  dev fp32 [num_kv_heads]: the cached value of KV head g is
 *                     k_scale[g] * e4m3(code) (and likewise for V).
 * Everything else, including the plan, workspace, partials, combine and the
 * bf16 q/out and fp32 lse, is as for da_decode_attention.  K/V bytes per token
 * are halved.  Plain decode (q_len 1, at most 8 query heads per KV head,
 * merge_in_decode 0) runs on the 5th-generation tensor cores (tcgen05, E4M3
 * operands, accumulators in tensor memory): q and the softmax weights enter as
 * two E4M3 terms each (hi + lo, 8 significant bits).  The other shapes widen
 * the codes to f16 (exact), convert q to f16 and round P to f16 for a
 * warp-level MMA.
 * Source: "Tencent HPC lands in SGLang, challenging default inference
 * kernels", sections "Why Tencent HPC matters for online model serving" (a
 * longer history means more cached data to read) and "What the 48.8% TPOT
 * claim does not prove" (cache precision is one of the settings a benchmark
 * must state).
 */
DA_API int da_decode_attention_fp8(const da_problem* prob, const da_plan_desc* desc, const void* q,
                                   const void* k_cache, const void* v_cache, const float* k_scale,
                                   const float* v_scale, const int32_t* block_table, const int32_t* seq_lens,
                                   const void* ws, float* partial_o, float* partial_lse, void* out, float* lse,
                                   void* stream);

/*
 * da_combine -- merge the partials of requests with two or more segments
 * (when desc->merge_in_decode is 1 the decode kernel has done it and this call
 * enqueues nothing):
 *   LSE = M + ln sum_i exp(lse_i - M),  M = max_i lse_i,
 *   out = sum_i exp(lse_i - LSE) o_i    (fp32 sums in a fixed order, then bf16),
 * and write out = 0, lse = -inf for requests with no segment.
 *   ws, partial_o, partial_lse: dev, as written by da_plan / da_decode_attention
 *     with the same descriptor; out, lse: dev outputs (out 8-byte aligned; 16-byte
 *     aligned and fp32 with out_format DA_OUT_F32, in which case every request is
 *     written here, those with one segment included).
 * Errors: DA_ERR_INVALID_ARG (null or unaligned pointer, descriptor mismatch),
 * DA_ERR_CUDA (launch refused).
 * Source: "Tencent HPC lands in SGLang, challenging default inference kernels",
 * section "Why Tencent HPC matters for online model serving": when one request's
 * tiles go to several CTAs, each CTA holds a softmax over part of the history;
 * the log-sum-exp merge that joins them is the exact re-association of one
 * softmax (a fact of the arithmetic; the article names no merge).
 */
DA_API int da_combine(const da_problem* prob, const da_plan_desc* desc, const void* ws, const float* partial_o,
                      const float* partial_lse, void* out, float* lse, void* stream);

/*
 * da_decode_step -- one whole decode step in one call: da_plan (or da_static_plan,
 * per desc->kind), the decode (bf16 cache when k_scale and v_scale are NULL, FP8
 * E4M3 cache with per-KV-head scales when both are given) and da_combine, enqueued
 * on `stream` in that order.  Arguments, layouts, results and errors are those of
 * the three calls, and every check of all three runs before the first launch, so
 * an error return has enqueued nothing (except DA_ERR_CUDA from a launch the CUDA
 * runtime refused).  Results are those of the separate calls, bit for bit.
 * Source: "Tencent HPC lands in SGLang, challenging default inference kernels",
 * section "Why Tencent HPC matters for online model serving" (the tile-to-CTA
 * mapping is rebuilt every decode step; the step's work then runs on it).
 */
DA_API int da_decode_step(const da_problem* prob, const da_plan_desc* desc, const void* q, const void* k_cache,
                          const void* v_cache, const float* k_scale, const float* v_scale,
                          const int32_t* block_table, const int32_t* seq_lens, void* ws, size_t ws_bytes,
                          float* partial_o, float* partial_lse, void* out, float* lse, void* stream);

/*
 * da_decode_step_host -- one whole decode step for a caller whose per-step
 * inputs and outputs live in host memory, in one call, all enqueued on
 * `stream` in this order:
 *   copy seq_lens_host, block_table_host, q_host to their device copies;
 *   plan (da_plan or da_static_plan, per desc->kind); decode (bf16 cache when
 *   k_scale and v_scale are NULL, FP8 E4M3 cache with per-KV-head scales when
 *   both are given); combine;
 *   copy out_dev, lse_dev to out_host, lse_host.
 * Host buffers in page-locked memory mapped into the device's address space
 * (every cudaHostAlloc / cudaMallocHost allocation under unified addressing,
 * cudaHostRegister with cudaHostRegisterMapped) need no copy call:
 *   - when seq_lens_host, block_table_host and q_host all are, the plan launch
 *     brings them in itself: its first block reads the lengths over the bus,
 *     writes seq_lens_dev and plans, while its other blocks copy the block
 *     table into block_table_dev and, when q is at most 1 MiB, q into q_dev;
 *     a larger q is read in place by the decode kernel (q_dev stays untouched),
 *     which spreads its bus traffic over the K/V stream;
 *   - out_host and lse_host, when mapped and 16-byte aligned, are written in
 *     place by the decode and combine kernels (out_dev, lse_dev stay untouched).
 * The step computed is the one the separate calls compute (same plan, kernels
 * and results).
 *   q_host, block_table_host, seq_lens_host  host, layouts as in da_problem;
 *     read by the copies, so they must stay unchanged until the stream passes them.
 *   k_cache, v_cache, k_scale, v_scale       dev, as for da_decode_attention(_fp8).
 *   q_dev, block_table_dev, seq_lens_dev     dev, the caller's device copies of
 *     the three inputs (same sizes and alignment rules as for da_decode_attention);
 *     always written, whichever way the inputs move.
 *   ws, ws_bytes, partial_o, partial_lse     dev, as for da_plan / da_decode_attention.
 *   out_dev, lse_dev                         dev outputs, as for da_decode_attention
 *     (required; used when out_host / lse_host are not used in place).
 *   out_host, lse_host                       host, bf16 / fp32, same layouts as out, lse.
 * Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister); with
 * pageable memory the copies are correct but may block the calling thread.
 * The host outputs are valid once the stream has passed the call (e.g. after
 * cudaStreamSynchronize); the call itself does not synchronise.  Every argument
 * check of the plan, decode and combine calls runs before anything is enqueued,
 * so an error return means nothing was enqueued, except DA_ERR_CUDA from a copy
 * or launch that the CUDA runtime refused.  Source: "Tencent HPC lands in SGLang,
 * challenging default inference kernels", section "Why Tencent HPC matters for
 * online model serving" (each decode step's schedule follows the current
 * request lengths, which the serving engine owns on the host).
 */
DA_API int da_decode_step_host(const da_problem* prob, const da_plan_desc* desc, const void* q_host,
                               const int32_t* block_table_host, const int32_t* seq_lens_host, const void* k_cache,
                               const void* v_cache, const float* k_scale, const float* v_scale, void* q_dev,
                               int32_t* block_table_dev, int32_t* seq_lens_dev, void* ws, size_t ws_bytes,
                               float* partial_o, float* partial_lse, void* out_dev, float* lse_dev, void* out_host,
                               float* lse_host, void* stream);

/*
 * da_append_kv -- write each request's newest token into the paged cache
 * (the step before attention in every decode step: lengths grow by one).
 *   new_k, new_v  dev bf16 [batch][num_kv_heads][head_dim], 16-byte aligned.
 *   seq_lens      dev int32 [batch], lengths that already count the new token:
 *                 request b's rows go to position seq_lens[b]-1, i.e. page
 *                 block_table[b][(seq_lens[b]-1)/page_size], slot
 *                 (seq_lens[b]-1) % page_size.  Requests with length 0 are skipped.
 *   k_cache, v_cache  dev, written in place (16-byte aligned).
 *   status        optional dev int32 [2], or NULL: the first bad request is
 *                 recorded as {DA_DEV_BAD_SEQLEN or DA_DEV_BAD_PAGE, b} and its
 *                 row skipped; the caller clears it.
 * The engine allocates pages: the block-table entry for a new page must be set
 * before the call.  Source: "Tencent HPC lands in SGLang, challenging default
 * inference kernels", section "Why Tencent HPC matters for online model
 * serving" (request lengths change during decoding).
 */
DA_API int da_append_kv(const da_problem* prob, const void* new_k, const void* new_v, const int32_t* block_table,
                        const int32_t* seq_lens, void* k_cache, void* v_cache, int32_t* status, void* stream);

/*
 * da_plan_append -- da_append_kv and da_plan (DA_PLAN_DYNAMIC) in one launch: the
 * step's bookkeeping before attention.  Block 0 of the grid builds the plan
 * while the other blocks write every request's new K/V rows, so the appends add
 * no time to the plan; the decode kernel that follows waits for the whole grid.
 * Arguments, layouts, checks and results are those of the two calls (seq_lens
 * counts the new token; `status` receives append errors, the plan's own status
 * goes to `ws` as usual).  Source: "Tencent HPC lands in SGLang, challenging
 * default inference kernels", section "Why Tencent HPC matters for online model
 * serving" (lengths grow every step and the mapping is rebuilt every step).
 */
DA_API int da_plan_append(const da_problem* prob, const da_plan_desc* desc, const int32_t* seq_lens, void* ws,
                          size_t ws_bytes, const void* new_k, const void* new_v, const int32_t* block_table,
                          void* k_cache, void* v_cache, int32_t* status, void* stream);

/*
 * da_merge_partials -- merge results computed over disjoint token slices of
 * the same requests (e.g. one slice per GPU when a long request's KV cache is
 * spread over several GPUs and each GPU runs the decode step on its slice):
 *   LSE = M + ln sum_j exp(lse_j - M),  M = max_j lse_j,
 *   out = sum_j exp(lse_j - LSE) * out_j   (fp32 sums in part order, then bf16);
 * parts with lse = -inf (empty slices) carry no weight; all empty gives 0, -inf.
 *   part_out  dev bf16 [num_parts][rows][head_dim] (each part's `out`, 8-byte aligned)
 *   part_lse  dev fp32 [num_parts][rows]
 *   out, lse  dev bf16 [rows][head_dim], fp32 [rows]; rows = batch * q_len * num_q_heads.
 * Source: "Tencent HPC lands in SGLang, challenging default inference
 * kernels", section "Why Tencent HPC matters for online model serving"
 * (longer histories mean more cached data to read).
 */
DA_API int da_merge_partials(int32_t num_parts, int64_t rows, int32_t head_dim, const void* part_out,
                             const float* part_lse, void* out, float* lse, void* stream);

/*
 * da_merge_partials_f32 -- da_merge_partials over fp32 parts: part_out is dev fp32
 * [num_parts][rows][head_dim] (16-byte aligned), each part being the `out` of a step
 * run with out_format DA_OUT_F32, so that no part is rounded to bf16 before the
 * merge; out is bf16 as for da_merge_partials.  Same formula, order, checks and
 * errors.  Source: as for da_merge_partials.
 */
DA_API int da_merge_partials_f32(int32_t num_parts, int64_t rows, int32_t head_dim, const float* part_out,
                                 const float* part_lse, void* out, float* lse, void* stream);

/*
 * da_read_status -- copy the device status word and first bad index out of
 * `ws` (host outputs; either may be NULL).  Synchronises `stream`; the only
 * call here that does.  Errors: DA_ERR_INVALID_ARG (ws NULL), DA_ERR_CUDA (the
 * copy or the synchronisation failed).
 * Source: "Tencent HPC lands in SGLang, challenging default inference kernels",
 * section "What the 48.8% TPOT claim does not prove": serving kernels must cope
 * with boundary shapes, cancellation and changing lengths, so bad lengths and
 * page ids are skipped and reported here instead of faulting the device.
 */
DA_API int da_read_status(const void* ws, int32_t* dev_status, int32_t* bad_index, void* stream);

/* Static text for a DA_OK / DA_ERR_* return code. */
DA_API const char* da_status_string(int32_t code);

/* Static text for a DA_DEV_* device status code. */
DA_API const char* da_dev_status_string(int32_t code);

/* cudaError_t of the last failing CUDA call made by this library on this thread (0 if none). */
DA_API int32_t da_last_cuda_error(void);

/*
 * da_test_stall_next_decode -- a test of the failure path; the article has no
 * counterpart.  The next decode launch made on this thread (da_decode_attention,
 * da_decode_attention_fp8, or the decode inside da_decode_step_host or
 * da_decode_step_noalloc) runs with its load stage idle: no K/V is requested,
 * so every wait of the consumers runs out after wait_limit_us microseconds
 * (1 .. 2,000,000) instead of the usual 2 s.  The kernel then records
 * DA_DEV_TIMEOUT in the workspace status word, ends every role's loop and
 * returns; nothing is trapped, the context stays usable, and the next step is
 * unaffected.  The stalled launch's out/lse are invalid.  Returns
 * DA_ERR_INVALID_ARG for a limit out of range.
 */
DA_API int da_test_stall_next_decode(uint32_t wait_limit_us);

/* Number of SMs of the current device (host out). */
DA_API int da_device_num_sms(int32_t* num_sms);

/* Size of the library-owned device scratch used by da_decode_step_noalloc. */
#define DA_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * da_decode_step_noalloc -- one whole decode step (dynamic plan, decode,
 * combine) that allocates nothing and takes no workspace from the caller.
 * The article has no counterpart to this call.  It is for callers that cannot
 * allocate device memory where they run a step: an op inside a host framework
 * whose per-call hook must not allocate, an engine that has given nearly all
 * device memory to its KV-cache pool, or a latency-critical path where a
 * cudaMalloc (which may synchronise the device) is not acceptable.
 *   tile_tokens, num_ctas  as for da_plan_desc_init with DA_PLAN_DYNAMIC (0 = defaults).
 *   q, k_cache, v_cache, block_table, seq_lens, out, lse  dev, as for
 *     da_decode_attention (bf16 cache); the caller still allocates inputs and outputs.
 * Scratch: a static device array of DA_NOALLOC_SCRATCH_BYTES (16 MiB) inside
 * the library, reserved on every GPU that loads the library's device code and
 * held until the process exits.  A problem fits when the three sizes from
 * da_workspace_size, each rounded up to 256 bytes, sum to at most 16 MiB
 * (e.g. 64 query heads, head_dim 128, C = 37: C + B - 1 <= 507 segments, so
 * batches up to 471 requests); otherwise the call returns DA_ERR_WORKSPACE.
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  The lookup is made again when the device's
 * context is no longer the one it was made in (after a cudaDeviceReset).
 * All calls share the one array and each call overwrites it, so calls that
 * can overlap on the GPU (other streams, other threads) race and must be
 * serialised by the caller.
 * Errors: every argument check, alignment rule and tensor map of the three
 * launches is done before the first enqueue, so an error return has enqueued
 * nothing, except DA_ERR_CUDA from a launch the CUDA runtime refused.  Codes
 * as for da_plan and da_decode_attention, plus DA_ERR_WORKSPACE for a problem
 * that does not fit the scratch.  Data errors found on the device (a bad
 * length or page id, a wait that timed out) go to the status word inside the
 * scratch: read them with da_noalloc_read_status before the next call.
 */
DA_API int da_decode_step_noalloc(const da_problem* prob, int32_t tile_tokens, int32_t num_ctas, const void* q,
                                  const void* k_cache, const void* v_cache, const int32_t* block_table,
                                  const int32_t* seq_lens, void* out, float* lse, void* stream);

/*
 * da_noalloc_read_status -- da_read_status for the last da_decode_step_noalloc
 * on the current device: the device status word and first bad index of that
 * step (host outputs; either may be NULL).  Synchronises `stream`, which must
 * be the step's stream (or one ordered after it).  The next call of
 * da_decode_step_noalloc on the device overwrites the word (its plan resets
 * it).  No counterpart in the article; it exists because the step's workspace
 * is the library's own scratch, which the caller has no pointer to.
 * Errors as for da_read_status.
 */
DA_API int da_noalloc_read_status(int32_t* dev_status, int32_t* bad_index, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DA_H */
