/*
 * pkv.h -- C ABI of a paged KV-cache attention library for NVIDIA B200
 * (sm_100a).
 *
 * The operation is attention computed directly on a paged KV cache: K and V
 * rows live in a shared pool of fixed-size pages, each request owns a page
 * table listing its pages in logical order, and attention reads the pages
 * through that table, with no contiguous copy of the cache and no score
 * matrix in memory.  Sources, by page and section:
 *   - page pool, page tables, on-demand pages, and "paged FlashAttention"
 *     (paging fused with an online softmax in one kernel): tiny-llm source
 *     reading, week 3, section "Paged KV Cache"; the same course's blog
 *     summary, week 3 ("Direct paged attention + paged FlashAttention");
 *   - mixed prefill/decode batches and chunked prefill: tiny-llm source
 *     reading, sections "Continuous Batching" and "Chunked Prefill";
 *   - GQA: tiny-llm source reading, week 1;
 *   - online softmax (FlashAttention-style) and PagedAttention in CUDA:
 *     tiny-vllm article, section "From Safetensors to PagedAttention";
 *   - split-K over the KV length (flash-decoding): mini-vllm advanced series
 *     design, section 4, Phase B, adv04.
 *
 * Conventions shared by every call
 * --------------------------------
 * Types: bf16 tensors are raw IEEE bfloat16 (2 bytes).  int32 arrays are
 * little-endian int32_t.
 *
 * Pools: k_pool and v_pool are separate arrays, each laid out
 *   [num_pages][num_kv_heads][page_size][head_dim]  (bf16, row-major),
 * so the rows of one (page, KV head) form one contiguous block.  A slot
 * number names one token row of the pool: slot = page * page_size + offset.
 *
 * Page tables: page_table is [batch][max_pages] int32, row r listing request
 * r's pool pages in logical order; token j of request r is row j % page_size
 * of page page_table[r][j / page_size].  Entries past a request's last page
 * are never read.
 *
 * GQA: num_q_heads must be a multiple of num_kv_heads; query head h reads KV
 * head h / (num_q_heads / num_kv_heads).  Supported group sizes: 1, 2, 4, 8.
 * Supported head_dim: 64, 128.  Supported page_size: 16, 32.
 *
 * Memory and ownership: every pointer except the host-side pool descriptor is
 * a DEVICE pointer owned by the caller; the library allocates, frees and
 * synchronises nothing (except pkv_device_error_flags, which is documented
 * as synchronous).  Every tensor pointer must be 16-byte aligned.  Calls are
 * asynchronous on `stream` (a cudaStream_t; NULL is the legacy default
 * stream).
 *
 * Errors: each call returns PKV_OK (0) or a negative pkv_status.  Argument
 * errors are found on the host before anything is launched.  PKV_ERR_CUDA
 * reports a failed launch.  Values that live in device memory (page ids,
 * lengths, slots) cannot be checked on the host; kernels check the ones that
 * would make them read or write outside the arrays given, skip that work,
 * and raise a bit in a device-side error word that pkv_device_error_flags
 * returns.  No kernel traps.
 */
#ifndef PKV_H_
#define PKV_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle as cudaStream_t, declared here so this header needs no CUDA
 * headers. */
typedef struct CUstream_st* pkv_stream_t;

typedef struct {
  int32_t num_pages;    /* pages in each pool */
  int32_t page_size;    /* P: token rows per page (16 or 32) */
  int32_t num_kv_heads; /* Hkv */
  int32_t head_dim;     /* d (64 or 128) */
} pkv_pool_desc;

enum pkv_status {
  PKV_OK = 0,
  PKV_ERR_NULL_POINTER = -1,  /* a required pointer is NULL */
  PKV_ERR_BAD_SHAPE = -2,     /* negative size, Hq % Hkv != 0, ... */
  PKV_ERR_UNSUPPORTED = -3,   /* head_dim, page_size or group size outside the supported set */
  PKV_ERR_MISALIGNED = -4,    /* a tensor pointer is not 16-byte aligned */
  PKV_ERR_WORKSPACE = -5,     /* workspace NULL or smaller than required */
  PKV_ERR_CUDA = -6,          /* a CUDA launch or runtime call failed */
  PKV_ERR_DEVICE = -7,        /* current device is not sm_100 */
  PKV_ERR_TENSOR_MAP = -8     /* the driver rejected a TMA tensor map */
};

/* Bits of the device-side error word (see pkv_device_error_flags). */
#define PKV_FLAG_WAIT_TIMEOUT   0x1u  /* a pipeline wait hit its ~2 s limit; the kernel gave up */
#define PKV_FLAG_BAD_LENGTH     0x2u  /* a kv_len/ctx/chunk length < 0 or beyond max_pages*page_size */
#define PKV_FLAG_BAD_SLOT       0x4u  /* kv_append slot < -1 or >= num_pages*page_size (row skipped) */
#define PKV_FLAG_BAD_QUERY_ROWS 0x8u  /* cu_q_lens not non-decreasing within [0, total_q], or a chunk longer than max_q_len */
#define PKV_FLAG_BAD_PAGE       0x10u /* a page-table entry outside [0, num_pages) was seen (page 0 or zeros read instead) */
#define PKV_FLAG_INTERNAL       0x20u /* a kernel found an internal invariant broken and skipped its work */
#define PKV_FLAG_NO_FREE_PAGE   0x40u /* copy-on-write append found the free page list exhausted */

/*
 * pkv_kv_append -- write the K/V rows of this step's new tokens into pool
 * pages through a slot mapping (on-demand pages of the tiny-llm source
 * reading, "Paged KV Cache"; the slot mapping is the batch's dynamic slot ->
 * request map of its TinyLlmBatch, "Continuous Batching").
 *
 *   k_new, v_new   [num_tokens][Hkv][d] bf16
 *   slot_mapping   [num_tokens] int32; row t goes to slot slot_mapping[t] of
 *                  both pools; -1 skips the row (padding)
 *   k_pool, v_pool pools as above, written in place
 *
 * A pure bit copy: each pool row equals its source row bit for bit.  Slots
 * beyond the pool, and negative slots other than -1, raise PKV_FLAG_BAD_SLOT
 * and are skipped.  Two rows with the same slot race (one of them wins).
 * num_tokens == 0 launches nothing.
 */
PKV_API int pkv_kv_append(const void* k_new, const void* v_new, const int32_t* slot_mapping,
                  int32_t num_tokens, void* k_pool, void* v_pool, pkv_pool_desc pool,
                  pkv_stream_t stream);

/*
 * pkv_decode_workspace_bytes -- bytes of workspace pkv_paged_attn_decode
 * needs for `batch` requests whose lengths are at most max_kv_len (pass
 * max_pages * page_size).  partition_tokens as in pkv_paged_attn_decode.
 */
PKV_API size_t pkv_decode_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t head_dim,
                                  int32_t max_kv_len, int32_t partition_tokens);

/*
 * pkv_paged_attn_decode -- q_len = 1 attention of each request over its whole
 * paged context (paged FlashAttention, decode).  One KV read serves all query
 * heads of a GQA group.  Long contexts are cut into split-K partitions
 * (flash-decoding) whose partials are merged by pkv_split_k_combine's rule.
 *
 *   q           [batch][Hq][d] bf16; request r's query sits at position
 *               kv_lens[r] - 1
 *   page_table  [batch][max_pages] int32
 *   kv_lens     [batch] int32, keys per request INCLUDING the token appended
 *               this step; 0 gives a zero output (lse -inf)
 *   scale       softmax scale (usually 1/sqrt(d))
 *   partition_tokens  split-K partition length in tokens: 0 = automatic
 *               (the batch's token-heads are cut into one equal slice per
 *               warp of the launch, at least 128 tokens; a request crossing
 *               slices is merged from partials); -1 = never split; otherwise
 *               a multiple of 32 in [32, 65536]
 *   workspace   device scratch of pkv_decode_workspace_bytes(...) bytes,
 *               holding split partials, two scheduling counters and the
 *               merge-tree counters of each (request, KV head).  It must be
 *               ZERO-FILLED before its first use (a new allocation at a
 *               reused address counts as a first use); every call that
 *               completes leaves the counters at zero again, and a call
 *               whose counters reach further than the previous call's on the
 *               same address (a larger batch) clears the difference on
 *               `stream` first.  After a call that raised
 *               PKV_FLAG_WAIT_TIMEOUT, zero it again.  Calls that share a
 *               workspace must not overlap in time.
 *   out         [batch][Hq][d] bf16 (written)
 *   out_lse     [batch][Hq] fp32 natural-log softmax denominators, or NULL
 *
 * Requests that are not split are written by the partition kernel directly.
 * Split ones go through fp32 partials.  With the automatic split, the pieces
 * of a (request, KV head) are merged inside the partition kernel by a tree
 * of merges of at most 8 (d = 128) or 16 (d = 64) partials each, every node
 * merged by the warp that finishes its last child, so one kernel does the
 * whole call.  With a fixed partition, a second, combine kernel merges the
 * split requests.
 */
PKV_API int pkv_paged_attn_decode(const void* q, int32_t batch, int32_t num_q_heads,
                          const void* k_pool, const void* v_pool, pkv_pool_desc pool,
                          const int32_t* page_table, int32_t max_pages,
                          const int32_t* kv_lens, float scale, int32_t partition_tokens,
                          void* workspace, size_t workspace_bytes, void* out,
                          float* out_lse, pkv_stream_t stream);

/*
 * pkv_paged_attn_decode_flags -- pkv_paged_attn_decode with option bits
 * (the pages have no counterpart; a scheduling option of this library):
 *   PKV_DECODE_METADATA_READY  the kernel just ahead of this call on
 *               `stream` writes neither kv_lens nor page_table (for instance
 *               it is pkv_kv_append or another decode, and the tables were
 *               copied in earlier).  With the automatic split the decode
 *               kernel then plans, and reads each warp's first page-table
 *               entries, while that kernel is still finishing; q, the pools
 *               and the workspace are still read only after it completes.
 *               Ignored for a fixed partition.
 * Unknown bits give PKV_ERR_BAD_SHAPE.  flags = 0 is pkv_paged_attn_decode.
 */
#define PKV_DECODE_METADATA_READY 1u
PKV_API int pkv_paged_attn_decode_flags(const void* q, int32_t batch, int32_t num_q_heads,
                                        const void* k_pool, const void* v_pool, pkv_pool_desc pool,
                                        const int32_t* page_table, int32_t max_pages,
                                        const int32_t* kv_lens, float scale, int32_t partition_tokens,
                                        void* workspace, size_t workspace_bytes, void* out,
                                        float* out_lse, uint32_t flags, pkv_stream_t stream);

/*
 * pkv_paged_attn_decode_append -- one decode step's kv_append and decode in
 * one launch (the decode step of the tiny-llm source reading, "Paged KV
 * Cache": the new token's K/V row goes into its page, then the query
 * attends to the whole context including it).  Request r's new row
 * (k_new[r], v_new[r]) is the key and value of position kv_lens[r] - 1: the
 * warp that streams that position first writes it bit for bit to its pool
 * slot (page_table[r][(kv_lens[r] - 1) / page_size], row (kv_lens[r] - 1) %
 * page_size), makes the write visible and then streams the page as usual;
 * no other warp of the launch reads that slot.  The result equals
 * pkv_kv_append of those rows at those slots followed by
 * pkv_paged_attn_decode_flags.
 *
 *   k_new, v_new   [batch][Hkv][d] bf16, 16-byte aligned; read only
 *   k_pool, v_pool written at the batch's new slots only
 *   other arguments as pkv_paged_attn_decode_flags
 *
 * Requests with kv_lens[r] = 0 append nothing.  A new row whose page id is
 * out of range, or whose kv_lens is out of range, is not written (the call
 * raises PKV_FLAG_BAD_PAGE or PKV_FLAG_BAD_LENGTH as decode does).  No two
 * requests may share the slot of their new rows.  PKV_ERR_UNSUPPORTED in a
 * build that streams pages with bulk copies (PKV_DECODE_CPASYNC=0).
 */
PKV_API int pkv_paged_attn_decode_append(const void* q, const void* k_new, const void* v_new,
                                         int32_t batch, int32_t num_q_heads, void* k_pool,
                                         void* v_pool, pkv_pool_desc pool,
                                         const int32_t* page_table, int32_t max_pages,
                                         const int32_t* kv_lens, float scale,
                                         int32_t partition_tokens, void* workspace,
                                         size_t workspace_bytes, void* out, float* out_lse,
                                         uint32_t flags, pkv_stream_t stream);

/*
 * pkv_split_k_combine -- merge split-K partials by their log-sum-exp weights
 * (mini-vllm advanced series design, adv04 "Flash-Decoding"; the formula is
 * the plain reading: M = max_s lse_s, w_s = exp(lse_s - M),
 * o = sum_s w_s o_s / sum_s w_s, lse = M + ln sum_s w_s).
 *
 *   part_o      [batch][Hq][max_splits][d] fp32, each partial normalised
 *               within its split
 *   part_lse    [batch][Hq][max_splits] fp32 natural-log denominators;
 *               -inf marks an empty split (weight 0)
 *   num_splits  [batch] int32, splits used by each request (<= max_splits)
 *   out         [batch][Hq][d] bf16; out_lse [batch][Hq] fp32 or NULL
 *
 * A request with no non-empty split gets a zero output and lse -inf.
 */
PKV_API int pkv_split_k_combine(const float* part_o, const float* part_lse, const int32_t* num_splits,
                        int32_t batch, int32_t num_q_heads, int32_t head_dim,
                        int32_t max_splits, void* out, float* out_lse, pkv_stream_t stream);

/*
 * pkv_paged_attn_chunked_prefill -- causal attention of prompt chunks at
 * per-request context offsets, on tensor cores (tcgen05, TMEM accumulators),
 * reading keys from the paged pool (tiny-llm source reading, "Chunked
 * Prefill": a long prompt is cut into bounded chunks interleaved with decode
 * steps of other requests).
 *
 *   q            [total_q][Hq][d] bf16: request r's chunk is rows
 *                cu_q_lens[r] .. cu_q_lens[r+1]-1
 *   cu_q_lens    [batch+1] int32, non-decreasing, cu_q_lens[0] = 0,
 *                cu_q_lens[batch] <= total_q
 *   max_q_len    an upper bound on any chunk length (sizes the grid); a
 *                chunk longer than it raises PKV_FLAG_BAD_QUERY_ROWS and its
 *                rows are not written
 *   ctx_offsets  [batch] int32: tokens of request r before its chunk; chunk
 *                row i sits at position ctx_offsets[r] + i and sees keys
 *                0 .. ctx_offsets[r] + i (diagonal included)
 *   page_table   [batch][max_pages] int32; the chunk's own K/V rows must
 *                already be in the pool (pkv_kv_append first)
 *   out          [total_q][Hq][d] bf16; rows past cu_q_lens[batch] are left
 *                untouched
 */
PKV_API int pkv_paged_attn_chunked_prefill(const void* q, const int32_t* cu_q_lens, int32_t batch,
                                   int32_t num_q_heads, int32_t total_q, int32_t max_q_len,
                                   const int32_t* ctx_offsets, const void* k_pool,
                                   const void* v_pool, pkv_pool_desc pool,
                                   const int32_t* page_table, int32_t max_pages, float scale,
                                   void* out, pkv_stream_t stream);

/*
 * pkv_verify_workspace_bytes -- bytes of workspace pkv_paged_attn_verify
 * needs for total_q chunk rows whose requests hold at most max_kv_len keys
 * (pass max_pages * page_size); partition_tokens as in the call (0: sized
 * for the smallest partition the automatic choice can take, 512 keys).
 */
PKV_API size_t pkv_verify_workspace_bytes(int32_t total_q, int32_t num_q_heads, int32_t head_dim,
                                          int32_t max_kv_len, int32_t partition_tokens);

/*
 * pkv_paged_attn_verify -- causal attention of short query chunks (2 to 16
 * rows per request, e.g. the draft tokens a speculative decoder verifies)
 * over long paged contexts, split along the keys (mini-vllm advanced series
 * design, Phase B: adv03 speculative decoding's verify step and adv04
 * flash-decoding's split-K; tiny-llm blog, week 3 optional chapter).  The
 * rows and their masking are those of pkv_paged_attn_chunked_prefill (row i
 * of request r sits at ctx_offsets[r] + i and sees keys 0 .. ctx_offsets[r]
 * + i); the keys of each request are cut into partitions of
 * partition_tokens, each handled by its own CTAs on the tensor cores, and
 * the partials of split requests are merged by pkv_split_k_combine's rule in
 * a second kernel (not launched when no request is split).
 *
 *   partition_tokens  0 = automatic: no split while the (request, KV head,
 *               128-row query tile) units number at least two per SM (each
 *               CTA slot already has a unit; splitting would only add
 *               partial writes), else the fewest splits of max_pages *
 *               page_size keys that give every slot a unit, none shorter
 *               than 512 keys; otherwise a multiple of 64
 *   workspace   device scratch of pkv_verify_workspace_bytes(...) bytes,
 *               256-byte aligned; no zeroing needed (the call clears what it
 *               needs on `stream`); calls sharing it must not overlap
 *   other arguments as pkv_paged_attn_chunked_prefill
 */
PKV_API int pkv_paged_attn_verify(const void* q, const int32_t* cu_q_lens, int32_t batch,
                                  int32_t num_q_heads, int32_t total_q, int32_t max_q_len,
                                  const int32_t* ctx_offsets, const void* k_pool, const void* v_pool,
                                  pkv_pool_desc pool, const int32_t* page_table, int32_t max_pages,
                                  float scale, int32_t partition_tokens, void* workspace,
                                  size_t workspace_bytes, void* out, pkv_stream_t stream);

/*
 * pkv_paged_attn_decode_static -- pkv_paged_attn_decode without a
 * caller-provided workspace.  (The source pages have no counterpart: this is
 * a deployment convenience, not part of the method.)
 *
 * For callers that cannot allocate device memory when they run decode --
 * code running inside another allocator's callbacks, plugins whose host
 * framework hands out only input and output buffers, processes that must not
 * grow their device footprint once serving has started.  The split-K scratch
 * lives in one array of 32 MiB compiled into the library, which every GPU
 * that loads the library holds until the process exits.  The call allocates
 * and frees nothing.
 *
 *   Arguments: as pkv_paged_attn_decode, minus workspace/workspace_bytes.
 *   Limit: returns PKV_ERR_WORKSPACE, launching nothing, when
 *     pkv_decode_workspace_bytes(batch, num_q_heads, head_dim,
 *     max_pages * page_size, partition_tokens) exceeds 32 MiB.
 *   First call per device: looks up the array's device address with
 *     cudaGetSymbolAddress (for the device current at the time); make that
 *     first call before any stream capture begins.
 *   Sharing: every call on a device uses the same array, and the array keeps
 *     the previous call's contents; each call clears the scheduling counters
 *     at its start (an asynchronous memset on `stream`).  Calls whose work
 *     overlaps on the GPU (other streams, other host threads) race on the
 *     array and give wrong results: issue them one after another on one
 *     stream.
 */
PKV_API int pkv_paged_attn_decode_static(const void* q, int32_t batch, int32_t num_q_heads,
                                         const void* k_pool, const void* v_pool,
                                         pkv_pool_desc pool, const int32_t* page_table,
                                         int32_t max_pages, const int32_t* kv_lens, float scale,
                                         int32_t partition_tokens, void* out, float* out_lse,
                                         pkv_stream_t stream);

/*
 * pkv_mixed_workspace_bytes -- bytes of workspace pkv_paged_attn_mixed needs
 * for batch_dec decode requests of at most max_kv_len keys (the decode
 * workspace of the automatic split).
 */
PKV_API size_t pkv_mixed_workspace_bytes(int32_t batch_dec, int32_t num_q_heads, int32_t head_dim,
                                         int32_t max_kv_len);

/*
 * pkv_paged_attn_mixed -- a continuous batch that mixes prefill chunks and
 * decode requests in ONE persistent launch (tiny-llm source reading,
 * "Continuous Batching": prefill and decode requests handled in the same
 * round; "Chunked Prefill").  The CTAs, two per SM, pull work units from one
 * queue: the chunks' query tiles first, heaviest request first, then the
 * decode work cut into equal slices (the automatic split), so CTAs that
 * finish their chunk tiles early stream decode KV while the last tiles run.
 * No CTA waits for another.  Results are those of
 * pkv_paged_attn_chunked_prefill (chunk rows) and pkv_paged_attn_decode with
 * partition_tokens = 0 (decode rows).
 *
 *   chunk part   q_pre, cu_q_lens, batch_pre, total_q, max_q_len,
 *                ctx_offsets, page_table_pre [batch_pre][max_pages_pre], out_pre:
 *                as pkv_paged_attn_chunked_prefill
 *   decode part  q_dec, batch_dec, page_table_dec [batch_dec][max_pages_dec],
 *                kv_lens, out_dec, out_lse_dec (nullable): as
 *                pkv_paged_attn_decode
 *   workspace    pkv_mixed_workspace_bytes(...) bytes, ZERO-FILLED before
 *                its first use, as the decode workspace (the call leaves its
 *                counters at zero); calls sharing it must not overlap
 *
 * Either part may be empty.  Group size 8, or a batch whose decode plan
 * does not fit two CTAs per SM, runs as the chunk kernel followed by the
 * decode kernel (same results, two launches).
 */
PKV_API int pkv_paged_attn_mixed(const void* q_pre, const int32_t* cu_q_lens, int32_t batch_pre,
                                 int32_t total_q, int32_t max_q_len, const int32_t* ctx_offsets,
                                 const int32_t* page_table_pre, int32_t max_pages_pre,
                                 const void* q_dec, int32_t batch_dec, const int32_t* page_table_dec,
                                 int32_t max_pages_dec, const int32_t* kv_lens, int32_t num_q_heads,
                                 const void* k_pool, const void* v_pool, pkv_pool_desc pool,
                                 float scale, void* workspace, size_t workspace_bytes, void* out_pre,
                                 void* out_dec, float* out_lse_dec, pkv_stream_t stream);

/*
 * pkv_qk_norm_rope_append -- the step before attention in one kernel: the
 * separate RMSNorm of each projected query and key head row, rotary position
 * encoding of both, and the write of the new K row (and the V row, as it is)
 * into the pool (tiny-llm source reading, week 1: Qwen3's "independent
 * RMSNorm of Q and K after projection" and RoPE; week 2 and the tiny-llm
 * blog, week 2: RMSNorm and RoPE fused into one kernel to save memory round
 * trips).
 *
 *   q            [num_tokens][Hq][d] bf16, the projected queries
 *   k, v         [num_tokens][Hkv][d] bf16, the projected keys and values
 *   q_norm_weight, k_norm_weight  [d] bf16, one weight per element, shared
 *                by the heads: row x -> x / sqrt(mean(x^2) + eps) * w
 *   positions    [num_tokens] int32, the position of each token (a decode
 *                token sits at kv_len - 1, chunk row i at ctx + i)
 *   slot_mapping [num_tokens] int32, the pool slot of each token's K/V row,
 *                -1 = skip (as pkv_kv_append)
 *   rope_theta   RoPE base (> 1): element i pairs with element i + d/2 and
 *                the pair turns by position * rope_theta^(-2i/d)
 *   q_out        [num_tokens][Hq][d] bf16, the normalised, rotated queries
 *                (may be q itself)
 *
 * Arithmetic is fp32 from the bf16 inputs, rounded once to bf16; the
 * rotation angles are formed in fp64.  Bad slots raise PKV_FLAG_BAD_SLOT and
 * skip the K/V write (the query row is still written).
 */
PKV_API int pkv_qk_norm_rope_append(const void* q, const void* k, const void* v, int32_t num_tokens,
                                    int32_t num_q_heads, const void* q_norm_weight,
                                    const void* k_norm_weight, const int32_t* positions,
                                    const int32_t* slot_mapping, float eps, float rope_theta,
                                    void* q_out, void* k_pool, void* v_pool, pkv_pool_desc pool,
                                    pkv_stream_t stream);

/*
 * pkv_kv_append_cow -- append new K/V rows to page tables that may share
 * pages (a common prompt prefix), copying a shared page before writing into
 * it (mini-vllm advanced series design, Phase C, adv05 "Radix Attention +
 * Copy-on-Write"; the main series' hash + ref_count).
 *
 *   k_new, v_new   [num_tokens][Hkv][d] bf16
 *   token_req      [num_tokens] int32: the request (row of page_table) of
 *                  each new row; a request's rows contiguous and in
 *                  increasing position
 *   token_pos      [num_tokens] int32: the row's position in its request
 *   page_table     [batch][max_pages] int32, UPDATED: an entry whose page
 *                  is copied is pointed at the copy
 *   page_refcount  [num_pages] int32, UPDATED: how many table entries name
 *                  each page
 *   free_pages     [num_free] int32: pages the call may take, in order
 *   free_used      one int32 (device): the caller sets it (usually to 0);
 *                  the call adds the number of pages it took, which are
 *                  free_pages[old value ..] in some order of requests
 *
 * The page holding a request's first new row, and each page a new row
 * starts at offset 0, is settled first: if no other table entry names it,
 * the rows go in place; otherwise the request takes the next free page,
 * rows 0 .. offset-1 of the shared page (every KV head, K and V) are copied
 * into it, its table entry and counts are updated, and the new rows go
 * there.  Which sharer keeps the page and which free page each request gets
 * depend on timing; what each request reads through its table does not.
 * Pages opened by the new rows must already be in the tables (count 1).
 * An exhausted free list raises PKV_FLAG_NO_FREE_PAGE and sets the entry to
 * -1 (its rows are skipped).  Two kernels, the second launched as a
 * programmatic dependent of the first.
 */
PKV_API int pkv_kv_append_cow(const void* k_new, const void* v_new, const int32_t* token_req,
                              const int32_t* token_pos, int32_t num_tokens, int32_t* page_table,
                              int32_t batch, int32_t max_pages, int32_t* page_refcount,
                              const int32_t* free_pages, int32_t num_free, int32_t* free_used,
                              void* k_pool, void* v_pool, pkv_pool_desc pool, pkv_stream_t stream);

/* Human-readable name of a pkv_status value (static string). */
PKV_API const char* pkv_status_string(int status);

/*
 * pkv_device_error_flags -- SYNCHRONOUS: waits for the current device, then
 * returns the device-side error word (PKV_FLAG_* bits raised by any kernel of
 * this library since the last clear) in *flags, and clears it when `clear`
 * is nonzero.
 */
PKV_API int pkv_device_error_flags(uint32_t* flags, int clear);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H_ */
