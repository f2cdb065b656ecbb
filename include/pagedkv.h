/*
 * pagedkv.h -- C ABI of libpagedkv.so: paged KV-cache decode for NVIDIA B200
 * (sm_100a).
 *
 * The library implements the data-parallel hot path of PagedAttention: the
 * KV cache lives in fixed-size physical blocks of 16 tokens, each sequence
 * owns a block table that maps its logical blocks to physical ones, and
 * decode attention gathers a sequence's keys and values through that table.
 * Pages this follows (cited by title and section):
 *   [P-ASC] ascendai.csdn.net article on KV Cache and PagedAttention,
 *           §二 核心突破：PagedAttention与虚拟内存 (Fig. 2, copy-on-write),
 *           §三 进阶优化：KV Cache量化与压缩.
 *   [P-WIKI] "KV Cache 与 PagedAttention" (ai-infra-wiki), §KV cache 有多大,
 *           §碎片问题, §三个直接推论 (KV 量化 FP8/INT8).
 *   [P-WMRH] "大模型推理的KV Cache管理从内存碎片到前缀缓存的优化实战" (wmrh.cn),
 *           §二 (KVCacheBlock, BlockTable, PagedKVCache.append_slot, copy_prefix),
 *           §四 (KVQuantizationCache: asymmetric uint8 with zero point).
 *   [P-LJT] "LLM 推理优化深度解析：KV Cache、Continuous Batching、PagedAttention
 *           与量化" (blog.longjiangtao.top), §KV Cache 的本质, §MQA 与 GQA,
 *           §PagedAttention：vLLM 的显存碎片治理.
 *
 * Conventions (every function):
 *   - returns PKV_OK (0) or a negative PKV_ERR_* code; on error nothing is
 *     launched and pkv_last_error() holds a message (thread-local);
 *   - device memory is owned by the caller; the library never allocates or
 *     frees device memory and never synchronises the stream (except the
 *     explicitly synchronous pkv_device_status and validation mode);
 *   - kernels are launched on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) on the CUDA device that is current for the calling thread;
 *   - all tensors are dense, row-major, without padding, in the layouts given;
 *   - block_size must be 16 and head_dim 64 or 128.
 *
 * Cache layout (per [P-WMRH] §二 KVCacheBlock: one block stores
 * [num_heads, block_size, head_dim]):
 *   k_cache, v_cache : [num_blocks, num_kv_heads, 16, head_dim] of cache_dtype
 *                      ([..., head_dim / 2] bytes for the 4-bit formats)
 *   k_scale, v_scale : [num_blocks, num_kv_heads, 16] fp32 (quantised caches
 *                      only; one scale per token and KV head)
 *   k_zero, v_zero   : [num_blocks, num_kv_heads, 16] uint8 (PKV_U8ASYM only;
 *                      one zero point per token and KV head)
 * Token at flat slot `slot` of KV head h is row cache[slot / 16][h][slot % 16].
 *
 * Device-side checks never fault: an out-of-range slot, block id, copy pair or
 * context length is skipped (or clamped) and a bit is set in a device status
 * word that pkv_device_status() reads.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define PKV_OK               0
#define PKV_ERR_INVALID_ARG (-1)  /* bad pointer, size, shape or alignment */
#define PKV_ERR_UNSUPPORTED (-2)  /* dtype / head_dim / group size not built */
#define PKV_ERR_NO_BLOCKS   (-3)  /* block allocator out of free blocks     */
#define PKV_ERR_CUDA        (-4)  /* a CUDA runtime/driver call failed      */
#define PKV_ERR_NOT_FOUND   (-5)  /* unknown sequence id                    */
#define PKV_ERR_EXISTS      (-6)  /* sequence id already present            */

/* ---- element types ------------------------------------------------------ */
#define PKV_F16     0   /* IEEE binary16                                   */
#define PKV_BF16    1   /* bfloat16                                        */
#define PKV_I8      2   /* int8 codes, symmetric absmax, range [-127, 127] */
#define PKV_FP8E4M3 3   /* OCP FP8 E4M3 (e4m3fn) codes, absmax maps to 448 */
#define PKV_U8ASYM  4   /* uint8 codes, min/max over head_dim, with a
                           per-(token, head) scale and uint8 zero point     */
#define PKV_I4      5   /* int4 codes, symmetric absmax, range [-7, 7],
                           two per byte (element 2k in the low nibble)      */
#define PKV_FP4E2M1 6   /* OCP FP4 E2M1 codes, absmax maps to 6, two per
                           byte (element 2k in the low nibble)              */

/* ---- device status bits (pkv_device_status) ----------------------------- */
#define PKV_DEV_BAD_SLOT     1u   /* slot >= num_blocks * 16 (write skipped)       */
#define PKV_DEV_BAD_BLOCK    2u   /* block-table entry outside [0, num_blocks)     */
#define PKV_DEV_BAD_CONTEXT  4u   /* context_len > max_context_len or table width  */
#define PKV_DEV_TIMEOUT      8u   /* a bounded wait on a copy barrier gave up      */
#define PKV_DEV_BAD_PAIR    16u   /* copy pair outside [0, num_blocks)             */

/* Thread-local message describing the last error of this thread. */
const char* pkv_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int pkv_version(void);

/*
 * pkv_kv_cache_write -- slot-mapped write of new tokens' K and V.
 *   [P-WMRH] §二 append_slot: token_idx lives in logical block
 *   token_idx // block_size; the slot number slot = physical * 16 + offset
 *   names that row.  [P-LJT] §KV Cache 的本质: each decode step appends the
 *   new token's K/V to the cache.
 * k, v          : device, [num_tokens, num_kv_heads, head_dim] of in_dtype
 *                 (PKV_F16 or PKV_BF16).
 * k_cache, v_cache : device, cache layout above, cache_dtype.
 * k_scale, v_scale : device fp32 scale arrays; required (non-NULL) iff
 *                 cache_dtype is quantised (PKV_I8, PKV_FP8E4M3, PKV_U8ASYM,
 *                 PKV_I4, PKV_FP4E2M1), else ignored.
 * k_zero, v_zero : device uint8 zero-point arrays; required iff cache_dtype
 *                 is PKV_U8ASYM, else ignored (may be NULL).
 * slot_mapping  : device int64 [num_tokens]; -1 skips the token.  Slots of
 *                 one call must be distinct (duplicates race).
 * For a 16-bit cache in_dtype must equal cache_dtype and the write is a bit
 * copy.  For a quantised cache each (token, head) row x is stored as
 *   a = max|x| (fp32), s = a / 127 (INT8) or a / 448 (FP8), code = round-to-
 *   nearest-even of x / s (IEEE fp32 division), clamped to +-127 / +-448
 *   before the e4m3 conversion; a = 0 stores s = 0 and zero codes.
 * PKV_U8ASYM follows [P-WMRH] §四 quantize_key with its per-channel
 * statistics (min and max over head_dim), in IEEE fp32 from the 16-bit
 * inputs, rounding half to even:
 *   s = (max - min) / 255, z = round(-min / s) clamped to [0, 255],
 *   code = round((x - min) / s) clamped to [0, 255];
 *   s = 0 (a constant row) stores s = 0, z = 0 and zero codes.
 * The page's 128-token grouped form leaves every (token, head) row's
 * statistics unchanged (they are taken over head_dim), so it stores the same.
 * PKV_I4 / PKV_FP4E2M1 ([P-ASC] §三 FP4 KV at a quarter of fp16; [P-WMRH] §四
 * INT4): the absmax rule with s = a / 7 (INT4, codes clamped to [-7, 7]) or
 * s = a / 6 (E2M1, x / s clamped to [-6, 6], round to nearest even).
 * Alignment: k, v, k_cache, v_cache 16 bytes; scales 4 bytes.
 */
int pkv_kv_cache_write(const void* k, const void* v, void* k_cache, void* v_cache,
                       float* k_scale, float* v_scale, uint8_t* k_zero, uint8_t* v_zero,
                       const int64_t* slot_mapping, int num_tokens,
                       int num_kv_heads, int head_dim, int block_size, int num_blocks,
                       int in_dtype, int cache_dtype, void* stream);

/*
 * pkv_decode_plan -- how pkv_paged_attention_decode will divide the work.
 *   The decode streams the ordered list of (sequence, KV head, block) items
 *   through warps that each own an equal contiguous share of it (a persistent
 *   grid of one CTA per SM by default: 8 warps for 16-bit caches, 12 (8
 *   for a GQA group above 8) for quantised ones).  A (sequence, head) pair whose
 *   blocks span several warps is merged from per-warp partial softmax results
 *   by a log-sum-exp rule.  This split is the library's choice; the pages do
 *   not prescribe one.
 * partition_tokens : 0 = automatic, else a multiple of 16 capping the tokens
 *                 one warp processes (more warps, more merging).  Pass the
 *                 same value to the decode call.
 * num_partitions_out   : the number of warp streams.
 * partition_tokens_out : the most tokens one stream processes (bounded with
 *                 max_context_len).
 * workspace_bytes_out : device workspace the decode needs: arrival counters
 *                 and partial results; needed whenever there is more than one
 *                 stream.
 * Depends only on its arguments and the current device's SM count.
 */
int pkv_decode_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                    int max_context_len, int cache_dtype, int partition_tokens,
                    int* num_partitions_out, int* partition_tokens_out,
                    size_t* workspace_bytes_out);

/* Workspace bytes for the automatic plan (pkv_decode_plan with partition_tokens 0). */
int pkv_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                              int max_context_len, int cache_dtype, size_t* bytes);

/*
 * pkv_paged_attention_decode -- single-query GQA decode attention through
 * block tables.
 *   [P-LJT] §KV Cache 的本质 (one query per step attends to all cached K/V),
 *   §PagedAttention (logical blocks map to scattered physical blocks),
 *   §MQA 与 GQA (query head i uses KV head i / (num_q_heads / num_kv_heads)).
 * For every sequence s and query head i, with h = i / G, G = Hq / Hkv and
 * K_s[j], V_s[j] the rows of token j < context_lens[s] found through
 * block_tables[s][j / 16]:
 *   out[s][i] = sum_j softmax_j(scale * q[s][i] . K_s[j]) V_s[j]
 * (quantised caches are read as code * scale of that token and head, and
 * PKV_U8ASYM caches as (code - zero point) * scale, [P-WMRH] §四
 * dequantize_key).  A context length of 0 gives a zero row.
 * out            : device, [num_seqs, num_q_heads, head_dim] of q_dtype.
 * q              : device, [num_seqs, num_q_heads, head_dim] of q_dtype
 *                  (PKV_F16 or PKV_BF16; equal to cache_dtype for 16-bit
 *                  caches; for quantised caches q is converted to fp16 and
 *                  must lie within fp16 range).
 * k_cache, v_cache, k_scale, v_scale, k_zero, v_zero : as for
 *                  pkv_kv_cache_write.
 * block_tables   : device int32 [num_seqs, max_blocks_per_seq].
 * context_lens   : device int32 [num_seqs], each in [0, max_context_len] and
 *                  <= max_blocks_per_seq * 16.
 * num_blocks     : physical blocks in the pool (entries of block_tables must
 *                  lie in [0, num_blocks)).
 * max_context_len: host-side upper bound of context_lens (sizes the grid).
 * sliding_window : 0 = attend the whole context; W > 0 = a query at position
 *                  P attends keys max(0, P - W + 1) .. P only ([P-WIKI]
 *                  §三个直接推论: keep only the most recent window).  Blocks
 *                  wholly before every query's window are not read, so their
 *                  block-table entries may be stale (e.g. already freed).
 * num_q_heads / num_kv_heads = G must be an integer in [1, 16].
 * partition_tokens: as for pkv_decode_plan.
 * workspace      : device scratch of at least the planned bytes, 256-byte
 *                  aligned (may be NULL when the plan has one stream).  Its
 *                  contents need no preparation: it starts with the arrival
 *                  counters (tagged with a per-call epoch) and the partials
 *                  follow them.  The library keeps a host-side record, per
 *                  (device, workspace address), of how many leading bytes hold
 *                  counters since the last call, and clears the rest of a
 *                  call's counter area with an asynchronous memset on the
 *                  call's stream: on the first use of an address, and when a
 *                  call has more (sequence, KV head) pairs than the previous
 *                  one on it.  Nothing else may write the workspace between
 *                  calls.  One workspace serves one call at a time: calls that
 *                  overlap on the GPU need separate workspaces.
 * The kernel is launched with programmatic stream serialisation: it may
 * start while the immediately preceding kernel on the stream is finishing,
 * and waits for that kernel to complete before it reads q, the caches, or
 * writes out.  (This library's KV write kernel allows that early start; any
 * other preceding kernel completes first as usual.)
 * Alignment: k_cache, v_cache, scales and zero points 16 bytes; q, out 4
 * bytes.
 */
int pkv_paged_attention_decode(void* out, const void* q,
                               const void* k_cache, const void* v_cache,
                               const float* k_scale, const float* v_scale,
                               const uint8_t* k_zero, const uint8_t* v_zero,
                               const int32_t* block_tables, const int32_t* context_lens,
                               int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                               int block_size, int num_blocks, int max_blocks_per_seq,
                               int max_context_len, float scale, int sliding_window, int q_dtype, int cache_dtype,
                               int partition_tokens, void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * pkv_multi_query_plan -- the work division pkv_paged_attention_multi_query
 *   will use (as pkv_decode_plan; the (token, head) columns of one KV head
 *   are cut into tiles of 8 or 16, each tile a pair of its own in the work
 *   list).  max_query_len bounds the new tokens of any sequence.  When the
 *   query-major kernel applies (see pkv_paged_attention_multi_query),
 *   *num_streams_out is its CTA count, num_seqs * num_kv_heads * the pairs
 *   of 128-row tiles of the longest run, and *partition_tokens_out the
 *   context bound rounded up to whole blocks (each CTA walks all its keys);
 *   *workspace_bytes_out is still the other kernel's need, used when q or
 *   out is not 16-byte aligned or the scale is not positive.
 */
int pkv_multi_query_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                         int max_context_len, int max_query_len, int cache_dtype,
                         int partition_tokens, int* num_streams_out,
                         int* partition_tokens_out, size_t* workspace_bytes_out);

/*
 * pkv_paged_attention_multi_query -- attention of several new tokens per
 * sequence over the paged cache, for chunked prefill (a long prompt cut into
 * chunks interleaved with decode steps, [P-LJT] §Continuous Batching and
 * §调优心法) and the verify pass of speculative decoding (the large model
 * scores all drafted positions in one pass, [P-LJT] §投机解码).
 * The n_s = query_start_loc[s+1] - query_start_loc[s] new tokens of sequence
 * s are the last n_s of its context_lens[s] tokens (their K/V already written
 * with pkv_kv_cache_write); new token t (0-based) attends keys
 * 0 .. context_lens[s] - n_s + t, i.e. causally among the new tokens and to
 * every earlier token:
 *   out[r][i] = sum_{j <= ctx - n + t} softmax_j(scale * q[r][i] . K_s[j]) V_s[j]
 * for r = query_start_loc[s] + t, KV head i / G as in decode.
 * out, q          : device, [num_q_tokens, num_q_heads, head_dim] of q_dtype,
 *                   rows grouped by sequence.
 * query_start_loc : device int32 [num_seqs + 1], non-decreasing, from 0 to
 *                   num_q_tokens; each n_s <= max_query_len and <= context.
 * max_query_len   : host-side bound of n_s (sizes the work list).
 * Everything else as for pkv_paged_attention_decode (with
 * pkv_multi_query_plan's workspace size).  Rows of new tokens beyond a
 * sequence's context or beyond max_query_len (invalid inputs) are written as
 * zeros and raise PKV_DEV_BAD_CONTEXT; query_start_loc entries outside
 * [0, num_q_tokens] are clamped to it.  With every n_s = 1 the result equals
 * decode.
 * Kernels: when max_query_len * (num_q_heads / num_kv_heads) >= 128, the
 * cache is 16-bit, head_dim is 64 or 128, 128 is a multiple of the group,
 * partition_tokens is 0, scale > 0 and q and out are 16-byte aligned, a
 * query-major kernel on the tcgen05 tensor cores runs (two tiles of 128
 * (token, head) rows per CTA sharing 128-key K/V tiles; scores,
 * probabilities and outputs in TMEM; sequences started longest first; no
 * workspace used); otherwise the decode kernel's multi-query mode (16
 * (token, head) columns per pass).  Both give the same result up to
 * rounding (bf16 probabilities are rounded toward zero in the first, to
 * nearest in the second).
 */
int pkv_paged_attention_multi_query(void* out, const void* q,
                                    const void* k_cache, const void* v_cache,
                                    const float* k_scale, const float* v_scale,
                                    const uint8_t* k_zero, const uint8_t* v_zero,
                                    const int32_t* block_tables, const int32_t* context_lens,
                                    const int32_t* query_start_loc, int num_seqs,
                                    int num_q_tokens, int max_query_len,
                                    int num_q_heads, int num_kv_heads, int head_dim,
                                    int block_size, int num_blocks, int max_blocks_per_seq,
                                    int max_context_len, float scale, int sliding_window, int q_dtype, int cache_dtype,
                                    int partition_tokens, void* workspace, size_t workspace_bytes,
                                    void* stream);

/*
 * pkv_paged_attention_decode_noalloc -- pkv_paged_attention_decode for
 * callers that cannot allocate device memory (no counterpart on the pages;
 * this is a library convenience).  Typical such callers: a plugin inside a
 * host framework that owns every device allocation and passes the plugin only
 * its input and output buffers, or a latency-critical loop in which a
 * cudaMalloc could synchronise the device.  The arguments mean what they mean
 * for pkv_paged_attention_decode; there is no workspace argument.
 *   - The split-KV partials go to one library-owned device array of
 *     PKV_NOALLOC_SCRATCH_BYTES (a file-scope __device__ array: every GPU that
 *     loads the library holds it until the process exits).  With
 *     partition_tokens = 0, when the automatic plan needs more
 *     (pkv_decode_plan's workspace_bytes_out), the call runs the same work in
 *     fewer, longer warp streams, as many as the array holds; a call that
 *     still needs more (or whose explicit partition does) is rejected with
 *     PKV_ERR_INVALID_ARG before anything is launched.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it for the
 *     device's current CUDA context (after a device reset, the first call
 *     looks it up again); make that first call before any stream capture.
 *   - Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents.  Its arrival counters are cleared like those of a caller's
 *     workspace (see pkv_paged_attention_decode: an asynchronous memset on
 *     the first call and whenever a call has more (sequence, KV head) pairs
 *     than the one before); partials are written before they are read.
 *     Calls that overlap on the GPU (concurrent streams, or other threads)
 *     race on it and give wrong results; serialise them, e.g. on one stream.
 */
#define PKV_NOALLOC_SCRATCH_BYTES (16u << 20)

int pkv_paged_attention_decode_noalloc(void* out, const void* q,
                                       const void* k_cache, const void* v_cache,
                                       const float* k_scale, const float* v_scale,
                                       const uint8_t* k_zero, const uint8_t* v_zero,
                                       const int32_t* block_tables, const int32_t* context_lens,
                                       int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                       int block_size, int num_blocks, int max_blocks_per_seq,
                                       int max_context_len, float scale, int sliding_window, int q_dtype, int cache_dtype,
                                       int partition_tokens, void* stream);

/*
 * pkv_copy_blocks -- copy whole physical blocks (K, V and, for quantised
 * caches, their scales and zero points): for each pair p, block
 * src_dst_pairs[2p+1] becomes a copy of block src_dst_pairs[2p].  This is
 * the copy behind copy-on-write prefix sharing ([P-ASC] §二 写时复制; [P-LJT] §意外的收获：prefix sharing).
 * src_dst_pairs : device int32 [num_pairs, 2].  Destinations must be
 *                 distinct and no destination may also be a source in the
 *                 same call (then the result equals copying all pairs at once).
 * k_scale, v_scale : required iff cache_dtype is quantised.
 * k_zero, v_zero   : required iff cache_dtype is PKV_U8ASYM.
 * Alignment: caches, scales and zero points 16 bytes.
 */
int pkv_copy_blocks(void* k_cache, void* v_cache, float* k_scale, float* v_scale,
                    uint8_t* k_zero, uint8_t* v_zero,
                    const int32_t* src_dst_pairs, int num_pairs,
                    int num_kv_heads, int head_dim, int block_size, int num_blocks,
                    int cache_dtype, void* stream);

/*
 * pkv_device_status -- read (and optionally clear) the device status word of
 * the current device: an OR of PKV_DEV_* bits set by kernels since the last
 * clear.  Synchronous (waits for the device).
 */
int pkv_device_status(unsigned int* status_out, int clear);

/*
 * pkv_set_validation -- when on, every launch first copies its index arrays
 * (slot_mapping, block_tables, context_lens, src_dst_pairs) to the host,
 * synchronously, and rejects invalid entries with PKV_ERR_INVALID_ARG before
 * launching anything.  Off by default (the hot path stays asynchronous).
 * Process-wide.
 */
int pkv_set_validation(int on);

/* ======================================================================= *
 * Host block allocator (CPU only; no device memory).  [P-WMRH] §二:
 * BlockTable keeps a free list and allocate() pops its end (LIFO), returning
 * failure when empty; free() pushes back; append_slot() maps logical block
 * token // 16 and allocates on demand; copy_prefix() lets a child alias the
 * parent's first ceil(prefix / 16) blocks and bumps their reference counts.
 * Copy-on-write ([P-ASC] §二; [P-LJT] §prefix sharing): appending into a
 * block with reference count > 1 takes a fresh block, reports (old, new) for
 * pkv_copy_blocks and drops the old count; the last holder writes in place.
 * A handle is not thread-safe; use one per thread or lock around it.
 * ======================================================================= */

/* Create an allocator over blocks [0, num_blocks).  initial_free_order
 * (host, may be NULL) gives the free list, popped from its end; NULL means
 * 0, 1, ..., num_blocks-1 (so block num_blocks-1 is handed out first). */
int pkv_alloc_create(int num_blocks, int block_size, const int32_t* initial_free_order,
                     void** handle_out);
int pkv_alloc_destroy(void* handle);

/* Register an empty sequence. */
int pkv_seq_add(void* handle, int64_t seq_id);

/* child shares parent's first ceil(prefix_len / 16) blocks and has length
 * prefix_len (prefix_len = -1: the whole parent). */
int pkv_seq_fork(void* handle, int64_t parent, int64_t child, int prefix_len);

/* Append n_tokens to a sequence.  slots_out (host int64 [n_tokens]) receives
 * each token's slot; cow_pairs_out (host int32 [cow_cap, 2]) the (src, dst)
 * block copies that must run before the tokens are written; num_cow_out their
 * count.  Transactional: on PKV_ERR_NO_BLOCKS nothing changed. */
int pkv_seq_append(void* handle, int64_t seq_id, int n_tokens, int64_t* slots_out,
                   int32_t* cow_pairs_out, int cow_cap, int* num_cow_out);

/* One token for each of n sequences (a decode step), transactional over the
 * whole batch.  slots_out [n]; cow pairs as above. */
int pkv_batch_append(void* handle, const int64_t* seq_ids, int n, int64_t* slots_out,
                     int32_t* cow_pairs_out, int cow_cap, int* num_cow_out);

/* Export block tables (host int32 [n, max_blocks], unused entries 0) and
 * context lengths (host int32 [n]) of n sequences. */
int pkv_batch_tables(void* handle, const int64_t* seq_ids, int n, int32_t* block_tables_out,
                     int max_blocks, int32_t* context_lens_out);

/* Release a sequence: every block's count drops by one; blocks reaching 0
 * return to the free list in table order. */
int pkv_seq_free(void* handle, int64_t seq_id);

int pkv_seq_block_table(void* handle, int64_t seq_id, int32_t* out, int cap, int* n_out);
int pkv_seq_len(void* handle, int64_t seq_id, int* len_out);
int pkv_block_refcount(void* handle, int32_t block, int* rc_out);

/* Free blocks, blocks shared by more than one sequence, and the longest run
 * of consecutive free block ids ([P-WMRH] §三 metrics table: fragmentation =
 * total free / largest contiguous free run). */
int pkv_alloc_stats(void* handle, int* num_free, int* num_shared, int* largest_free_run);

/* ======================================================================= *
 * Automatic prefix caching in the allocator ([P-WMRH] §三
 * AutomaticPrefixCache / PrefixRadixTree): the longest cached prefix of a
 * request's token ids is found in a radix tree and rounded down to whole
 * blocks; the cache key is the 16-byte BLAKE2b digest of the token ids as
 * little-endian int32; least recently used entries are evicted.
 *   - Every full block of a cached sequence is one tree node whose edge is
 *     that block's 16 token ids (the KV of a sequence covers each of its
 *     prefixes), so a hit is the longest run of whole leading blocks that
 *     some cached sequence shares with the request.
 *   - The cache holds one reference on each cached block.  A cached block is
 *     evictable when no sequence holds it and no cached block lies below it
 *     in the tree; eviction takes the least recently used evictable block (a
 *     logical clock ticks once per insert / match / add-cached call; ties go
 *     to the older node) and returns it to the free list.
 *   - An append that finds the free list empty evicts one block that way
 *     before failing with PKV_ERR_NO_BLOCKS (a failed append restores the
 *     cache too).
 * ======================================================================= */

/* BLAKE2b-128 (RFC 7693, no key) of n token ids as little-endian int32;
 * key_out: 16 bytes. */
int pkv_prefix_key(const int32_t* token_ids, int n_tokens, uint8_t* key_out);

/* Cache the first floor(min(n_tokens, length) / 16) blocks of a sequence
 * whose first tokens are token_ids (host int32 [n_tokens]).  A block whose
 * prefix is already cached is left as it is (its last use is refreshed);
 * newly_cached_out (nullable) counts blocks that became cached. */
int pkv_prefix_cache_insert(void* handle, int64_t seq_id, const int32_t* token_ids, int n_tokens,
                            int* newly_cached_out);

/* Longest cached whole-block prefix of token_ids: hit_tokens_out (a multiple
 * of 16), key_out (nullable; 16 bytes: the key of the hit prefix, zeros on a
 * miss).  Counts one lookup, and one hit when hit_tokens > 0. */
int pkv_prefix_cache_match(void* handle, const int32_t* token_ids, int n_tokens, int* hit_tokens_out,
                           uint8_t* key_out);

/* Register a sequence whose block table starts with the blocks of the
 * longest cached prefix of token_ids (their counts + 1) and whose length is
 * the hit (hit_tokens_out); the caller then appends and computes the rest.
 * A fully cached request gets all its tokens; pass one token fewer to have
 * the last one recomputed. */
int pkv_seq_add_cached(void* handle, int64_t seq_id, const int32_t* token_ids, int n_tokens,
                       int* hit_tokens_out);

/* Evict until at most max_cached_blocks blocks are cached or nothing more is
 * evictable ([P-WMRH] §三 evict_lru, with the budget in blocks). */
int pkv_prefix_cache_evict(void* handle, int max_cached_blocks, int* evicted_out);

/* Cached blocks, evictable blocks now, lookups, hits (hit rate = hits /
 * lookups, [P-WMRH] §三 metrics table), evictions so far.  Outputs nullable. */
int pkv_prefix_cache_stats(void* handle, int* cached_blocks, int* evictable_blocks, int64_t* lookups,
                           int64_t* hits, int64_t* evictions);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
