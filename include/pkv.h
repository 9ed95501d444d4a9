/*
 * pkv.h -- C ABI of libpkv.so, a B200 (sm_100a) library for the hot path of a
 * paged KV cache: the slot-mapped write of new tokens, the copy-on-write block
 * copy, and decode attention read through per-sequence block tables.
 *
 * Method (pages on vLLM's PagedAttention):
 *   - The KV cache is split into fixed-size blocks of `block_size` tokens that
 *     can sit anywhere in a preallocated physical pool; a per-sequence block
 *     table maps logical block j to a physical block id, like a page table
 *     (wkbse.com "加速 LLM 推理：深入了解 vllm 引擎", section 3.1;
 *     intelliparadigm.com article 2012396, section 2.1, storage levels 1-2).
 *   - Token position pos lives in logical block pos / block_size at offset
 *     pos % block_size (ruibaoantu.com article 3727998, section 1.1 sketch).
 *   - The attention kernel finds the physical blocks through the table and
 *     reads the non-contiguous K/V from them (wkbse.com section 3.1).
 *   - Shared blocks serve several sequences; a shared block is copied before a
 *     sequence writes into it (copy-on-write, intelliparadigm.com section 2.1).
 *
 * Physical pool layout (both caches, bf16):
 *     cache[num_blocks][num_kv_heads][block_size][head_dim]
 * so one (block, head) tile of block_size x head_dim is contiguous and every
 * token row is head_dim*2 bytes (a multiple of 16).  A slot names one token row
 * of the pool: slot = physical_block * block_size + offset.
 *
 * Conventions shared by every call:
 *   - Pointers are device pointers owned by the caller unless stated "host".
 *     The library allocates no device memory; it keeps one 4-byte device error
 *     word per GPU and the scratch array of paged_attn_decode_static_ws (both
 *     module globals).
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and returns before it finishes.
 *   - Host validation covers shapes, null pointers and 16-byte alignment only;
 *     the host never reads device arrays.  Data-dependent faults found on the
 *     device (slot or block id outside the pool, context length outside the
 *     table) set bits in the device error word, and the offending access is
 *     skipped or clamped.  Read and clear it with pkv_get_device_error().
 *   - Supported: head_dim in {64, 128}; block_size a multiple of 16 in
 *     [16, 1024]; num_q_heads = g * num_kv_heads with 1 <= g <= 16.
 */
#ifndef PKV_H_
#define PKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *pkv_stream_t; /* same type as cudaStream_t */

typedef enum pkv_status {
    PKV_OK = 0,
    PKV_EINVAL = 1,      /* bad size, null pointer, misaligned pointer, bad workspace */
    PKV_ERANGE = 2,      /* host-visible index outside the pool (copy pairs) */
    PKV_EALIAS = 3,      /* copy pairs: a destination repeats or is also a source */
    PKV_ECUDA = 4,       /* a CUDA runtime/driver call failed (launch, tensor map) */
    PKV_EDEVICE = 5,     /* pkv_get_device_error found a non-zero device error word */
    PKV_EUNSUPPORTED = 6 /* valid request outside the supported shapes */
} pkv_status;

/* Bits of the device error word. */
#define PKV_DEVERR_SLOT 0x1u     /* pkv_write: slot >= num_blocks * block_size (token skipped) */
#define PKV_DEVERR_BLOCK 0x2u    /* decode: block table entry outside [0, num_blocks) (tile reads zeros) */
#define PKV_DEVERR_CONTEXT 0x4u  /* decode: context_lens[s] < 0 or above the table / max_context_len (clamped) */
#define PKV_DEVERR_TIMEOUT 0x8u  /* a bounded on-chip wait gave up (the call's results are invalid) */
#define PKV_DEVERR_LAYOUT 0x10u  /* decode: shared memory window not 1 KB-aligned (results invalid) */

/* Describes one physical pool (k_cache and v_cache share it).  Calls that
 * move whole blocks (copy, device copy, swap) size them by kv_dtype; write,
 * decode and prefill accept only their own element type (else PKV_EINVAL). */
typedef struct pkv_pool {
    int32_t num_blocks;
    int32_t num_kv_heads;
    int32_t block_size;
    int32_t head_dim;
    int32_t kv_dtype; /* PKV_KV_BF16 (0) or PKV_KV_E4M3 (1): the element type of k_cache / v_cache */
} pkv_pool;

#define PKV_KV_BF16 0 /* bf16 elements, 2 bytes */
#define PKV_KV_E4M3 1 /* FP8 e4m3 codes, 1 byte (see pkv_write_fp8) */

/*
 * pkv_write -- slot-mapped write of new tokens' K/V into their blocks.
 * Follows: new tokens' KV go into a block of the sequence and the block table
 * is updated (wkbse.com section 3.1, "flexible memory management"); the slot
 * decodes as block = slot / block_size, offset = slot % block_size
 * (ruibaoantu.com section 1.1).
 *
 *   k, v          bf16 [num_tokens][num_kv_heads][head_dim], contiguous, 16-B aligned
 *   slot_mapping  int64 [num_tokens]; slot < 0 marks a padding token (skipped)
 *   k_cache, v_cache  pool of layout above, 16-B aligned
 * For every token t with slot >= 0 and every kv head h:
 *   cache[slot / bs][h][slot % bs][:] = k[t][h][:]   (same for v), bit-exact.
 * Two tokens with the same slot: which one lands is unspecified.
 * Slots >= num_blocks * block_size set PKV_DEVERR_SLOT and are skipped.
 * num_tokens == 0 is a no-op.
 */
pkv_status pkv_write(const void *k, const void *v, const int64_t *slot_mapping, int32_t num_tokens,
                     void *k_cache, void *v_cache, pkv_pool pool, pkv_stream_t stream);

/*
 * pkv_copy_blocks -- copy-on-write block copy for shared prefixes
 * (intelliparadigm.com section 2.1: COW for prefix sharing; a block holds a
 * key region and a value region).
 *
 *   src_dst_pairs  HOST int32 [num_pairs][2] = (src, dst) physical block ids.
 *                  The block manager that decides copy-on-write lives on the
 *                  host, so the pairs are read there, validated completely and
 *                  passed to the kernel by value (no device staging buffer).
 * For every pair, block dst of both caches (all heads, all offsets) becomes a
 * bit-exact copy of block src.  The pairs act as if simultaneous; to make that
 * unambiguous a destination may appear only once and may not be any pair's
 * source (PKV_EALIAS).  Ids outside [0, num_blocks) give PKV_ERANGE.  Nothing
 * is enqueued when validation fails.  num_pairs == 0 is a no-op.
 */
pkv_status pkv_copy_blocks(const int32_t *src_dst_pairs, int32_t num_pairs, void *k_cache,
                           void *v_cache, pkv_pool pool, pkv_stream_t stream);

/*
 * pkv_swap_out / pkv_swap_in -- move whole blocks between the pool and host
 * memory: cold blocks go to CPU memory when device memory runs short
 * (intelliparadigm.com section 2.1, item 3), and a preempted request's KV
 * cache is swapped out and later back in (ai-stack.site "Nano-vLLM 原理",
 * practice 5).  The block manager picks the blocks on the host (see
 * pkv_lru_victims); one launch per 2048 ids moves them.
 *
 *   block_ids        HOST int32 [n], ids in [0, num_blocks) (else PKV_ERANGE)
 *   host_k, host_v   pinned host memory the device can address (cudaHostAlloc /
 *                    cudaMallocHost / a pinned torch tensor), 16-B aligned, each
 *                    n * num_kv_heads * block_size * head_dim bf16, packed in
 *                    list order: entry i is [num_kv_heads][block_size][head_dim].
 *                    Pageable or device memory gives PKV_EINVAL.
 * swap_out: host_k[i] / host_v[i] become bit-exact copies of block ids[i] of
 *           k_cache / v_cache (the pool is only read; ids may repeat).
 * swap_in:  block ids[i] of both caches becomes host_k[i] / host_v[i]; ids must
 *           be distinct (PKV_EALIAS).
 * Asynchronous on `stream`: the host buffers must stay alive and untouched
 * until the stream reaches the call.  n == 0 is a no-op; nothing is enqueued
 * when validation fails.
 */
pkv_status pkv_swap_out(const void *k_cache, const void *v_cache, pkv_pool pool, const int32_t *block_ids,
                        int32_t n, void *host_k, void *host_v, pkv_stream_t stream);
pkv_status pkv_swap_in(const void *host_k, const void *host_v, const int32_t *block_ids, int32_t n,
                       void *k_cache, void *v_cache, pkv_pool pool, pkv_stream_t stream);

/*
 * pkv_lru_victims -- host-side choice of blocks to swap out, least recently
 * used first (intelliparadigm.com section 2.1, item 3: block heat managed by
 * LRU).  Among blocks b with evictable[b] != 0 (host arrays of num_blocks),
 * writes the min(k, #evictable) with the oldest last_use[b] (smaller is older;
 * equal values by lower id) to victims, oldest first, and their number to
 * *count.  Pure host code: no device memory, no stream.
 */
pkv_status pkv_lru_victims(const int64_t *last_use, const uint8_t *evictable, int32_t num_blocks, int32_t k,
                           int32_t *victims, int32_t *count);

/*
 * pkv_decode_workspace_bytes -- device scratch needed by paged_attn_decode for
 * these sizes (a work list and the split-K partial results).  Returns 0 for
 * invalid sizes.  partition_tokens as for paged_attn_decode (0 = library's
 * choice).
 */
size_t pkv_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                  int32_t head_dim, int32_t max_context_len,
                                  int32_t partition_tokens);

/*
 * paged_attn_decode -- decode attention of one query token per sequence over
 * its paged K/V (wkbse.com section 3.1: the custom kernel looks up the block
 * table and reads the non-contiguous blocks; section 3.3: scale, softmax and
 * weighted sum fused in one kernel).  For every sequence s and query head hq:
 *   hkv   = hq / (num_q_heads / num_kv_heads)              (contiguous GQA groups)
 *   z_i   = scale * <q[s][hq], K_i>,  i < context_lens[s]
 *   out[s][hq] = sum_i softmax(z)_i * V_i
 * where K_i, V_i are the rows of position i found through
 * block_tables[s][i / block_size] at offset i % block_size.  Accumulation is
 * fp32 with an online softmax; out is rounded to bf16 (nearest-even).  MHA
 * (one query head per kv head) runs on CUDA cores with fp32 weights; GQA
 * groups of 2 to 16 heads run on the tensor cores, where the softmax weights
 * enter the weighted sum rounded to bf16.
 * Long contexts are split into partitions of partition_tokens tokens whose
 * (max, sum, acc) are merged by a log-sum-exp reduce.
 *
 *   q             bf16 [num_seqs][num_q_heads][head_dim], 16-B aligned
 *   k_cache, v_cache  pool (layout above); pool.num_kv_heads == num_kv_heads
 *   block_tables  int32 [num_seqs][max_blocks_per_seq]; entries at and after
 *                 ceil(context_len / block_size) are never read
 *   context_lens  int32 [num_seqs]; 0 gives a zero output row
 *   max_context_len  host upper bound of context_lens (sizes the workspace)
 *   partition_tokens 0 = library's choice (512 tokens, or 2048 when
 *                 max_context_len > 16384), else a multiple of 16 in [16, 65536]
 *   out           bf16 [num_seqs][num_q_heads][head_dim], 16-B aligned
 *   workspace     device scratch of at least pkv_decode_workspace_bytes(...)
 *                 bytes, 256-B aligned; contents need no initialisation; one
 *                 workspace must not be used by two calls that run concurrently
 * Launches up to three kernels on `stream` (plan, attention, reduce).
 */
pkv_status paged_attn_decode(const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *block_tables, int32_t max_blocks_per_seq,
                             const int32_t *context_lens, int32_t num_seqs, int32_t num_q_heads,
                             float scale, int32_t num_kv_heads, void *out, pkv_pool pool,
                             int32_t max_context_len, int32_t partition_tokens, void *workspace,
                             size_t workspace_bytes, pkv_stream_t stream);

/*
 * paged_attn_decode_static_ws -- paged_attn_decode for callers that cannot
 * allocate device memory.  The pages have no counterpart of this call; it is
 * a convenience of this library.
 *
 * Some callers have no way to obtain scratch memory: a plugin running inside
 * a host engine that has reserved all device memory for its own pools and
 * offers plugins no allocation hook, or a latency-critical path where a
 * cudaMalloc (which can synchronise the device) is not acceptable.  This
 * entry point takes the same arguments as paged_attn_decode except the
 * workspace: its scratch is a file-scope device array of
 * PKV_STATIC_WS_BYTES bytes inside libpkv.so.  Every GPU that loads the
 * library holds that array until the process exits.  The call allocates
 * nothing.
 *
 *   - A request whose pkv_decode_workspace_bytes(...) exceeds
 *     PKV_STATIC_WS_BYTES returns PKV_EUNSUPPORTED and enqueues nothing;
 *     invalid sizes return PKV_EINVAL as in paged_attn_decode.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is kept for the life of the
 *     process, which assumes one CUDA context per device for that long: after
 *     a cudaDeviceReset, or with a driver-API context other than the primary
 *     one current, the kept address no longer names this array.
 *   - All calls on a device share the one array, and it keeps the previous
 *     call's contents.  Nothing in it needs to start at zero (every call
 *     rewrites what it reads).  Calls whose kernels overlap on the GPU (for
 *     example on two streams) race on the array; order them on one stream.
 */
#define PKV_STATIC_WS_BYTES ((size_t)32 << 20)

pkv_status paged_attn_decode_static_ws(const void *q, const void *k_cache, const void *v_cache,
                                       const int32_t *block_tables, int32_t max_blocks_per_seq,
                                       const int32_t *context_lens, int32_t num_seqs, int32_t num_q_heads,
                                       float scale, int32_t num_kv_heads, void *out, pkv_pool pool,
                                       int32_t max_context_len, int32_t partition_tokens,
                                       pkv_stream_t stream);

/*
 * pkv_prefill_workspace_bytes -- device scratch needed by paged_attn_prefill
 * (its work list).  Returns 0 for invalid sizes.
 */
size_t pkv_prefill_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                   int32_t max_query_len);

/*
 * paged_attn_prefill -- chunked-prefill attention: several new query tokens per
 * sequence, each attending causally to the sequence's cached context read
 * through the block table (wkbse.com section 3.1; a token sees itself and the
 * tokens before it).  The chunk's own K/V must already be in the cache
 * (pkv_write of its tokens' slots).  For sequence s with q_len =
 * query_start[s+1] - query_start[s] and ctx = context_lens[s] (counting the
 * chunk), query row t = query_start[s] + i is at position pos = ctx - q_len + i
 * and, for every query head hq (kv head hq / (num_q_heads / num_kv_heads)):
 *   out[t][hq] = sum_{j <= pos} softmax_j(scale * <q[t][hq], K_j>) V_j
 * in fp32 with bf16 (nearest-even) output.  decode is the case q_len = 1.
 *
 *   q, out        bf16 [num_tokens][num_q_heads][head_dim], 16-B aligned; query_start[num_seqs]
 *                 <= num_tokens (rows past query_start[num_seqs] are neither read as queries nor written)
 *   query_start   int32 [num_seqs + 1], non-decreasing, query_start[0] = 0
 *   context_lens  int32 [num_seqs]; q_len <= context_len
 *   scale         finite and > 0 (else PKV_EINVAL)
 *   max_query_len / max_context_len  host upper bounds (size the work list)
 *   workspace     at least pkv_prefill_workspace_bytes(...), 256-B aligned
 * A query length above its context or the bounds sets PKV_DEVERR_CONTEXT and is
 * clamped (rows past the clamp are not written).  Launches a plan kernel and
 * the attention kernel on `stream`.  The attention kernel runs on the
 * tcgen05 tensor cores: tiles of 128 query rows (query token x head of the GQA
 * group), 64-key blocks, accumulators in tensor memory; two persistent CTAs
 * per SM, each holding 256 columns of tensor memory.
 */
pkv_status paged_attn_prefill(const void *q, const void *k_cache, const void *v_cache,
                              const int32_t *block_tables, int32_t max_blocks_per_seq,
                              const int32_t *context_lens, const int32_t *query_start, int32_t num_seqs,
                              int32_t num_tokens, int32_t num_q_heads, float scale, int32_t num_kv_heads,
                              void *out, pkv_pool pool, int32_t max_query_len, int32_t max_context_len,
                              void *workspace, size_t workspace_bytes, pkv_stream_t stream);

/*
 * FP8 KV cache -- the pool holds OCP FP8 E4M3 codes (1 sign, 4 exponent bits
 * with bias 7, 3 mantissa bits, no infinities, S.1111.111 NaN, largest finite
 * 448), one byte per element, same [num_blocks][num_kv_heads][block_size]
 * [head_dim] layout; half the bytes of bf16 per token.  The pages name FP8
 * mixed precision as a way to cut memory and raise throughput (ai-stack.site
 * "Nano-vLLM 原理", case study).  Each kv head has a static dequantisation
 * scale for K and one for V (fp32 device arrays [num_kv_heads], chosen by the
 * caller, e.g. from calibration): the value of a code c is e4m3(c) * scale.
 *
 * pkv_write_fp8: as pkv_write, storing for every element
 *   code = e4m3_rne_satfinite(fp32(x) * fp32(1 / scale[h]))
 * (IEEE round-to-nearest reciprocal and product; ties to the even code;
 * magnitudes beyond 448 saturate).  Codes are bit-exact with that rule.
 *
 * paged_attn_decode_fp8: as paged_attn_decode over an FP8 pool, reading
 * K = e4m3(code) * k_scale[h] and V = e4m3(code) * v_scale[h].  Supported at
 * head_dim 128 (else PKV_EUNSUPPORTED) for every GQA group <= 16: group 1
 * on CUDA cores, groups 2-16 on the tensor cores; the codes are multiplied
 * exactly as f16 with fp32 accumulation.  The workspace is the same as
 * paged_attn_decode's.
 */
pkv_status pkv_write_fp8(const void *k, const void *v, const int64_t *slot_mapping, int32_t num_tokens,
                         const float *k_scale, const float *v_scale, void *k_cache, void *v_cache, pkv_pool pool,
                         pkv_stream_t stream);
pkv_status paged_attn_decode_fp8(const void *q, const void *k_cache, const void *v_cache, const float *k_scale,
                                 const float *v_scale, const int32_t *block_tables, int32_t max_blocks_per_seq,
                                 const int32_t *context_lens, int32_t num_seqs, int32_t num_q_heads, float scale,
                                 int32_t num_kv_heads, void *out, pkv_pool pool, int32_t max_context_len,
                                 int32_t partition_tokens, void *workspace, size_t workspace_bytes,
                                 pkv_stream_t stream);

/*
 * Block manager on the device -- the bookkeeping of the pages' block manager
 * (wkbse.com section 3.1, "flexible memory management": blocks allocated only
 * as new tokens need them, the block table updated, blocks returned when a
 * sequence ends; "KV cache sharing": parallel samples map the same physical
 * blocks; intelliparadigm.com section 2.1, items 1-3 and the allocation
 * sketch: a free list popped on allocation, copy-on-write for shared
 * prefixes, a block free, allocated or shareable, LRU for block heat), so a
 * serving step needs no host round trip.
 *
 * Block states: free (on the free stack), allocated (refcount > 0), cached
 * (refcount 0 but still holding a prefix key: a prefix lookup can map it
 * again).  A block whose count reaches zero is cached if it holds a key and
 * free otherwise.  Allocation pops the free stack first; when it is empty it
 * evicts cached blocks, the least recently released first, dropping their
 * keys.  A prefix hit or a share on a cached block takes it off the eviction
 * order.
 *
 * State: one device buffer of pkv_bm_state_bytes(num_blocks), 256-B aligned,
 * owned by the caller (num_blocks <= 2^29), laid out as
 *   int32 [0] top, [1] error word (PKV_BM_ERR_* bits; the caller clears it),
 *         [2] cached blocks, [3] and [4] head and tail of the eviction order
 *   at 256:            int32 free_stack[num_blocks]  (free_stack[0 .. top) are free,
 *                      the next allocation pops free_stack[top - 1])
 *   at 256 + A:        int32 refcount[num_blocks]     (sequences mapping each block)
 *   at 256 + 2A..4A:   three int32 scratch arrays kept at their rest values
 *   at 256 + 5A:       uint64 block_hash[num_blocks]  (the prefix-cache key a block
 *                      holds, 0: none; dropped when the block is evicted)
 *   at 256 + 5A + H:   uint32 lru_pos[num_blocks]     (a cached block's position in the
 *                      eviction order; 0xffffffff for any other block)
 *   at 256 + 6A + H:   int32 ring[2 num_blocks]       (the eviction order: entry at
 *                      absolute position p is ring[p % (2 num_blocks)], live while
 *                      lru_pos of its block equals p; head .. tail in release order)
 *   at 256 + 6A + 2H:  int32 scratch[num_blocks]
 * with A = num_blocks * 4 and H = num_blocks * 8, each rounded up to 256.
 * Every call is one kernel on
 * `stream` (one CTA walking its list in order with block-wide scans), so its
 * results are exactly the sequential, request-order ones; device-side
 * failures set bits in the error word and leave the failing request (and,
 * for alloc and append, every later one) unserved.  All arrays are device
 * memory.  Calls on one state must be ordered (one stream).
 */
#define PKV_BM_ERR_NOSPACE 1u    /* too few free blocks, or no room in ids, for a request */
#define PKV_BM_ERR_RANGE 2u      /* a block id outside [0, num_blocks) */
#define PKV_BM_ERR_DOUBLEFREE 4u /* a block freed more often than referenced */
#define PKV_BM_ERR_TABLE 8u      /* a sequence outgrew its block-table row, or its context was outside it */

size_t pkv_bm_state_bytes(int32_t num_blocks);
/* All blocks free, popped 0, 1, 2, ... first; reference counts 0; no keys, none
 * cached; error word 0. */
pkv_status pkv_bm_init(void *state, int32_t num_blocks, pkv_stream_t stream);
/* Request r (of n) receives counts[r] blocks (reference count 1) at
 * ids[offsets[r] .. offsets[r+1]) (offsets: int32 [n+1]); requests are served
 * in order while free and cached blocks and the capacity of ids last. */
pkv_status pkv_bm_alloc(void *state, int32_t num_blocks, const int32_t *counts, int32_t n, int32_t *offsets,
                        int32_t *ids, int32_t capacity, pkv_stream_t stream);
/* Every listed block drops one reference, in list order; a block whose count
 * reaches zero at that point is cached (appended to the eviction order) if it
 * holds a prefix key, and otherwise pushed back on the free list. */
pkv_status pkv_bm_free(void *state, int32_t num_blocks, const int32_t *block_ids, int32_t n, pkv_stream_t stream);
/* Every listed block gains one reference (a new sequence maps it, e.g. a fork);
 * a cached block leaves the eviction order. */
pkv_status pkv_bm_share(void *state, int32_t num_blocks, const int32_t *block_ids, int32_t n, pkv_stream_t stream);
/*
 * One step's slots for num_new[b] new tokens of each sequence b < num_seqs, in
 * sequence order: (1) if the tokens go into a partly filled last block that
 * other sequences still map (reference count > 1), it is replaced by a fresh
 * private block and the pair (old, fresh) is appended to cow_pairs (int32
 * [num_seqs][2]; count in *num_cow_pairs) -- copy-on-write; of k sharers of one
 * such block appending in the same step, the first min(k, refs - 1) copy and
 * the last writes in place; (2) fresh blocks fill the table entries the new
 * tokens reach; (3) slot_mapping[off_b + t] = table[b][p / bs] * bs + p % bs
 * for p = context_lens[b] + t (off_b = the sum of num_new over earlier
 * sequences; int64 [slot_capacity]; entries past the capacity are not written
 * and set PKV_BM_ERR_NOSPACE), ready for pkv_write; (4) context_lens[b]
 * grows by num_new[b].  block_tables is int32 [num_seqs][max_blocks_per_seq],
 * updated in place.  Fresh blocks come from the free stack, then from the
 * cached blocks (least recently released first).  The first sequence that
 * finds too few blocks or outgrows its row, and every later one, is left
 * unchanged with slots -1.
 * Run pkv_copy_blocks_dev on the pairs before writing the new tokens.
 */
pkv_status pkv_bm_append_slots(void *state, int32_t num_blocks, int32_t *block_tables, int32_t max_blocks_per_seq,
                               int32_t *context_lens, const int32_t *num_new, int32_t num_seqs, int32_t block_size,
                               int64_t *slot_mapping, int64_t slot_capacity, int32_t *cow_pairs,
                               int32_t *num_cow_pairs, pkv_stream_t stream);
/*
 * Prefix caching (intelliparadigm.com section 3.1, --enable-prefix-caching:
 * prompt sharing; section 2.1's allocation sketch shares an existing block
 * whose prefix matches instead of allocating one).  Full prompt blocks are
 * keyed by FNV-1a 64 (offset basis 14695981039346656037, prime
 * 1099511628211, per byte xor then multiply) chained over the prefix:
 * d_i = FNV-1a of the block's block_size tokens as little-endian int32 bytes,
 * key_i = FNV-1a of le64(key_{i-1}) || le64(d_i), key_{-1} = 0, a key of 0
 * stored as 1.  The cache is a caller-owned device buffer of
 * pkv_prefix_cache_bytes(capacity) (capacity a power of two, 256-B aligned):
 * an open-addressing table of (key, block) pairs.  An entry counts while its
 * block still holds the key (block_hash): allocated, or cached and not yet
 * evicted.
 * tokens: int32 prompts concatenated, query_start: int32 [num_seqs + 1].
 *
 * pkv_prefix_lookup: for each sequence, the longest run of leading full
 *   prompt blocks with a valid holder -- leaving at least one prompt token to
 *   compute -- is written into its block-table row (int32 [num_seqs]
 *   [max_blocks_per_seq]) with one reference each (a cached holder leaves the
 *   eviction order); num_cached[s] (int32
 *   [num_seqs]) = the tokens covered.  Then pkv_bm_append_slots with
 *   context_lens = num_cached and num_new = prompt length - num_cached.
 * pkv_prefix_insert: after the prompt's K/V is written, in sequence order,
 *   every full prompt block whose key has no valid holder becomes its holder
 *   (the first sequence in order wins); a full table sets PKV_BM_ERR_NOSPACE.
 */
size_t pkv_prefix_cache_bytes(int32_t capacity);
pkv_status pkv_prefix_cache_init(void *cache, int32_t capacity, pkv_stream_t stream);
pkv_status pkv_prefix_lookup(void *state, int32_t num_blocks, void *cache, int32_t capacity, const int32_t *tokens,
                             const int32_t *query_start, int32_t num_seqs, int32_t block_size,
                             int32_t *block_tables, int32_t max_blocks_per_seq, int32_t *num_cached,
                             pkv_stream_t stream);
pkv_status pkv_prefix_insert(void *state, int32_t num_blocks, void *cache, int32_t capacity, const int32_t *tokens,
                             const int32_t *query_start, int32_t num_seqs, int32_t block_size,
                             const int32_t *block_tables, int32_t max_blocks_per_seq, pkv_stream_t stream);

/*
 * pkv_copy_blocks sourced from the device: copies the first *num_pairs of
 * cow_pairs (device int32 [max_pairs][2], as pkv_bm_append_slots leaves them)
 * without a host round trip.  The destinations must be fresh blocks that are
 * no pair's source (true of append's pairs); ids outside the pool set
 * PKV_DEVERR_BLOCK and are skipped.
 */
pkv_status pkv_copy_blocks_dev(const int32_t *cow_pairs, const int32_t *num_pairs, int32_t max_pairs, void *k_cache,
                               void *v_cache, pkv_pool pool, pkv_stream_t stream);

/*
 * pkv_get_device_error -- copies the current device's error word to
 * *code_out and clears it, ordered after the work already on `stream`, and
 * waits for it.  Returns PKV_EDEVICE when the word was non-zero.
 */
pkv_status pkv_get_device_error(int32_t *code_out, pkv_stream_t stream);

/*
 * pkv_selftest_bounded_wait -- diagnostic of this library (the pages have no
 * counterpart).  Runs, in one CTA, the bounded on-chip wait that the attention
 * kernel uses for its pipeline barriers, against barriers that nothing ever
 * arrives on: one warp gives up after limit_ns nanoseconds (0 < limit_ns <=
 * 1e9), sets PKV_DEVERR_TIMEOUT and the CTA's abort flag, and a second warp,
 * waiting with the kernel's 2 s limit, must then give up early.  Writes to
 * result_dev (device int32[3]): [0] first wait completed (expected 0),
 * [1] second wait completed (expected 0), [2] microseconds the second warp
 * waited.  No fault and no hang: both waits end by themselves.
 */
pkv_status pkv_selftest_bounded_wait(int64_t limit_ns, int32_t *result_dev, pkv_stream_t stream);

/* Static description of a status code. */
const char *pkv_status_string(pkv_status status);

/* ABI version: major * 10000 + minor * 100 + patch. */
int32_t pkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H_ */
