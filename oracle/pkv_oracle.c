/*
 * pkv_oracle.c -- plain, slow CPU oracle for the paged KV-cache decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this code.  It shares no source,
 * header, table or helper with the CUDA library, and neither side includes
 * or links the other.
 *
 * What it computes, following the pages on vLLM's PagedAttention:
 *   - KV cache split into fixed-size blocks of `bs` tokens, located through a
 *     per-sequence block table (wkbse.com "加速 LLM 推理：深入了解 vllm 引擎",
 *     section 3.1; intelliparadigm.com article 2012396, section 2.1).
 *   - token position -> (logical block = pos / bs, offset = pos % bs)
 *     (ruibaoantu.com article 3727998, section 1.1, the PagedAttention sketch).
 *   - the paged attention kernel reads the same K/V through the table and
 *     computes ordinary attention over it (wkbse.com section 3.1, third point
 *     of the list), i.e. softmax(q K^T * scale) V.
 *   - copy-on-write of a shared block (intelliparadigm.com section 2.1, item 2).
 *   - the block manager: a free list popped on allocation, blocks allocated as
 *     new tokens need them and the block table updated, blocks returned when
 *     a sequence ends, shared blocks counted by reference and copied before a
 *     sharer writes into them (wkbse.com section 3.1, "flexible memory
 *     management" and "KV cache sharing"; intelliparadigm.com section 2.1,
 *     items 1-2 and the block-allocation sketch).
 *   - prefix caching (intelliparadigm.com section 3.1, --enable-prefix-caching:
 *     prompt sharing; section 2.1's allocation sketch: a block whose prefix
 *     matches is shared instead of allocated): full prompt blocks are keyed
 *     by a chained FNV-1a 64-bit hash of their tokens and the key of the
 *     block before, and looked up before allocation.  A keyed block whose
 *     last sequence ends stays cached (section 2.1 item 1: a block is free,
 *     allocated or shareable) until allocation runs out of free blocks and
 *     evicts it, least recently released first (item 3: LRU keeps the block
 *     heat).
 *   - an FP8 KV cache (ai-stack.site "Nano-vLLM 原理", case study: FP8 mixed
 *     precision): the pool holds OCP E4M3 codes with a static scale per kv
 *     head for K and for V; a value is stored as the code nearest to
 *     fp32(x) * fp32(1 / scale) and read back as the code's value times scale.
 *   - swap of cold blocks to CPU memory and back, victims chosen least
 *     recently used first (intelliparadigm.com section 2.1, item 3; ai-stack.site
 *     "Nano-vLLM 原理", practice 5, preemption by swapping a request's KV cache).
 *
 * Pool layout (the library's ABI; the oracle reads it through pool_row()):
 *   cache[num_blocks][num_kv_heads][bs][d], bf16 bit patterns (uint16).
 * Floating point: every product and sum in double; bf16 inputs are widened
 * exactly (a bf16 is the top half of an IEEE binary32).
 *
 * Return codes: 0 ok, 1 bad argument, 2 index out of range.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* exact bf16 -> double */
static double bf16_to_f64(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* index of token row (block, head, offset) in a pool of layout
 * [num_blocks][num_kv_heads][bs][d] (units of elements) */
static size_t pool_row(int64_t block, int head, int offset, int num_kv_heads, int bs, int d) {
    return (((size_t)block * (size_t)num_kv_heads + (size_t)head) * (size_t)bs + (size_t)offset) * (size_t)d;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads used by later parallel regions (timing only; results do not depend
 * on it).  Returns the previous count. */
int oracle_set_num_threads(int n) {
    int prev = oracle_num_threads();
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
    return prev;
}

/*
 * Write: for every new token t with slot_mapping[t] >= 0, block = slot / bs,
 * offset = slot % bs, and for every kv head h the row
 * cache[block][h][offset][:] becomes k[t][h][:] (same for v).  Tokens are
 * applied in ascending t.  A negative slot marks padding and is skipped.
 */
int oracle_kv_write(uint16_t *k_cache, uint16_t *v_cache, const uint16_t *k, const uint16_t *v,
                    const int64_t *slot_mapping, int num_tokens, int num_blocks, int num_kv_heads,
                    int bs, int d) {
    if (num_tokens < 0 || num_blocks <= 0 || num_kv_heads <= 0 || bs <= 0 || d <= 0) return 1;
    for (int t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= (int64_t)num_blocks * bs) return 2;
        int64_t block = slot / bs;
        int offset = (int)(slot % bs);
        for (int h = 0; h < num_kv_heads; ++h) {
            size_t dst = pool_row(block, h, offset, num_kv_heads, bs, d);
            size_t src = ((size_t)t * num_kv_heads + h) * (size_t)d;
            for (int i = 0; i < d; ++i) {
                k_cache[dst + i] = k[src + i];
                v_cache[dst + i] = v[src + i];
            }
        }
    }
    return 0;
}

/*
 * Copy-on-write block copy: every pair (src, dst) makes block dst of both
 * caches (all heads, all offsets) equal to block src.  The pairs act as if
 * simultaneous: every source block is read before any destination is
 * written.
 */
int oracle_copy_blocks(uint16_t *k_cache, uint16_t *v_cache, const int32_t *pairs, int num_pairs,
                       int num_blocks, int num_kv_heads, int bs, int d) {
    if (num_pairs < 0 || num_blocks <= 0) return 1;
    size_t block_elems = (size_t)num_kv_heads * bs * d;
    for (int p = 0; p < num_pairs; ++p) {
        int32_t s = pairs[2 * p], t = pairs[2 * p + 1];
        if (s < 0 || s >= num_blocks || t < 0 || t >= num_blocks) return 2;
    }
    if (num_pairs == 0) return 0;
    uint16_t *snap_k = (uint16_t *)malloc(sizeof(uint16_t) * block_elems * num_pairs);
    uint16_t *snap_v = (uint16_t *)malloc(sizeof(uint16_t) * block_elems * num_pairs);
    if (!snap_k || !snap_v) { free(snap_k); free(snap_v); return 1; }
    for (int p = 0; p < num_pairs; ++p) {
        size_t src = (size_t)pairs[2 * p] * block_elems;
        memcpy(snap_k + (size_t)p * block_elems, k_cache + src, sizeof(uint16_t) * block_elems);
        memcpy(snap_v + (size_t)p * block_elems, v_cache + src, sizeof(uint16_t) * block_elems);
    }
    for (int p = 0; p < num_pairs; ++p) {
        size_t dst = (size_t)pairs[2 * p + 1] * block_elems;
        memcpy(k_cache + dst, snap_k + (size_t)p * block_elems, sizeof(uint16_t) * block_elems);
        memcpy(v_cache + dst, snap_v + (size_t)p * block_elems, sizeof(uint16_t) * block_elems);
    }
    free(snap_k);
    free(snap_v);
    return 0;
}

/*
 * Attention of one (sequence s, query head hq) over the token range
 * [t_begin, t_end) of that sequence, returning the unnormalised pieces:
 *   z_i   = scale * sum_c q[c] * K_i[c]                 (i in range)
 *   m     = max_i z_i
 *   l     = sum_i exp(z_i - m)
 *   acc_c = sum_i exp(z_i - m) * V_i[c]
 * where K_i, V_i are the rows of token i of the sequence, found through the
 * block table: physical block = table[i / bs], offset = i % bs, kv head
 * hkv = hq / (Hq / Hkv).  An empty range gives m = -inf, l = 0, acc = 0.
 */
static int attend_range(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                        const int32_t *table, int num_blocks, int Hq, int Hkv, int d, int bs,
                        int hq, int t_begin, int t_end, double scale, double *m_out, double *l_out,
                        double *acc) {
    int g = Hq / Hkv;
    int hkv = hq / g;
    for (int c = 0; c < d; ++c) acc[c] = 0.0;
    if (t_end <= t_begin) {
        *m_out = -INFINITY;
        *l_out = 0.0;
        return 0;
    }
    int n = t_end - t_begin;
    double *z = (double *)malloc(sizeof(double) * (size_t)n);
    if (!z) return 1;
    double m = -INFINITY;
    for (int i = t_begin; i < t_end; ++i) {
        int32_t block = table[i / bs];
        if (block < 0 || block >= num_blocks) { free(z); return 2; }
        const uint16_t *krow = k_cache + pool_row(block, hkv, i % bs, Hkv, bs, d);
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += bf16_to_f64(q[c]) * bf16_to_f64(krow[c]);
        z[i - t_begin] = scale * dot;
        if (z[i - t_begin] > m) m = z[i - t_begin];
    }
    double l = 0.0;
    for (int i = t_begin; i < t_end; ++i) {
        int32_t block = table[i / bs];
        const uint16_t *vrow = v_cache + pool_row(block, hkv, i % bs, Hkv, bs, d);
        double w = exp(z[i - t_begin] - m);
        l += w;
        for (int c = 0; c < d; ++c) acc[c] += w * bf16_to_f64(vrow[c]);
    }
    free(z);
    *m_out = m;
    *l_out = l;
    return 0;
}

/*
 * Decode attention for a batch: out[s][hq][:] = softmax_i(z_i) . V_i over the
 * context_lens[s] tokens of sequence s (z_i as in attend_range).  A sequence
 * with context length 0 gets a zero output.  q is bf16 [B][Hq][d], tables are
 * int32 [B][max_blocks_per_seq], out is double [B][Hq][d].
 * (s, hq) pairs are independent and are spread over OpenMP threads; the
 * arithmetic of each pair is the sequential sum above.
 */
int oracle_paged_attention(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                           const int32_t *block_tables, int max_blocks_per_seq,
                           const int32_t *context_lens, int B, int Hq, int Hkv, int d, int bs,
                           int num_blocks, double scale, double *out) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || bs <= 0) return 1;
    for (int s = 0; s < B; ++s) {
        if (context_lens[s] < 0) return 1;
        if ((int64_t)context_lens[s] > (int64_t)max_blocks_per_seq * bs) return 2;
    }
    int status = 0;
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int s = 0; s < B; ++s) {
        for (int hq = 0; hq < Hq; ++hq) {
            double *o = out + ((size_t)s * Hq + hq) * (size_t)d;
            double *acc = (double *)malloc(sizeof(double) * (size_t)d);
            double m, l;
            int rc = acc ? attend_range(q + ((size_t)s * Hq + hq) * (size_t)d, k_cache, v_cache,
                                        block_tables + (size_t)s * max_blocks_per_seq, num_blocks,
                                        Hq, Hkv, d, bs, hq, 0, context_lens[s], scale, &m, &l, acc)
                         : 1;
            if (rc) {
#pragma omp atomic write
                status = rc;
            } else {
                for (int c = 0; c < d; ++c) o[c] = (l > 0.0) ? acc[c] / l : 0.0;
            }
            free(acc);
        }
    }
    return status;
}

/*
 * Split-K pieces: for (s, hq) and token range [t_begin, t_end) return m, l and
 * the unnormalised acc[d] of attend_range.
 */
int oracle_attention_partial(const uint16_t *q_row, const uint16_t *k_cache, const uint16_t *v_cache,
                             const int32_t *table, int num_blocks, int Hq, int Hkv, int d, int bs,
                             int hq, int t_begin, int t_end, double scale, double *m, double *l,
                             double *acc) {
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || t_begin < 0) return 1;
    return attend_range(q_row, k_cache, v_cache, table, num_blocks, Hq, Hkv, d, bs, hq, t_begin,
                        t_end, scale, m, l, acc);
}

/*
 * Log-sum-exp merge of P partial results (m_p, l_p, acc_p[d]) of disjoint
 * token ranges that together cover a context:
 *   M = max_p m_p,  L = sum_p l_p e^{m_p - M},  out = sum_p acc_p e^{m_p - M} / L.
 * Empty pieces (m = -inf) contribute nothing.  L = 0 gives a zero output.
 */
int oracle_lse_merge(const double *m, const double *l, const double *acc, int P, int d, double *out) {
    if (P < 0 || d <= 0) return 1;
    double M = -INFINITY;
    for (int p = 0; p < P; ++p) if (m[p] > M) M = m[p];
    double L = 0.0;
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    if (M == -INFINITY) return 0;
    for (int p = 0; p < P; ++p) {
        if (m[p] == -INFINITY) continue;
        double w = exp(m[p] - M);
        L += l[p] * w;
        for (int c = 0; c < d; ++c) out[c] += acc[(size_t)p * d + c] * w;
    }
    for (int c = 0; c < d; ++c) out[c] = (L > 0.0) ? out[c] / L : 0.0;
    return 0;
}

/*
 * Chunked prefill (multi-token query, wkbse.com section 3.1 attention read
 * through the block table, with the causal rule of autoregressive decoding:
 * a token sees itself and the tokens before it).  Sequence s holds
 * context_lens[s] tokens in the cache, the last q_len = query_start[s+1] -
 * query_start[s] of which are the new chunk; query row i of the chunk is at
 * position pos = context_lens[s] - q_len + i and attends to positions
 * [0, pos].  q and out are [T][Hq][d] with T = query_start[B]; out in double.
 */
int oracle_paged_prefill(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                         const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                         const int32_t *query_start, int B, int Hq, int Hkv, int d, int bs, int num_blocks,
                         double scale, double *out) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || bs <= 0) return 1;
    for (int s = 0; s < B; ++s) {
        int q_len = query_start[s + 1] - query_start[s];
        if (q_len < 0 || q_len > context_lens[s]) return 1;
        if ((int64_t)context_lens[s] > (int64_t)max_blocks_per_seq * bs) return 2;
    }
    int T = query_start[B];
    int status = 0;
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int t = 0; t < T; ++t) {
        for (int hq = 0; hq < Hq; ++hq) {
            int s = 0;
            while (query_start[s + 1] <= t) ++s;
            int q_len = query_start[s + 1] - query_start[s];
            int pos = context_lens[s] - q_len + (t - query_start[s]);
            double *o = out + ((size_t)t * Hq + hq) * (size_t)d;
            double *acc = (double *)malloc(sizeof(double) * (size_t)d);
            double m, l;
            int rc = acc ? attend_range(q + ((size_t)t * Hq + hq) * (size_t)d, k_cache, v_cache,
                                        block_tables + (size_t)s * max_blocks_per_seq, num_blocks, Hq, Hkv, d,
                                        bs, hq, 0, pos + 1, scale, &m, &l, acc)
                         : 1;
            if (rc) {
#pragma omp atomic write
                status = rc;
            } else {
                for (int c = 0; c < d; ++c) o[c] = (l > 0.0) ? acc[c] / l : 0.0;
            }
            free(acc);
        }
    }
    return status;
}

/*
 * Swap-out: host_k[i] and host_v[i] (each num_kv_heads * bs * d elements, all
 * heads of one block) become copies of block ids[i] of the two caches, for
 * i < n.  The caches are not changed; an id may repeat.
 */
int oracle_swap_out(const uint16_t *k_cache, const uint16_t *v_cache, const int32_t *ids, int n, int num_blocks,
                    int num_kv_heads, int bs, int d, uint16_t *host_k, uint16_t *host_v) {
    if (n < 0 || num_blocks <= 0) return 1;
    size_t block_elems = (size_t)num_kv_heads * bs * d;
    for (int i = 0; i < n; ++i)
        if (ids[i] < 0 || ids[i] >= num_blocks) return 2;
    for (int i = 0; i < n; ++i) {
        for (size_t e = 0; e < block_elems; ++e) {
            host_k[(size_t)i * block_elems + e] = k_cache[(size_t)ids[i] * block_elems + e];
            host_v[(size_t)i * block_elems + e] = v_cache[(size_t)ids[i] * block_elems + e];
        }
    }
    return 0;
}

/*
 * Swap-in: block ids[i] of the two caches becomes host_k[i] / host_v[i], for
 * i < n.  Ids must be distinct (two copies into one block would leave it
 * undefined): 3 otherwise.
 */
int oracle_swap_in(const uint16_t *host_k, const uint16_t *host_v, const int32_t *ids, int n, int num_blocks,
                   int num_kv_heads, int bs, int d, uint16_t *k_cache, uint16_t *v_cache) {
    if (n < 0 || num_blocks <= 0) return 1;
    size_t block_elems = (size_t)num_kv_heads * bs * d;
    for (int i = 0; i < n; ++i)
        if (ids[i] < 0 || ids[i] >= num_blocks) return 2;
    for (int i = 0; i < n; ++i)
        for (int j = i + 1; j < n; ++j)
            if (ids[i] == ids[j]) return 3;
    for (int i = 0; i < n; ++i) {
        for (size_t e = 0; e < block_elems; ++e) {
            k_cache[(size_t)ids[i] * block_elems + e] = host_k[(size_t)i * block_elems + e];
            v_cache[(size_t)ids[i] * block_elems + e] = host_v[(size_t)i * block_elems + e];
        }
    }
    return 0;
}

/*
 * LRU victim choice: among the blocks with evictable[b] != 0, the k with the
 * oldest last_use[b] (smallest value; equal values by lower block id), in that
 * order, written to victims[0 .. min(k, #evictable)).  Returns the count
 * through *count.  Plain repeated selection of the minimum.
 */
int oracle_lru_victims(const int64_t *last_use, const uint8_t *evictable, int num_blocks, int k, int32_t *victims,
                       int *count) {
    if (num_blocks < 0 || k < 0) return 1;
    uint8_t *taken = (uint8_t *)calloc((size_t)num_blocks + 1, 1);
    if (!taken) return 1;
    int c = 0;
    while (c < k) {
        int best = -1;
        for (int b = 0; b < num_blocks; ++b) {
            if (!evictable[b] || taken[b]) continue;
            if (best < 0 || last_use[b] < last_use[best]) best = b;
        }
        if (best < 0) break;
        taken[best] = 1;
        victims[c++] = best;
    }
    free(taken);
    *count = c;
    return 0;
}

/* ------------------------------------------------------------------------
 * Block manager.  State: free_stack[0 .. *top) holds the free block ids; an
 * allocation pops free_stack[*top - 1]; refcount[b] counts the sequences that
 * map block b.  err collects the bits BM_ERR_* below.  Everything is a plain
 * sequential loop in request order.
 * ------------------------------------------------------------------------ */
#define BM_ERR_NOSPACE 1u    /* a request found too few free blocks (or output room) */
#define BM_ERR_RANGE 2u      /* a block id outside the pool */
#define BM_ERR_DOUBLEFREE 4u /* a block freed more often than it was referenced */
#define BM_ERR_TABLE 8u      /* a sequence outgrew its block-table row */

/* Block states (intelliparadigm.com section 2.1, item 1):
 *   free       refcount 0, on the free stack, no key;
 *   allocated  refcount > 0 (it may hold a prefix key);
 *   cached     refcount 0 but still holding a prefix key: shareable again by
 *              a prefix lookup, evictable by allocation.  lru_stamp[b] is the
 *              value of the release clock when its count reached zero; every
 *              other block has lru_stamp -1.
 * Allocation takes the free stack first; when it is empty, the cached block
 * with the smallest stamp (the least recently released, item 3) is evicted:
 * its key is dropped and it is handed out. */
int oracle_bm_init(int32_t *free_stack, int32_t *top, int32_t *refcount, uint64_t *block_hash, int64_t *lru_stamp,
                   int64_t *clock, int num_blocks) {
    if (num_blocks <= 0) return 1;
    for (int i = 0; i < num_blocks; ++i) {
        free_stack[i] = num_blocks - 1 - i; /* block 0 is popped first */
        refcount[i] = 0;
        block_hash[i] = 0;
        lru_stamp[i] = -1;
    }
    *top = num_blocks;
    *clock = 0;
    return 0;
}

/* Blocks allocation can hand out: the free stack and the cached blocks. */
static int bm_available(const int32_t *top, const int64_t *lru_stamp, int num_blocks) {
    int n = *top;
    for (int b = 0; b < num_blocks; ++b)
        if (lru_stamp[b] >= 0) ++n;
    return n;
}

static int32_t bm_pop(int32_t *free_stack, int32_t *top, int32_t *refcount, uint64_t *block_hash, int64_t *lru_stamp,
                      int num_blocks) {
    int32_t b = -1;
    if (*top > 0) {
        b = free_stack[--*top];
    } else {
        for (int c = 0; c < num_blocks; ++c) /* the least recently released cached block */
            if (lru_stamp[c] >= 0 && (b < 0 || lru_stamp[c] < lru_stamp[b])) b = c;
        block_hash[b] = 0; /* evicted: its content no longer backs a prefix */
        lru_stamp[b] = -1;
    }
    refcount[b] = 1;
    return b;
}

/* Request r receives counts[r] blocks, written to ids[offsets[r] .. offsets[r+1]).
 * Requests are served in order while the free and cached blocks and the
 * output room last; the first one that does not fit, and every later one,
 * receives none. */
int oracle_bm_alloc(int32_t *free_stack, int32_t *top, int32_t *refcount, uint64_t *block_hash, int64_t *lru_stamp,
                    int64_t *clock, int num_blocks, const int32_t *counts, int n, int32_t *offsets, int32_t *ids,
                    int capacity, uint32_t *err) {
    (void)clock;
    if (num_blocks <= 0 || n < 0 || capacity < 0) return 1;
    int failed = 0;
    offsets[0] = 0;
    for (int r = 0; r < n; ++r) {
        int c = counts[r] < 0 ? 0 : counts[r];
        if (!failed && c <= bm_available(top, lru_stamp, num_blocks) && offsets[r] + c <= capacity) {
            for (int k = 0; k < c; ++k)
                ids[offsets[r] + k] = bm_pop(free_stack, top, refcount, block_hash, lru_stamp, num_blocks);
            offsets[r + 1] = offsets[r] + c;
        } else {
            if (c > 0 || failed) { failed = 1; *err |= BM_ERR_NOSPACE; }
            offsets[r + 1] = offsets[r];
        }
    }
    return 0;
}

/* Each listed id drops one reference, in list order.  A block whose count
 * reaches zero becomes cached (stamped with the release clock, which then
 * advances) if it holds a prefix key, and is otherwise pushed back onto the
 * free stack, at that moment. */
int oracle_bm_free(int32_t *free_stack, int32_t *top, int32_t *refcount, uint64_t *block_hash, int64_t *lru_stamp,
                   int64_t *clock, int num_blocks, const int32_t *ids, int n, uint32_t *err) {
    if (num_blocks <= 0 || n < 0) return 1;
    for (int i = 0; i < n; ++i) {
        int32_t b = ids[i];
        if (b < 0 || b >= num_blocks) { *err |= BM_ERR_RANGE; continue; }
        if (refcount[b] <= 0) { *err |= BM_ERR_DOUBLEFREE; continue; }
        if (--refcount[b] == 0) {
            if (block_hash[b] != 0) lru_stamp[b] = (*clock)++;
            else free_stack[(*top)++] = b;
        }
    }
    return 0;
}

/* Each listed id gains one reference (a new sequence maps the block); a cached
 * block mapped again is no longer evictable. */
int oracle_bm_share(int32_t *refcount, int64_t *lru_stamp, int num_blocks, const int32_t *ids, int n, uint32_t *err) {
    if (num_blocks <= 0 || n < 0) return 1;
    for (int i = 0; i < n; ++i) {
        if (ids[i] < 0 || ids[i] >= num_blocks) { *err |= BM_ERR_RANGE; continue; }
        if (refcount[ids[i]] == 0) lru_stamp[ids[i]] = -1;
        refcount[ids[i]] += 1;
    }
    return 0;
}

/* One step's slots for num_new[b] new tokens of every sequence b, in order:
 *   - if the tokens go into a partly filled last block that other sequences
 *     still map (refcount > 1), that block is first replaced by a private
 *     copy: a new block, the pair (old, new) appended to pairs, one reference
 *     of the old block dropped (copy-on-write);
 *   - blocks for the logical indices the new tokens reach beyond the table
 *     are popped in logical order (free stack first, then cached blocks, the
 *     least recently released first);
 *   - slot_mapping[off_b + t] = table[b][p / bs] * bs + p % bs for position
 *     p = context_lens[b] + t, off_b the sum of num_new over earlier b;
 *   - context_lens[b] grows by num_new[b].
 * A sequence that finds too few blocks or outgrows its table row, and every
 * later one, is left unchanged with slots -1 (padding). */
int oracle_bm_append_slots(int32_t *free_stack, int32_t *top, int32_t *refcount, uint64_t *block_hash,
                           int64_t *lru_stamp, int64_t *clock, int num_blocks, int32_t *block_tables, int mbs,
                           int32_t *context_lens, const int32_t *num_new, int B, int bs, int64_t *slot_mapping,
                           int32_t *pairs, int32_t *num_pairs, uint32_t *err) {
    (void)clock;
    if (num_blocks <= 0 || B < 0 || bs <= 0 || mbs <= 0) return 1;
    int failed = 0;
    int64_t off = 0;
    *num_pairs = 0;
    for (int b = 0; b < B; ++b) {
        int n = num_new[b] < 0 ? 0 : num_new[b];
        int32_t pos0 = context_lens[b];
        int32_t *row = block_tables + (size_t)b * mbs;
        if (pos0 < 0 || pos0 > mbs * bs) { /* the context is not inside its own table row */
            if (!failed) *err |= BM_ERR_TABLE;
            failed = 1;
            for (int t = 0; t < n; ++t) slot_mapping[off + t] = -1;
            off += n;
            continue;
        }
        int first_new = (pos0 + bs - 1) / bs;              /* first logical block not yet mapped */
        int last = n > 0 ? (pos0 + n - 1) / bs : first_new - 1;
        int need_new = last >= first_new ? last - first_new + 1 : 0;
        int cow = 0;
        if (n > 0 && pos0 % bs != 0) {
            int32_t cur = row[pos0 / bs];
            if (cur < 0 || cur >= num_blocks) { *err |= BM_ERR_RANGE; failed = 1; }
            else if (refcount[cur] > 1) cow = 1;
        }
        if (!failed && n > 0 && last >= mbs) { *err |= BM_ERR_TABLE; failed = 1; }
        if (!failed && need_new + cow > bm_available(top, lru_stamp, num_blocks)) { *err |= BM_ERR_NOSPACE; failed = 1; }
        if (failed) {
            for (int t = 0; t < n; ++t) slot_mapping[off + t] = -1;
            off += n;
            continue;
        }
        if (cow) {
            int32_t old = row[pos0 / bs];
            int32_t fresh = bm_pop(free_stack, top, refcount, block_hash, lru_stamp, num_blocks);
            refcount[old] -= 1;
            row[pos0 / bs] = fresh;
            pairs[2 * *num_pairs] = old;
            pairs[2 * *num_pairs + 1] = fresh;
            *num_pairs += 1;
        }
        for (int L = first_new; L <= last; ++L)
            row[L] = bm_pop(free_stack, top, refcount, block_hash, lru_stamp, num_blocks);
        for (int t = 0; t < n; ++t) {
            int32_t p = pos0 + t;
            slot_mapping[off + t] = (int64_t)row[p / bs] * bs + p % bs;
        }
        context_lens[b] = pos0 + n;
        off += n;
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * FP8 E4M3 (the OCP "E4M3FN" encoding): 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits; exponent field 0 holds the subnormals m/8 * 2^-6;
 * no infinities; S.1111.111 is NaN; the largest finite value is 448.
 * ------------------------------------------------------------------------ */
double oracle_e4m3_decode(uint8_t c) {
    int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sgn ? -v : v;
}

/* The code nearest to x (ties to the even code, i.e. the even mantissa), with
 * magnitudes beyond 448 saturating to +-448 and NaN to 0x7F. */
uint8_t oracle_e4m3_encode(double x) {
    if (x != x) return 0x7F;
    uint8_t sgn = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= 448.0) return (uint8_t)(sgn | 0x7E);
    int best = 0;
    double best_err = a;
    for (int c = 1; c <= 0x7E; ++c) {
        double err = fabs(oracle_e4m3_decode((uint8_t)c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0)) { best = c; best_err = err; }
    }
    return (uint8_t)(sgn | best);
}

int oracle_e4m3_encode_array(const double *x, int n, uint8_t *codes) {
    for (int i = 0; i < n; ++i) codes[i] = oracle_e4m3_encode(x[i]);
    return 0;
}

/* FP8 write: like oracle_kv_write, but row elements become e4m3 codes of
 * fp32(x) * fp32(1 / scale[h]) (both products single-precision, rounded to
 * nearest), with per-kv-head scales for K and V. */
int oracle_kv_write_fp8(uint8_t *k_cache, uint8_t *v_cache, const uint16_t *k, const uint16_t *v,
                        const int64_t *slot_mapping, const float *k_scale, const float *v_scale, int num_tokens,
                        int num_blocks, int num_kv_heads, int bs, int d) {
    if (num_tokens < 0 || num_blocks <= 0 || num_kv_heads <= 0 || bs <= 0 || d <= 0) return 1;
    for (int t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= (int64_t)num_blocks * bs) return 2;
        int64_t block = slot / bs;
        int offset = (int)(slot % bs);
        for (int h = 0; h < num_kv_heads; ++h) {
            float inv_k = 1.0f / k_scale[h], inv_v = 1.0f / v_scale[h];
            size_t dst = pool_row(block, h, offset, num_kv_heads, bs, d);
            size_t src = ((size_t)t * num_kv_heads + h) * (size_t)d;
            for (int c = 0; c < d; ++c) {
                float xk = (float)bf16_to_f64(k[src + c]) * inv_k;
                float xv = (float)bf16_to_f64(v[src + c]) * inv_v;
                k_cache[dst + c] = oracle_e4m3_encode((double)xk);
                v_cache[dst + c] = oracle_e4m3_encode((double)xv);
            }
        }
    }
    return 0;
}

/* FP8 decode attention: the paged attention of oracle_paged_attention with
 * K = e4m3(code) * k_scale[hkv] and V = e4m3(code) * v_scale[hkv], in double. */
int oracle_paged_attention_fp8(const uint16_t *q, const uint8_t *k_cache, const uint8_t *v_cache,
                               const float *k_scale, const float *v_scale, const int32_t *block_tables,
                               int max_blocks_per_seq, const int32_t *context_lens, int B, int Hq, int Hkv, int d,
                               int bs, int num_blocks, double scale, double *out) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || bs <= 0) return 1;
    for (int s = 0; s < B; ++s) {
        if (context_lens[s] < 0) return 1;
        if ((int64_t)context_lens[s] > (int64_t)max_blocks_per_seq * bs) return 2;
    }
    int g = Hq / Hkv, status = 0;
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int s = 0; s < B; ++s) {
        for (int hq = 0; hq < Hq; ++hq) {
            int hkv = hq / g, n = context_lens[s];
            double *o = out + ((size_t)s * Hq + hq) * (size_t)d;
            double *z = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
            if (!z) {
#pragma omp atomic write
                status = 1;
                continue;
            }
            const uint16_t *qr = q + ((size_t)s * Hq + hq) * (size_t)d;
            double m = -INFINITY;
            int bad = 0;
            for (int i = 0; i < n; ++i) {
                int32_t block = block_tables[(size_t)s * max_blocks_per_seq + i / bs];
                if (block < 0 || block >= num_blocks) { bad = 1; break; }
                const uint8_t *kr = k_cache + pool_row(block, hkv, i % bs, Hkv, bs, d);
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += bf16_to_f64(qr[c]) * (oracle_e4m3_decode(kr[c]) * k_scale[hkv]);
                z[i] = scale * dot;
                if (z[i] > m) m = z[i];
            }
            if (bad) {
#pragma omp atomic write
                status = 2;
                free(z);
                continue;
            }
            double l = 0.0;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (int i = 0; i < n; ++i) {
                int32_t block = block_tables[(size_t)s * max_blocks_per_seq + i / bs];
                const uint8_t *vr = v_cache + pool_row(block, hkv, i % bs, Hkv, bs, d);
                double w = exp(z[i] - m);
                l += w;
                for (int c = 0; c < d; ++c) o[c] += w * (oracle_e4m3_decode(vr[c]) * v_scale[hkv]);
            }
            for (int c = 0; c < d; ++c) o[c] = (l > 0.0) ? o[c] / l : 0.0;
            free(z);
        }
    }
    return status;
}

/* ------------------------------------------------------------------------
 * Prefix caching.  FNV-1a 64-bit (Fowler-Noll-Vo, "1a" order: xor the byte,
 * then multiply): offset basis 14695981039346656037, prime 1099511628211.
 * Block i of a prompt has digest d_i = FNV-1a over its bs tokens as
 * little-endian int32 bytes and key k_i = FNV-1a over the 16 bytes
 * le64(k_{i-1}) || le64(d_i) (k_{-1} = 0); a key of 0 is stored as 1 (0 marks
 * an empty slot).  The cache maps keys to blocks; a mapping counts only while
 * the block still holds that key (block_hash[b] == key): allocated, or cached
 * and not yet evicted.
 * ------------------------------------------------------------------------ */
static uint64_t fnv1a(uint64_t h, const uint8_t *p, size_t n) {
    for (size_t i = 0; i < n; ++i) {
        h ^= p[i];
        h *= 1099511628211ull;
    }
    return h;
}

static uint64_t block_key(uint64_t prev, const int32_t *tokens, int bs) {
    uint64_t d = 14695981039346656037ull;
    for (int t = 0; t < bs; ++t) {
        uint8_t b[4] = {(uint8_t)tokens[t], (uint8_t)(tokens[t] >> 8), (uint8_t)(tokens[t] >> 16),
                        (uint8_t)(tokens[t] >> 24)};
        d = fnv1a(d, b, 4);
    }
    uint8_t buf[16];
    for (int i = 0; i < 8; ++i) {
        buf[i] = (uint8_t)(prev >> (8 * i));
        buf[8 + i] = (uint8_t)(d >> (8 * i));
    }
    uint64_t k = fnv1a(14695981039346656037ull, buf, 16);
    return k ? k : 1;
}

uint64_t oracle_fnv1a64(const uint8_t *bytes, int n) { return fnv1a(14695981039346656037ull, bytes, (size_t)n); }

int oracle_prefix_keys(const int32_t *tokens, int n_tokens, int bs, uint64_t *keys) {
    uint64_t prev = 0;
    for (int i = 0; i < n_tokens / bs; ++i) {
        prev = block_key(prev, tokens + (size_t)i * bs, bs);
        keys[i] = prev;
    }
    return 0;
}

/* The cache itself: parallel arrays of cap (key, block) pairs, cap a power of
 * two; the oracle searches it linearly (a plain map, no probing). */
static int cache_find(const uint64_t *keys, const int32_t *vals, int cap, uint64_t key) {
    for (int i = 0; i < cap; ++i)
        if (keys[i] == key) return vals[i];
    return -1;
}

static int valid_holder(int32_t b, uint64_t key, const uint64_t *block_hash, int nb) {
    return b >= 0 && b < nb && block_hash[b] == key;
}

/* Lookup, in sequence order: the longest run of leading full prompt blocks of
 * sequence s whose keys have a valid holder -- leaving at least one prompt
 * token uncached -- is mapped into its table row (one reference each; a
 * cached holder is taken off the eviction order); num_cached[s] = the tokens
 * covered. */
int oracle_prefix_lookup(int32_t *refcount, int64_t *lru_stamp, const uint64_t *block_hash, int num_blocks,
                         const uint64_t *ckeys, const int32_t *cvals, int cap, const int32_t *tokens,
                         const int32_t *query_start, int B, int bs, int32_t *block_tables, int mbs,
                         int32_t *num_cached) {
    if (num_blocks <= 0 || B < 0 || bs <= 0 || mbs <= 0) return 1;
    for (int s = 0; s < B; ++s) {
        int n = query_start[s + 1] - query_start[s];
        int look = n > 0 ? (n - 1) / bs : 0;
        if (look > mbs) look = mbs;
        uint64_t prev = 0;
        int hits = 0;
        for (int i = 0; i < look; ++i) {
            uint64_t key = block_key(prev, tokens + query_start[s] + (size_t)i * bs, bs);
            prev = key;
            int32_t b = cache_find(ckeys, cvals, cap, key);
            if (!valid_holder(b, key, block_hash, num_blocks)) break;
            block_tables[(size_t)s * mbs + i] = b;
            if (refcount[b] == 0) lru_stamp[b] = -1;
            refcount[b] += 1;
            ++hits;
        }
        num_cached[s] = hits * bs;
    }
    return 0;
}

/* Insert, in sequence order, after the prompt's blocks hold its K/V: every full
 * prompt block i of sequence s (block id table[s][i]) whose key has no valid
 * holder becomes its holder (the first sequence in order wins); a block that
 * already holds its key is left as it is. */
int oracle_prefix_insert(uint64_t *block_hash, int num_blocks, uint64_t *ckeys,
                         int32_t *cvals, int cap, const int32_t *tokens, const int32_t *query_start, int B, int bs,
                         const int32_t *block_tables, int mbs, uint32_t *err) {
    if (num_blocks <= 0 || B < 0 || bs <= 0 || mbs <= 0) return 1;
    for (int s = 0; s < B; ++s) {
        int n = query_start[s + 1] - query_start[s];
        int full = n / bs;
        if (full > mbs) full = mbs;
        uint64_t prev = 0;
        for (int i = 0; i < full; ++i) {
            uint64_t key = block_key(prev, tokens + query_start[s] + (size_t)i * bs, bs);
            prev = key;
            int32_t b = block_tables[(size_t)s * mbs + i];
            if (b < 0 || b >= num_blocks) { *err |= BM_ERR_RANGE; break; }
            if (block_hash[b] == key) continue;
            int slot = -1;
            for (int j = 0; j < cap; ++j)
                if (ckeys[j] == key) { slot = j; break; }
            if (slot >= 0 && valid_holder(cvals[slot], key, block_hash, num_blocks)) continue;
            if (slot < 0) {
                for (int j = 0; j < cap; ++j)
                    if (ckeys[j] == 0) { slot = j; break; }
                if (slot < 0) { *err |= BM_ERR_NOSPACE; continue; }
                ckeys[slot] = key;
            }
            cvals[slot] = b;
            block_hash[b] = key;
        }
    }
    return 0;
}
