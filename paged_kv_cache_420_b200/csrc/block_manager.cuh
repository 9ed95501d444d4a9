// block_manager.cuh -- the block manager's per-step bookkeeping on the device.
//
// The pages' block manager (wkbse.com "加速 LLM 推理：深入了解 vllm 引擎",
// section 3.1, "flexible memory management" and "KV cache sharing";
// intelliparadigm.com article 2012396, section 2.1, items 1-2 and the block
// allocation sketch): a free list popped on allocation, blocks allocated only
// as new tokens need them with the block table updated, blocks returned when a
// sequence ends, shared blocks counted by reference and copied before a sharer
// writes into them.
//
// State (one caller-owned device buffer, layout in pkv.h): the free stack
// (free_stack[0 .. top) free, the next allocation pops free_stack[top - 1]),
// reference counts, an error word, and per-block scratch kept at its rest
// value between calls.  Every kernel is one CTA of 1024 threads walking its
// items in chunks of 1024, in order, with block-wide scans: results are the
// sequential (request-order) ones, bit for bit, without host round trips.
//
// Cached blocks (intelliparadigm.com section 2.1, item 1: a block is free,
// allocated or shareable; item 3: LRU keeps the block heat): a block that
// holds a prefix key keeps it when its count reaches zero and waits in the
// eviction order instead of on the free stack.  The order is a ring of
// 2 * num_blocks entries addressed by absolute position (head .. tail): a
// release appends the block at the tail and records the position in
// lru_pos[b]; an entry is live while lru_pos[its block] equals its position,
// so a prefix hit or a share takes a block out by clearing lru_pos alone.
// Allocation pops the free stack first and then takes the live entries from
// the head (least recently released first), dropping their keys.  When an
// append would overflow the ring, the live entries are first compacted
// toward the head, in order.
#pragma once

#include <climits>
#include <cstdint>

#include "ptx.cuh"

namespace pkv {

constexpr int kBmThreads = 1024;

// error bits of the state's error word
constexpr uint32_t kBmErrNoSpace = 1u;     // too few free blocks (or output room) for a request
constexpr uint32_t kBmErrRange = 2u;       // a block id outside the pool
constexpr uint32_t kBmErrDoubleFree = 4u;  // a block freed more often than referenced
constexpr uint32_t kBmErrTable = 8u;       // a sequence outgrew its block-table row

struct BmState {
    int32_t *hdr;         // [0] top, [1] error word, [2] cached blocks, [3] ring head, [4] ring tail
    int32_t *free_stack;  // [NB]
    int32_t *refcount;    // [NB]
    int32_t *last_idx;    // [NB] scratch: last list position of a block in a free batch (rest: -1)
    int32_t *zeroed;      // [NB] scratch: its count reached zero in this batch (rest: 0)
    int32_t *cow_rank;    // [NB] scratch: copy-on-write candidates seen so far in a chunk (rest: 0)
    uint64_t *block_hash; // [NB] prefix-cache key the block holds (0: none)
    uint32_t *lru_pos;    // [NB] absolute ring position of a cached block's entry (kNotCached otherwise)
    int32_t *ring;        // [2 NB] eviction order: ring[pos % (2 NB)] = block
    int32_t *evicted;     // [NB] scratch: the blocks one allocation call takes from the ring, in order
};

constexpr uint32_t kNotCached = 0xffffffffu;

__device__ __forceinline__ void bm_error(const BmState &s, uint32_t bits) {
    atomicOr(reinterpret_cast<unsigned int *>(s.hdr + 1), bits);
}

__device__ __forceinline__ int bm_cached(const BmState &s, int nb) { return min(max(s.hdr[2], 0), nb); }
__device__ __forceinline__ uint32_t ring_head(const BmState &s) { return (uint32_t)s.hdr[3]; }
__device__ __forceinline__ uint32_t ring_tail(const BmState &s) { return (uint32_t)s.hdr[4]; }

// Whether the ring entry at absolute position pos is live (its block's
// current entry); returns the block, or -1.
__device__ __forceinline__ int32_t ring_live(const BmState &s, int nb, uint32_t pos) {
    const int32_t b = s.ring[pos % (uint32_t)(2 * nb)];
    return (b >= 0 && b < nb && s.lru_pos[b] == pos) ? b : -1;
}

// A block mapped again (a prefix hit or a share) whose count was zero leaves
// the eviction order.
__device__ __forceinline__ void bm_revive(const BmState &s, int32_t b) {
    if (s.lru_pos[b] != kNotCached) {
        s.lru_pos[b] = kNotCached;
        atomicSub(&s.hdr[2], 1);
    }
}

// The stack top as stored, clamped into [0, nb] (a corrupted state cannot
// send a pop or push outside the stack).
__device__ __forceinline__ int bm_top(const BmState &s, int nb) { return min(max(s.hdr[0], 0), nb); }

// Block-wide exclusive scan of one int per thread (a block of any multiple of
// 32 threads up to 1024); returns the exclusive prefix and writes the block
// total to *total (all threads).
__device__ __forceinline__ int block_scan_excl(int v, int *warp_sums, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        warp_sums[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int before = warp == 0 ? 0 : warp_sums[warp - 1];
    *total = warp_sums[31];
    __syncthreads();  // warp_sums reusable after return
    return before + x - v;
}

// N exclusive scans at once (one pass, three block barriers): v[k] becomes
// its exclusive prefix and total[k] the block total.  warp_sums holds N * 32
// ints.
template <int N>
__device__ __forceinline__ void block_scan_excl_n(int (&v)[N], int *warp_sums, int (&total)[N]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x[N];
#pragma unroll
    for (int k = 0; k < N; ++k) {
        x[k] = v[k];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x[k], o);
            if (lane >= o) x[k] += y;
        }
        if (lane == 31) warp_sums[k * 32 + warp] = x[k];
    }
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int k = 0; k < N; ++k) {
            int w = lane < (int)(blockDim.x >> 5) ? warp_sums[k * 32 + lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            warp_sums[k * 32 + lane] = w;  // inclusive over warps
        }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < N; ++k) {
        const int before = warp == 0 ? 0 : warp_sums[k * 32 + warp - 1];
        total[k] = warp_sums[k * 32 + 31];
        v[k] = before + x[k] - v[k];
    }
    __syncthreads();  // warp_sums reusable after return
}

__global__ void __launch_bounds__(256) bm_init_kernel(BmState s, int nb) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nb; i += gridDim.x * blockDim.x) {
        s.free_stack[i] = nb - 1 - i;  // block 0 is popped first
        s.refcount[i] = 0;
        s.last_idx[i] = -1;
        s.zeroed[i] = 0;
        s.cow_rank[i] = 0;
        s.block_hash[i] = 0;
        s.lru_pos[i] = kNotCached;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        s.hdr[0] = nb;
        s.hdr[1] = 0;
        s.hdr[2] = 0;  // cached blocks
        s.hdr[3] = 0;  // ring head
        s.hdr[4] = 0;  // ring tail
    }
}

// Block-wide maximum of one int per thread (1024 threads), on all threads.
__device__ __forceinline__ int block_max(int v, int *warp_buf) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((threadIdx.x & 31) == 0) warp_buf[threadIdx.x >> 5] = v;
    __syncthreads();
    int w = (threadIdx.x & 31) < (blockDim.x >> 5) ? warp_buf[threadIdx.x & 31] : INT_MIN;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) w = max(w, __shfl_xor_sync(0xffffffffu, w, o));
    __syncthreads();
    return w;
}

// Takes live ring entries from *cursor on until `target` blocks are in
// s.evicted (the least recently released first): each taken block loses its
// key and leaves the order.  Block-wide; `collected` (blocks already in
// s.evicted) and *cursor are the same on every thread.  Returns the new
// collected count (short of target only if the ring ran out, an inconsistent
// state).
__device__ int ring_collect(const BmState &s, int nb, int target, int collected, uint32_t *cursor,
                            int *warp_buf) {
    const uint32_t tail = ring_tail(s);
    uint32_t cur = *cursor;
    while (collected < target && cur != tail) {
        const uint32_t span = min((uint32_t)blockDim.x, tail - cur);
        const int32_t b = threadIdx.x < span ? ring_live(s, nb, cur + threadIdx.x) : -1;
        int tot;
        const int excl = block_scan_excl(b >= 0 ? 1 : 0, warp_buf, &tot);
        const bool take = b >= 0 && collected + excl < target;
        if (take) {
            s.evicted[collected + excl] = b;
            s.block_hash[b] = 0;  // evicted: its content no longer backs a prefix
            s.lru_pos[b] = kNotCached;
        }
        const int took = min(tot, target - collected);
        // past the whole span, or (stopped inside it) past the last entry taken
        const uint32_t adv = took < tot ? (uint32_t)block_max(take ? (int)threadIdx.x + 1 : 0, warp_buf) : span;
        collected += took;
        cur += adv;
    }
    *cursor = cur;
    __syncthreads();  // s.evicted visible to the whole block
    return collected;
}

// Moves the live ring entries, in order, to positions 0 .. n-1 (through the
// s.evicted scratch) and sets head = 0, tail = n.  Keeps the ring's span and
// its absolute positions small.  Block-wide.
__device__ void ring_compact(const BmState &s, int nb, int *warp_buf) {
    const uint32_t head = ring_head(s), tail = ring_tail(s);
    int n = 0;
    for (uint32_t base = head; base != tail;) {
        const uint32_t span = min((uint32_t)kBmThreads, tail - base);
        const int32_t b = threadIdx.x < span ? ring_live(s, nb, base + threadIdx.x) : -1;
        int tot;
        const int excl = block_scan_excl(b >= 0 ? 1 : 0, warp_buf, &tot);
        if (b >= 0 && n + excl < nb) s.evicted[n + excl] = b;
        n += tot;
        base += span;
    }
    n = min(n, nb);
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kBmThreads) {
        const int32_t b = s.evicted[i];
        s.ring[i] = b;
        s.lru_pos[b] = (uint32_t)i;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        s.hdr[3] = 0;
        s.hdr[4] = n;
    }
    __syncthreads();
}

// The j-th block one allocation call hands out: the free stack first, then
// the blocks collected from the eviction order.
__device__ __forceinline__ int32_t bm_pop_at(const BmState &s, int top0, int collected, int j) {
    if (j < top0) return s.free_stack[top0 - 1 - j];
    return j - top0 < collected ? s.evicted[j - top0] : -1;
}

// Request r receives counts[r] blocks at ids[offsets[r] .. offsets[r+1]),
// requests served in order while the free and cached blocks and the output
// room last.  The inclusive sum of counts only grows, so the served requests
// are a prefix.
__global__ void __launch_bounds__(kBmThreads) bm_alloc_kernel(BmState s, int nb, const int32_t *counts, int n,
                                                               int32_t *offsets, int32_t *ids, int capacity) {
    __shared__ int warp_buf[32];
    const int top0 = bm_top(s, nb);
    const int limit = min(top0 + bm_cached(s, nb), capacity);
    int run = 0;     // counts of earlier chunks
    int served = 0;  // blocks handed out (the largest fitting inclusive sum)
    bool failed = false;
    for (int base = 0; base < n; base += kBmThreads) {
        const int r = base + threadIdx.x;
        const int c = r < n ? max(__ldg(counts + r), 0) : 0;
        int tot;
        const int incl = run + block_scan_excl(c, warp_buf, &tot) + c;
        const bool fits = r < n && incl <= limit;
        served = max(served, block_max(fits ? incl : 0, warp_buf));
        failed = __syncthreads_or(r < n && !fits) || failed;
        run += tot;
    }
    // blocks beyond the free stack come from the eviction order
    uint32_t cursor = ring_head(s);
    const int want = max(0, served - top0);
    const int got = ring_collect(s, nb, want, 0, &cursor, warp_buf);
    // second walk: ids and offsets (the unserved tail needs the final total)
    run = 0;
    if (threadIdx.x == 0) offsets[0] = 0;
    for (int base = 0; base < n; base += kBmThreads) {
        const int r = base + threadIdx.x;
        const int c = r < n ? max(__ldg(counts + r), 0) : 0;
        int tot;
        const int excl = run + block_scan_excl(c, warp_buf, &tot);
        const int incl = excl + c;
        if (r < n) offsets[r + 1] = incl <= limit ? incl : served;
        if (r < n && incl <= limit) {
            for (int k = 0; k < c; ++k) {
                const int32_t blk = bm_pop_at(s, top0, got, excl + k);
                ids[excl + k] = blk;
                if (blk >= 0) s.refcount[blk] = 1;
            }
        }
        run += tot;
    }
    if (threadIdx.x == 0) {
        s.hdr[0] = top0 - min(served, top0);
        s.hdr[2] -= got;
        s.hdr[3] = (int32_t)cursor;
        if (failed) bm_error(s, kBmErrNoSpace);
        if (got < want) bm_error(s, kBmErrDoubleFree);  // fewer cached blocks than counted: inconsistent state
    }
}

// Each listed id drops a reference; a block whose count reaches zero goes back
// on the free list, pushed in list order at its last occurrence in the batch
// (the sequential order when no block is freed more often than referenced).
__global__ void __launch_bounds__(kBmThreads) bm_free_kernel(BmState s, int nb, const int32_t *list, int n) {
    __shared__ int warp_sums[32];
    for (int i = threadIdx.x; i < n; i += kBmThreads) {
        const int32_t b = __ldg(list + i);
        if (b < 0 || b >= nb) {
            bm_error(s, kBmErrRange);
            continue;
        }
        const int old = atomicSub(&s.refcount[b], 1);
        if (old <= 0) {
            atomicAdd(&s.refcount[b], 1);
            bm_error(s, kBmErrDoubleFree);
        } else if (old == 1) {
            s.zeroed[b] = 1;
        }
        atomicMax(&s.last_idx[b], i);
    }
    __syncthreads();
    // a block whose count reached zero, at its last occurrence: cached if it
    // holds a prefix key (appended to the eviction order), else free (pushed)
    auto released = [&](int i, int32_t &b) -> int {  // 0: none, 1: free, 2: cached
        if (i >= n) return 0;
        b = __ldg(list + i);
        if (b < 0 || b >= nb || s.last_idx[b] != i || !s.zeroed[b]) return 0;
        return s.block_hash[b] != 0 ? 2 : 1;
    };
    int cached_total = 0;
    for (int base = 0; base < n; base += kBmThreads) {
        int32_t b;
        cached_total += __syncthreads_count(released(base + threadIdx.x, b) == 2);
    }
    // room in the ring (2 num_blocks entries) and small absolute positions
    const uint32_t span = ring_tail(s) - ring_head(s);
    if (cached_total > 0 && (span + (uint32_t)cached_total > (uint32_t)(2 * nb) ||
                             ring_tail(s) + (uint32_t)cached_total >= 0x7fffffffu))
        ring_compact(s, nb, warp_sums);
    const int top0 = bm_top(s, nb);
    const uint32_t tail0 = ring_tail(s);
    int run = 0, run_c = 0;
    for (int base = 0; base < n; base += kBmThreads) {
        int32_t b = -1;
        const int kind = released(base + threadIdx.x, b);
        int tot, tot_c;
        const int excl = run + block_scan_excl(kind == 1, warp_sums, &tot);
        const int excl_c = run_c + block_scan_excl(kind == 2, warp_sums, &tot_c);
        if (kind == 1) {
            if (top0 + excl < nb) s.free_stack[top0 + excl] = b;
            else bm_error(s, kBmErrDoubleFree);  // more free blocks than the pool: the state was inconsistent
        } else if (kind == 2) {
            const uint32_t pos = tail0 + (uint32_t)excl_c;
            s.ring[pos % (uint32_t)(2 * nb)] = b;
            s.lru_pos[b] = pos;
        }
        run += tot;
        run_c += tot_c;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kBmThreads) {  // scratch back to rest
        const int32_t b = __ldg(list + i);
        if (b >= 0 && b < nb) {
            s.last_idx[b] = -1;
            s.zeroed[b] = 0;
        }
    }
    if (threadIdx.x == 0) {
        s.hdr[0] = min(top0 + run, nb);
        s.hdr[2] += run_c;
        s.hdr[4] = (int32_t)(tail0 + (uint32_t)run_c);
    }
}

__global__ void __launch_bounds__(256) bm_share_kernel(BmState s, int nb, const int32_t *list, int n) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const int32_t b = __ldg(list + i);
        if (b < 0 || b >= nb) bm_error(s, kBmErrRange);
        else if (atomicAdd(&s.refcount[b], 1) == 0) bm_revive(s, b);
    }
}

struct AppendParams {
    BmState s;
    int32_t *tables;  // [B][mbs]
    int32_t *ctx;     // [B], grown in place
    const int32_t *num_new;
    int64_t *slots;   // [slot_cap]: sum num_new entries written, the rest untouched
    int64_t slot_cap;
    int32_t *pairs;   // [B][2]
    int32_t *num_pairs;
    int nb, mbs, B, bs;
};

// One step's slots, by the sequential rule: in sequence order, a sequence
// whose new tokens go into a partly filled last block that others still map
// first gets a private copy of it (copy-on-write), then blocks for the logical
// indices its tokens reach, then its slots; the first sequence that finds too
// few free blocks or outgrows its table row, and every later one, is left as
// it was with slots -1.  A shared block with R references and k appending
// sharers is copied for the first min(k, R - 1) of them in sequence order and
// the last sharer writes in place; a candidate's rank among earlier
// candidates on the same block comes from __match_any_sync within its warp
// and a per-block counter walked warp by warp.
// Launched with one thread per sequence or per four output slots, whichever
// is more, rounded up to a warp (at most kBmThreads): a decode batch of 128
// takes four warps, and every block barrier waits for those alone.
__global__ void __launch_bounds__(kBmThreads) bm_append_slots_kernel(const AppendParams p) {
    __shared__ int warp_buf[3 * 32];
    // per sequence of the chunk, for the cooperative slot pass: its first
    // slot index, and its first position (-1 unless it fits)
    __shared__ int sh_slot0[kBmThreads], sh_pos0[kBmThreads];
    const BmState &s = p.s;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int top0 = bm_top(s, p.nb);
    const int avail0 = top0 + bm_cached(s, p.nb);  // free, then cached blocks
    uint32_t cursor = ring_head(s);               // eviction order: next entry to look at
    int collected = 0;                            // blocks taken from it so far (in s.evicted)
    int run_need = 0;   // blocks wanted by earlier sequences
    int run_flags = 0;  // range / table failures at earlier sequences
    int run_slots = 0;  // slot-mapping offset
    int run_pairs = 0;
    int handed = 0;     // blocks handed out
    const int nthr = blockDim.x;
    for (int base = 0; base < p.B; base += nthr) {
        const int b = base + threadIdx.x;
        const bool live = b < p.B;
        int n = 0, pos0 = 0, first_new = 0, last = -1, need_new = 0;
        int32_t cur = -1;
        bool cand = false, bad_range = false, overflow = false;
        int32_t *row = p.tables + (size_t)(live ? b : 0) * p.mbs;
        if (live) {
            n = max(__ldg(p.num_new + b), 0);
            pos0 = p.ctx[b];
            if (pos0 < 0 || pos0 > p.mbs * p.bs) {
                overflow = true;  // a context length outside its own table row (its slots stay -1)
            } else {
                first_new = (pos0 + p.bs - 1) / p.bs;
                last = n > 0 ? (pos0 + n - 1) / p.bs : first_new - 1;
                need_new = last >= first_new ? last - first_new + 1 : 0;
                if (n > 0 && pos0 % p.bs != 0) {
                    cur = row[pos0 / p.bs];
                    if (cur < 0 || cur >= p.nb) bad_range = true;
                    else cand = true;
                }
                overflow = n > 0 && last >= p.mbs;
            }
        }
        // references of a candidate's block, after earlier chunks' copies
        const int R = cand ? s.refcount[cur] : 0;
        // Only a block with more than one holder needs the ranking (its first
        // R - 1 writers copy, the last keeps it); a block with one holder is
        // written in place whatever its rank, and no other sequence holds it.
        const bool shared = cand && R > 1;
        const unsigned same = __match_any_sync(0xffffffffu, shared ? cur : -2 - (int)threadIdx.x);
        const int rank_in_warp = __popc(same & ((1u << lane) - 1u));
        int rank = 0;
        if (__syncthreads_or(shared)) {  // only when some sequence writes into a shared block
            const int live_warps = (min(nthr, p.B - base) + 31) / 32;
            for (int w = 0; w < live_warps; ++w) {
                if (warp == w && shared) {
                    rank = s.cow_rank[cur] + rank_in_warp;
                    __syncwarp(same);
                    if (rank_in_warp == 0) s.cow_rank[cur] += __popc(same);
                }
                __syncthreads();
            }
        }
        const int cow = (shared && rank < R - 1) ? 1 : 0;
        const int need = live ? need_new + cow : 0;
        const int flag = (bad_range || overflow) ? 1 : 0;
        int sc1[3] = {flag, need, n}, tot1[3];
        block_scan_excl_n<3>(sc1, warp_buf, tot1);
        const int tot_flags = tot1[0], tot_need = tot1[1], tot_n = tot1[2];
        const int flags_before = run_flags + sc1[0];
        const int excl_need = run_need + sc1[1];
        const int excl_slots = run_slots + sc1[2];
        const bool earlier_ok = flags_before == 0 && excl_need <= avail0;
        const bool fits = live && earlier_ok && !flag && excl_need + need <= avail0;
        int sc2[2] = {fits ? cow : 0, fits ? need : 0}, tot2[2];
        block_scan_excl_n<2>(sc2, warp_buf, tot2);
        const int tot_pairs = tot2[0], tot_handed = tot2[1];
        const int excl_pairs = run_pairs + sc2[0];
        // this chunk's pops beyond the free stack come from the eviction order
        collected = ring_collect(s, p.nb, max(0, handed + tot_handed - top0), collected, &cursor, warp_buf);
        if (live && bad_range) bm_error(s, kBmErrRange);
        if (live && earlier_ok && !fits && !bad_range) bm_error(s, overflow ? kBmErrTable : kBmErrNoSpace);
        if (fits) {
            int k = 0;
            if (cow) {
                const int32_t fresh = bm_pop_at(s, top0, collected, excl_need);
                s.refcount[fresh] = 1;
                atomicSub(&s.refcount[cur], 1);
                row[pos0 / p.bs] = fresh;
                p.pairs[2 * excl_pairs] = cur;
                p.pairs[2 * excl_pairs + 1] = fresh;
                k = 1;
            }
            for (int L = first_new; L <= last; ++L, ++k) {
                const int32_t fresh = bm_pop_at(s, top0, collected, excl_need + k);
                s.refcount[fresh] = 1;
                row[L] = fresh;
            }
            p.ctx[b] = pos0 + n;
        }
        sh_slot0[threadIdx.x] = live ? excl_slots : 0;
        sh_pos0[threadIdx.x] = fits ? pos0 : -1;
        __syncthreads();
        // slots of the whole chunk, all threads: entry j belongs to the last
        // sequence whose first slot is <= j (binary search over the chunk; a
        // sequence without new tokens shares its first slot with the next one,
        // so the last such sequence is always one that owns entry j)
        const int chunk_first = sh_slot0[0];
        const int nlive = min(nthr, p.B - base);
        for (int j = chunk_first + threadIdx.x; j < run_slots + tot_n; j += nthr) {
            int lo = 0, hi = nlive - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (sh_slot0[mid] <= j) lo = mid;
                else hi = mid - 1;
            }
            if (j >= p.slot_cap) continue;
            const int q0 = sh_pos0[lo];
            if (q0 < 0) {
                p.slots[j] = -1;
            } else {
                const int pos = q0 + (j - sh_slot0[lo]);
                const int32_t *qrow = p.tables + (size_t)(base + lo) * p.mbs;
                p.slots[j] = (int64_t)qrow[pos / p.bs] * p.bs + pos % p.bs;
            }
        }
        if (live && (int64_t)excl_slots + n > p.slot_cap) bm_error(s, kBmErrNoSpace);  // output too short
        if (shared) s.cow_rank[cur] = 0;  // scratch back to rest
        __syncthreads();
        run_need += tot_need;
        run_flags += tot_flags;
        run_slots += tot_n;
        run_pairs += tot_pairs;
        handed += tot_handed;
    }
    if (threadIdx.x == 0) {
        *p.num_pairs = run_pairs;
        s.hdr[0] = top0 - min(handed, top0);
        s.hdr[2] -= collected;
        s.hdr[3] = (int32_t)cursor;
    }
}

// ------------------------------------------------------------ prefix cache --
// Full prompt blocks are keyed by FNV-1a 64 (offset basis 14695981039346656037,
// prime 1099511628211, xor then multiply per byte) chained over the prefix:
// d_i = FNV-1a of the block's tokens as little-endian int32 bytes, key_i =
// FNV-1a of le64(key_{i-1}) || le64(d_i) with key_{-1} = 0; key 0 is stored as
// 1.  The cache is an open-addressing table of (key, block) pairs with linear
// probing; an entry counts only while its block still holds the key
// (block_hash): allocated, or cached and not yet evicted.
constexpr uint64_t kFnvBasis = 14695981039346656037ull;
constexpr uint64_t kFnvPrime = 1099511628211ull;

struct PrefixCache {
    unsigned long long *keys;  // [cap], 0 = empty
    int32_t *vals;             // [cap] block ids
    int32_t *claim;            // [cap] scratch: earliest inserting sequence (rest: INT32_MAX)
    int cap;                   // power of two
};

__device__ __forceinline__ uint64_t fnv_u32(uint64_t h, uint32_t w) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        h ^= (w >> (8 * i)) & 0xffu;
        h *= kFnvPrime;
    }
    return h;
}

__device__ __forceinline__ uint64_t prefix_block_key(uint64_t prev, const int32_t *tok, int bs) {
    uint64_t d = kFnvBasis;
    for (int t = 0; t < bs; ++t) d = fnv_u32(d, (uint32_t)__ldg(tok + t));
    uint64_t k = kFnvBasis;
    k = fnv_u32(k, (uint32_t)prev);
    k = fnv_u32(k, (uint32_t)(prev >> 32));
    k = fnv_u32(k, (uint32_t)d);
    k = fnv_u32(k, (uint32_t)(d >> 32));
    return k ? k : 1;
}

// Slot holding key, or -1 (an empty slot ends the probe).
__device__ __forceinline__ int cache_find(const PrefixCache &c, uint64_t key) {
    int slot = (int)(key & (uint64_t)(c.cap - 1));
    for (int n = 0; n < c.cap; ++n) {
        const unsigned long long k = c.keys[slot];
        if (k == key) return slot;
        if (k == 0ull) return -1;
        slot = (slot + 1) & (c.cap - 1);
    }
    return -1;
}

__device__ __forceinline__ bool holder_valid(const BmState &s, int nb, int32_t b, uint64_t key) {
    return b >= 0 && b < nb && s.block_hash[b] == key;
}

__global__ void __launch_bounds__(256) prefix_cache_init_kernel(PrefixCache c) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < c.cap; i += gridDim.x * blockDim.x) {
        c.keys[i] = 0ull;
        c.vals[i] = -1;
        c.claim[i] = 0x7fffffff;
    }
}

struct PrefixParams {
    BmState s;
    PrefixCache c;
    const int32_t *tokens;       // prompts, concatenated
    const int32_t *query_start;  // [B+1]
    int32_t *tables;             // [B][mbs]
    int32_t *num_cached;         // [B] (lookup)
    int nb, B, bs, mbs;
};

// Keys of blocks base .. base+31 of one prompt, one warp: lane l hashes the
// tokens of block base + l (its digest), then every lane walks the chain over
// the shuffled digests in lockstep and keeps the key of its own block.  prev
// enters as the key of block base - 1 (0 before block 0) and leaves as the key
// of the group's last block; lanes past `count` get 0.
__device__ __forceinline__ uint64_t warp_block_keys(const int32_t *tok0, int base, int count, int bs, uint64_t &prev) {
    const int lane = threadIdx.x & 31;
    const int i = base + lane;
    uint64_t d = kFnvBasis;
    if (i < count)
        for (int t = 0; t < bs; ++t) d = fnv_u32(d, (uint32_t)__ldg(tok0 + (size_t)i * bs + t));
    uint64_t mine = 0;
    const int n = min(32, count - base);
    for (int j = 0; j < n; ++j) {
        const uint64_t dj = __shfl_sync(0xffffffffu, d, j);
        uint64_t k = kFnvBasis;
        k = fnv_u32(k, (uint32_t)prev);
        k = fnv_u32(k, (uint32_t)(prev >> 32));
        k = fnv_u32(k, (uint32_t)dj);
        k = fnv_u32(k, (uint32_t)(dj >> 32));
        prev = k ? k : 1;
        if (lane == j) mine = prev;
    }
    return mine;
}

// Lookup, one warp per sequence: the leading prompt blocks whose keys have a
// valid holder -- at least one prompt token is left to compute -- are mapped
// into the sequence's table row with one reference each (a cached holder
// leaves the eviction order).
__global__ void __launch_bounds__(256) prefix_lookup_kernel(const PrefixParams p) {
    const int s = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (s >= p.B) return;  // whole warps
    const int q0 = __ldg(p.query_start + s);
    const int n = __ldg(p.query_start + s + 1) - q0;
    const int look = min(n > 0 ? (n - 1) / p.bs : 0, p.mbs);
    uint64_t prev = 0;
    int hits = 0;
    for (int base = 0; base < look; base += 32) {
        const uint64_t key = warp_block_keys(p.tokens + q0, base, look, p.bs, prev);
        const int i = base + lane;
        int32_t b = -1;
        bool valid = false;
        if (i < look) {
            const int slot = cache_find(p.c, key);
            b = slot >= 0 ? p.c.vals[slot] : -1;
            valid = holder_valid(p.s, p.nb, b, key);
        }
        const unsigned hit = __ballot_sync(0xffffffffu, valid);
        const int lead = hit == 0xffffffffu ? 32 : __ffs(~hit) - 1;  // leading run of hits
        if (lane < lead) {
            p.tables[(size_t)s * p.mbs + i] = b;
            if (atomicAdd(&p.s.refcount[b], 1) == 0) bm_revive(p.s, b);  // a cached holder is mapped again
        }
        hits += lead;
        if (lead < min(32, look - base)) break;
    }
    if (lane == 0) p.num_cached[s] = hits * p.bs;
}

// Insert, one warp per sequence over all sequences at once, in three launches
// (a kernel boundary orders the passes grid-wide): pass 0 puts each new key in
// the table (CAS into an empty slot) and, when the key has no valid holder,
// claims the slot with the sequence index (atomicMin: the earliest sequence
// wins, as in sequence order); pass 1 lets the winners record their blocks;
// pass 2 returns the claims to rest.  A block id outside the pool stops the
// sequence there (and is reported).
template <int PASS>
__global__ void __launch_bounds__(256) prefix_insert_kernel(const PrefixParams p) {
    const int s = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (s >= p.B) return;  // whole warps
    const int q0 = __ldg(p.query_start + s);
    const int full = min((__ldg(p.query_start + s + 1) - q0) / p.bs, p.mbs);
    uint64_t prev = 0;
    for (int gb = 0; gb < full; gb += 32) {
        const uint64_t key = warp_block_keys(p.tokens + q0, gb, full, p.bs, prev);
        const int i = gb + lane;
        const int32_t b = i < full ? p.tables[(size_t)s * p.mbs + i] : 0;
        const unsigned bad = __ballot_sync(0xffffffffu, i < full && (b < 0 || b >= p.nb));
        const int stop = bad ? __ffs(bad) - 1 : 32;  // blocks from here on are not inserted
        if (PASS == 0 && bad && lane == stop) bm_error(p.s, kBmErrRange);
        if (i < full && lane < stop) {
            if (PASS == 0) {
                if (p.s.block_hash[b] != key) {
                    int slot = (int)(key & (uint64_t)(p.c.cap - 1));
                    int found = -1;
                    for (int t = 0; t < p.c.cap; ++t) {
                        const unsigned long long k = atomicCAS(&p.c.keys[slot], 0ull, (unsigned long long)key);
                        if (k == 0ull || k == key) {
                            found = slot;
                            break;
                        }
                        slot = (slot + 1) & (p.c.cap - 1);
                    }
                    if (found < 0) bm_error(p.s, kBmErrNoSpace);
                    else if (!holder_valid(p.s, p.nb, p.c.vals[found], key)) atomicMin(&p.c.claim[found], s);
                }
            } else {
                const int slot = cache_find(p.c, key);
                if (slot >= 0) {
                    if (PASS == 1 && p.c.claim[slot] == s) {
                        p.c.vals[slot] = b;
                        p.s.block_hash[b] = key;
                    } else if (PASS == 2) {
                        p.c.claim[slot] = 0x7fffffff;
                    }
                }
            }
        }
        if (bad) break;
    }
}

// Copy-on-write pairs kept on the device (as bm_append_slots leaves them):
// grid.y = pair slot up to max_pairs; slots at or past *num_pairs do nothing.
// The pairs' destinations are fresh blocks, never another pair's source.
constexpr int kCopyDevThreads = 256;
constexpr int kCopyDevVec = 4;

__global__ void __launch_bounds__(kCopyDevThreads) copy_blocks_dev_kernel(uint4 *k_cache, uint4 *v_cache,
                                                                          const int32_t *pairs,
                                                                          const int32_t *num_pairs,
                                                                          int64_t vec_per_block, int nb, int first) {
    const int pr = blockIdx.y;  // pair first + pr of the list; pairs points at pair first
    if (first + pr >= *num_pairs) return;
    const int32_t src = __ldg(pairs + 2 * pr), dst = __ldg(pairs + 2 * pr + 1);
    if (src < 0 || src >= nb || dst < 0 || dst >= nb) {
        if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(PKV_DEVERR_BLOCK);
        return;
    }
    const int64_t base = (int64_t)blockIdx.x * (kCopyDevThreads * kCopyDevVec) + threadIdx.x;
    uint4 kv[kCopyDevVec], vv[kCopyDevVec];
#pragma unroll
    for (int u = 0; u < kCopyDevVec; ++u) {
        const int64_t e = base + u * kCopyDevThreads;
        if (e < vec_per_block) {
            kv[u] = k_cache[src * vec_per_block + e];
            vv[u] = v_cache[src * vec_per_block + e];
        }
    }
#pragma unroll
    for (int u = 0; u < kCopyDevVec; ++u) {
        const int64_t e = base + u * kCopyDevThreads;
        if (e < vec_per_block) {
            k_cache[dst * vec_per_block + e] = kv[u];
            v_cache[dst * vec_per_block + e] = vv[u];
        }
    }
}

}  // namespace pkv
