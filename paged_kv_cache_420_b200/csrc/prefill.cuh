// prefill.cuh -- chunked-prefill paged attention for sm_100a: several new
// query tokens per sequence, causal within the new chunk, keys and values read
// through the block table (wkbse.com "加速 LLM 推理：深入了解 vllm 引擎",
// section 3.1; a token attends to itself and its past).
//
// Sequence s holds context_lens[s] tokens in the cache, the last q_len of which
// are the new chunk (query_start[s] .. query_start[s+1]-1 in q/out).  Query
// token i of the chunk is at position pos = ctx - q_len + i and attends to
// positions [0, pos].
//
// This header holds what the attention kernel (prefill_tc.cuh) builds on: the
// call's parameters, the clamped lengths of a sequence, and the planner that
// lists the (sequence, query tile) items, longest first.  No split-K: an item
// walks its whole causal key range.
#pragma once

#include "decode.cuh"

namespace pkv {

struct PrefillParams {
    const __nv_bfloat16 *q;       // [T][Hq][D]
    __nv_bfloat16 *out;           // [T][Hq][D]
    const int32_t *block_tables;  // [B][MBS]
    const int32_t *context_lens;  // [B]
    const int32_t *query_start;   // [B+1]
    int2 *entries;                // workspace: (seq, query tile), longest first
    int2 *staged;                 // workspace: the same entries in sequence order
    int32_t *num_entries;
    int32_t *work_counter;
    int B, Hq, Hkv, g, MBS, bs, NB, max_ctx, max_q, QT, T;
    int pool_rows;
    float scale_log2;
};

// Query length and cached prefix of sequence s, clamped to what the table, the
// workspace and the context allow (reported once, by the planner).
// From the loaded values: ctx = context_lens[s], q_begin = query_start[s],
// q_end = query_start[s + 1].
__device__ __forceinline__ void prefill_lengths_of(const PrefillParams &p, int ctx, int q_begin, int q_end,
                                                   bool report, int &q_len, int &prefix) {
    const long long cap = min((long long)p.MBS * p.bs, (long long)p.max_ctx);
    int ql = q_end - q_begin;
    bool bad = false;
    if (q_begin < 0 || q_begin > p.T) { bad = true; ql = 0; }
    else if (ql > p.T - q_begin) { bad = true; ql = p.T - q_begin; }
    if (ctx < 0 || ctx > cap) { bad = true; ctx = ctx < 0 ? 0 : (int)cap; }
    if (ql < 0 || ql > p.max_q || ql > ctx) { bad = true; ql = max(0, min(min(ql, p.max_q), ctx)); }
    if (bad && report) raise_error(PKV_DEVERR_CONTEXT);
    q_len = ql;
    prefix = ctx - ql;
}

__device__ __forceinline__ void prefill_lengths(const PrefillParams &p, int s, bool report, int &q_len,
                                                int &prefix) {
    prefill_lengths_of(p, __ldg(p.context_lens + s), __ldg(p.query_start + s), __ldg(p.query_start + s + 1),
                       report, q_len, prefix);
}

// Keys an item walks, in 64-key units, as the planner's sort key (an item's
// cost grows with it); items longer than the histogram share its last bucket.
constexpr int kPlanBuckets = 4096;
__device__ __forceinline__ int prefill_sort_key(const PrefillParams &p, int q_len, int prefix, int tile) {
    const int n_keys = prefix + min(q_len, (tile + 1) * p.QT);
    return min(n_keys >> 6, kPlanBuckets - 1);
}

// Planner: lists the (s, tile) entries, longest first, and zeroes the work
// counter.  The attention kernel's CTAs claim items in list order, so the
// last items claimed are the shortest and the CTAs finish close together.
// Entries go to `staged` in sequence order with a histogram of their sort
// keys; a descending scan of the histogram gives each key's first slot and
// the entries are scattered to `entries` (order within a key is arbitrary:
// items are independent).
__global__ void __launch_bounds__(kPlanThreads) plan_prefill_kernel(PrefillParams p) {
    __shared__ int s_off[kPlanThreads + 1];
    __shared__ int s_warp[kPlanThreads / 32];
    __shared__ int s_carry;
    __shared__ int s_ql[kPlanThreads], s_pre[kPlanThreads];
    __shared__ int s_hist[kPlanBuckets];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    grid_launch_dependents();
    for (int i = tid; i < kPlanBuckets; i += kPlanThreads) s_hist[i] = 0;
    if (tid == 0) s_carry = 0;
    __syncthreads();
    for (int base = 0; base < p.B; base += kPlanThreads) {
        const int s = base + tid;
        int tiles = 0, ql = 0, prefix = 0;
        if (s < p.B) {
            prefill_lengths(p, s, true, ql, prefix);
            tiles = (ql + p.QT - 1) / p.QT;
        }
        s_ql[tid] = ql;
        s_pre[tid] = prefix;
        int x = tiles;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) s_warp[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int w = s_warp[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            s_warp[lane] = w;
        }
        __syncthreads();
        s_off[tid + 1] = x + (warp > 0 ? s_warp[warp - 1] : 0);
        if (tid == 0) s_off[0] = 0;
        __syncthreads();
        const int chunk_total = s_off[kPlanThreads];
        const int carry = s_carry;
        for (int e = tid; e < chunk_total; e += kPlanThreads) {
            int lo = 0, hi = kPlanThreads - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_off[mid] <= e) lo = mid; else hi = mid - 1;
            }
            const int n_tiles = s_off[lo + 1] - s_off[lo];
            const int tile = n_tiles - 1 - (e - s_off[lo]);
            p.staged[carry + e] = make_int2(base + lo, tile);
            atomicAdd(&s_hist[prefill_sort_key(p, s_ql[lo], s_pre[lo], tile)], 1);
        }
        __syncthreads();
        if (tid == 0) s_carry = carry + chunk_total;
        __syncthreads();
    }
    const int total = s_carry;
    // first slot of each key, longest key first: exclusive scan of the
    // histogram from the top bucket down (thread t owns 4 buckets)
    static_assert(kPlanBuckets == 4 * kPlanThreads, "four buckets per thread");
    {
        const int b0 = kPlanBuckets - 1 - 4 * tid;  // this thread's buckets: b0, b0-1, b0-2, b0-3
        int c[4], sum = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            c[i] = s_hist[b0 - i];
            sum += c[i];
        }
        int x = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) s_warp[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int w = s_warp[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            s_warp[lane] = w;
        }
        __syncthreads();
        int start = x - sum + (warp > 0 ? s_warp[warp - 1] : 0);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            s_hist[b0 - i] = start;
            start += c[i];
        }
    }
    __syncthreads();
    for (int e = tid; e < total; e += kPlanThreads) {
        const int2 st = p.staged[e];
        int ql, prefix;
        prefill_lengths(p, st.x, false, ql, prefix);
        p.entries[atomicAdd(&s_hist[prefill_sort_key(p, ql, prefix, st.y)], 1)] = st;
    }
    if (tid == 0) {
        *p.num_entries = total;
        *p.work_counter = 0;
    }
}

}  // namespace pkv
