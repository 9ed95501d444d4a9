// decode.cuh -- paged decode attention for sm_100a.
//
// Method (wkbse.com "加速 LLM 推理：深入了解 vllm 引擎", sections 3.1 and 3.3):
// every sequence's query attends over its context, whose K/V rows are found
// through the block table (logical block i / bs -> physical id, offset
// i % bs); scale, softmax and the weighted sum of V are fused in one pass
// (online softmax in fp32, exp2 with scale*log2(e) folded in).
//
// Work decomposition.  A unit (sequence s, kv head h) is cut into partitions
// of PT tokens; an item = (s, h, partition).  A one-CTA planner kernel writes
// the (s, partition) list in sequence-major order.  The attention kernel is
// persistent: CTAs claim items from a global counter in list order.  Inside a CTA one
// producer warp walks the items' 16-token stages and fills a ring of NS
// shared-memory slots with TMA tensor loads (K and V tiles of 16 rows x D,
// 128-byte swizzle) addressed through the block table; W consumer warps take
// the stages round-robin, each keeping its own online-softmax state, and merge
// their partial (m, l, acc) per item through shared memory.  A unit with one
// partition writes bf16 out directly; otherwise the partition's (m, l, acc)
// goes to the workspace and a reduce kernel merges them by log-sum-exp.
//
// Two consumer arithmetic paths:
//  * MHA (g = 1): CUDA cores.  A lane owns D/32 elements of every row; q.k
//    partial sums of the 16 tokens are reduced by a transposing butterfly of
//    warp shuffles; p is broadcast by shuffles for the PV sum.
//  * 2 <= g <= 16: the g query heads of one kv head form a tile, so QK^T and
//    PV run on tensor cores (mma.sync m16n8k16 bf16, fp32 accumulate):
//    S^T[16 tokens x 8 heads] = K_tile . Q^T, O^T[D x 8 heads] += V^T . P^T,
//    with P^T moved from accumulator to operand layout by movmatrix.
#pragma once

#include "ptx.cuh"

namespace pkv {

constexpr int kStageTok = 16;                     // tokens per pipeline stage (one TMA box height)
constexpr int kConsumerWarps = 4;                 // W
static_assert(32 % kConsumerWarps == 0, "stage groups must tile the 32-entry table prefetch");
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr int kPlanThreads = 1024;
constexpr int kReduceWarps = 4;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded on-chip waits: 2 s
// Online softmax keeps a reference max m per head and raises it only when a
// stage's max exceeds it by more than this (log2 units), so most stages skip
// the rescale of acc and l.  Weights 2^(s - m) then stay below 2^8: exact
// enough in fp32, and the final out = acc / l does not depend on m.
constexpr float kRescaleSlack = 8.0f;
#define PKV_NEG_INF (-__int_as_float(0x7f800000))

struct DecodeParams {
    const __nv_bfloat16 *q;       // [B][Hq][D]
    __nv_bfloat16 *out;           // [B][Hq][D]
    const int32_t *block_tables;  // [B][MBS]
    const int32_t *context_lens;  // [B]
    int2 *entries;                // workspace: (seq, partition), sequence-major
    int32_t *num_entries;         // workspace: number of entries
    int32_t *work_counter;        // workspace: next unclaimed item (zeroed by the planner)
    float2 *part_ml;              // workspace: [B][Hq][maxP] = (m in log2 units, l)
    float *part_acc;              // workspace: [B][Hq][maxP][D]
    int B, Hq, Hkv, g, MBS, bs, NB, max_ctx, PT, maxP;
    int pool_rows;                // NB * Hkv * bs: first out-of-range TMA row
    float scale_log2;             // scale * log2(e)
    const float *k_scale = nullptr;  // FP8 pool: dequantisation scale per kv head (nullptr: bf16 pool)
    const float *v_scale = nullptr;
};

// A context length clamped to what the table and the workspace can hold.  A
// value outside [0, cap] is reported (once, by the planner).
__device__ __forceinline__ int clamp_context(const DecodeParams &p, int n, bool report) {
    const long long table_cap = (long long)p.MBS * p.bs;
    const int cap = (int)min(table_cap, (long long)p.max_ctx);
    if (n < 0 || n > cap) {
        if (report) raise_error(PKV_DEVERR_CONTEXT);
        return n < 0 ? 0 : cap;
    }
    return n;
}

__device__ __forceinline__ int clamped_context(const DecodeParams &p, int s, bool report) {
    return clamp_context(p, __ldg(p.context_lens + s), report);
}

// ------------------------------------------------------------- planner ----
// Entry flag: the entry is a partition group, W consecutive partitions
// (part .. part + W - 1) of one sequence.  Its W partitions stream
// interleaved, one per consumer warp, and each warp writes its partition's
// (m, l, acc) record itself, so the item needs no merge across warps.
constexpr int kGroupFlag = 1 << 30;

// Partition groups of a sequence with `parts` partitions: only split calls
// (the records go to the workspace anyway) on the tensor-core path (a group
// saves the merge of W multi-head partials; on the single-head CUDA-core path
// the merge is cheap and groups measured slower), and only whole groups of W.
__device__ __forceinline__ int group_count(const DecodeParams &p, int parts) {
    return (p.maxP > 1 && p.g > 1) ? parts / kConsumerWarps : 0;
}

// Split-K records of a sequence with `parts` partitions: one per partition
// group (its W partitions merged inside the CTA), then one per single
// partition.  Index of the record that holds partition `part`.
__device__ __forceinline__ int record_index(const DecodeParams &p, int parts, int part) {
    const int groups = group_count(p, parts);
    return part < groups * kConsumerWarps ? part / kConsumerWarps : part - (kConsumerWarps - 1) * groups;
}

// Writes the entry list and its count, and zeroes the attention kernel's work
// counter.  Every sequence's partition groups come first, then the remaining
// single partitions (each sequence-major): the large items are claimed first
// and the small ones fill the end of the kernel.  Zero-length sequences get a
// zero output row here (they have no items).
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(DecodeParams p, int D) {
    __shared__ int s_goff[kPlanThreads + 1], s_soff[kPlanThreads + 1];
    __shared__ int s_n[kPlanThreads];
    __shared__ int s_warp[kPlanThreads / 32];
    __shared__ int s_any_zero;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // The attention kernel may start its prologue now; it waits for this
    // grid's results with griddepcontrol.wait before reading them.
    grid_launch_dependents();
    if (tid == 0) s_any_zero = 0;
    __syncthreads();
    // block-wide inclusive scan of one int per thread (all threads return)
    auto scan = [&](int x) {
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
            s_warp[lane] = w;  // inclusive over warps
        }
        __syncthreads();
        const int incl = x + (warp > 0 ? s_warp[warp - 1] : 0);
        __syncthreads();  // s_warp reusable
        return incl;
    };
    // no sequence can hold a group: one scan per chunk (the planner runs
    // before the attention kernel can read anything)
    const bool can_group = group_count(p, p.maxP) > 0;
    // Single partitions go after all groups: with more sequences than one
    // chunk the total of groups is counted first.
    int groups_total = 0;
    if (can_group && p.B > kPlanThreads) {
        for (int base = 0; base < p.B; base += kPlanThreads) {
            const int s = base + tid;
            int c = 0;
            if (s < p.B) c = group_count(p, (clamped_context(p, s, false) + p.PT - 1) / p.PT);
            const int incl = scan(c);
            if (tid == kPlanThreads - 1) s_goff[kPlanThreads] = incl;  // the chunk's total
            __syncthreads();
            groups_total += s_goff[kPlanThreads];
            __syncthreads();
        }
    }
    int carry_g = 0, carry_s = 0;
    for (int base = 0; base < p.B; base += kPlanThreads) {
        const int s = base + tid;
        int groups = 0, singles = 0, n = 0;
        if (s < p.B) {
            n = clamped_context(p, s, true);
            const int parts = (n + p.PT - 1) / p.PT;
            groups = group_count(p, parts);
            singles = parts - groups * kConsumerWarps;
            if (n == 0) s_any_zero = 1;
        }
        s_n[tid] = n;
        const int ig = can_group ? scan(groups) : 0;
        const int is = scan(singles);
        s_goff[tid + 1] = ig;
        s_soff[tid + 1] = is;
        if (tid == 0) { s_goff[0] = 0; s_soff[0] = 0; }
        __syncthreads();
        const int chunk_g = s_goff[kPlanThreads], chunk_s = s_soff[kPlanThreads];
        if (p.B <= kPlanThreads) groups_total = chunk_g;
        // cooperative fill: entry e of this chunk belongs to the last seq
        // whose exclusive offset is <= e
        for (int e = tid; e < chunk_g + chunk_s; e += kPlanThreads) {
            const bool is_group = e < chunk_g;
            const int *off = is_group ? s_goff : s_soff;
            const int ee = is_group ? e : e - chunk_g;
            int lo = 0, hi = kPlanThreads - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (off[mid] <= ee) lo = mid; else hi = mid - 1;
            }
            const int i = ee - off[lo];
            if (is_group) {
                p.entries[carry_g + ee] = make_int2(base + lo, (i * kConsumerWarps) | kGroupFlag);
            } else {
                const int parts = (s_n[lo] + p.PT - 1) / p.PT;
                p.entries[groups_total + carry_s + ee] =
                    make_int2(base + lo, group_count(p, parts) * kConsumerWarps + i);
            }
        }
        carry_g += chunk_g;
        carry_s += chunk_s;
        __syncthreads();
    }
    if (tid == 0) {
        *p.num_entries = carry_g + carry_s;
        *p.work_counter = 0;
    }
    __syncthreads();
    if (s_any_zero) {
        const int vec_per_seq = p.Hq * D / 8;
        uint4 *out = reinterpret_cast<uint4 *>(p.out);
        for (long long i = tid; i < (long long)p.B * vec_per_seq; i += kPlanThreads) {
            const int s = (int)(i / vec_per_seq);
            if (clamped_context(p, s, false) == 0) out[i] = make_uint4(0, 0, 0, 0);
        }
    }
}

// ------------------------------------------------------ attention kernel ----

struct __align__(16) StageInfo {
    int s, h;
    int part;    // first partition, | kGroupFlag for a partition group (warp w owns partition part + w)
    int nparts;  // partitions of the sequence
    int k, npad; // stage index within the item, stages padded to a multiple of W
    int valid;   // valid tokens in this stage (0 = padding stage)
    int ord;     // CTA-local item ordinal (selects the q buffer); -1 ends the stream
};

// An item as the producer sees it.  A single partition streams its stages in
// order; a partition group interleaves its W partitions (stage K is stage
// K / W of partition part + K % W), so consumer warp w, which takes stages
// w, w + W, ..., walks partition part + w alone.
static_assert(kConsumerWarps == 4, "a partition group is 4 partitions: stage K -> (K & 3, K >> 2)");

struct ItemMeta {
    int s, h, part, grp, n, nparts;
    int npad;  // stages, padded to a multiple of W

    // partition (relative to part) and first token of stage K
    __device__ __forceinline__ int stage_sub(int K) const { return grp ? (K & 3) : 0; }
    __device__ __forceinline__ int stage_token(int K, int PT) const {
        return (part + stage_sub(K)) * PT + (grp ? (K >> 2) : K) * kStageTok;
    }
    // valid tokens of stage K (0: a padding stage)
    __device__ __forceinline__ int stage_valid(int K, int PT) const {
        const int sub = stage_sub(K);
        const int tok = stage_token(K, PT);
        const int t1 = min(n, (part + sub + 1) * PT);
        return tok < t1 ? min(kStageTok, t1 - tok) : 0;
    }
};

template <int D, int GP, int NS, bool KV8 = false>
struct DecodeSmem {
    static constexpr int kW = kConsumerWarps;
    static constexpr int kElem = KV8 ? 1 : 2;             // bytes per K/V element (e4m3 or bf16)
    static constexpr int kHalfTile = kStageTok * 128;     // one TMA box: 16 rows x 128 bytes = 2 KB
    static constexpr int kBoxes = D * kElem / 128;        // boxes per row of a tile
    static constexpr int kTile = kStageTok * D * kElem;   // one K (or V) stage tile
    static constexpr int kStage = 2 * kTile;
    static constexpr int kQBuf = GP * D * 2;              // the query heads of one kv head
    static constexpr int kMergeStride = D + 4;            // floats, padded against bank conflicts
    static constexpr int oTiles = 0;
    static constexpr int oQ = oTiles + NS * kStage;
    static constexpr int oMergeO = oQ + 2 * kQBuf;
    static constexpr int oMergeM = oMergeO + kW * GP * kMergeStride * 4;
    static constexpr int oMergeL = oMergeM + kW * GP * 4;
    static constexpr int oBars = (oMergeL + kW * GP * 4 + 7) / 8 * 8;
    static constexpr int kNumBars = 2 * NS + 6;  // full, empty, qfull[2], qempty[2], mfull, mempty
    static constexpr int oInfo = oBars + kNumBars * 8;
    static constexpr int oAbort = oInfo + NS * (int)sizeof(StageInfo);
    static constexpr int kBytes = oAbort + 16;
    static constexpr int kAlloc = kBytes;  // the dynamic window is 1 KB-aligned (checked in the kernel)
};

// Bounded wait that also gives up when another warp has aborted.  After the
// first test the warp sleeps on the barrier (up to kWaitSleepNs per test, woken
// by the phase's completion), so waiting warps do not take issue slots from
// the warps that compute.
constexpr uint32_t kWaitSleepNs = 20000;
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                              uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > limit_ns) {
            raise_error(PKV_DEVERR_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
}

// The producer's wait for a free ring slot.  The consumers free slots at the
// rate they compute, so while the ring is full the producer backs off with a
// short sleep between tests instead of spinning: on the CUDA-core path the
// consumer warps are close to issue-bound and a spinning producer (one per
// CTA, up to six CTAs per SM) would take their issue slots.
constexpr uint32_t kProducerBackoffNs = 128;
__device__ __forceinline__ bool wait_slot(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        __nanosleep(kProducerBackoffNs);
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            raise_error(PKV_DEVERR_TIMEOUT);
            *abort_flag = 1;
            return false;
        }
    }
}

// Byte address of element (row r, column c) of a stage tile in shared memory.
// The tile is [D/64][16][64] bf16; each 128-byte line (one row of one half)
// has its 16-byte chunks XOR-swizzled with (r & 7) by the TMA unit.
__device__ __forceinline__ uint32_t tile_addr(uint32_t tile, int r, int c) {
    const int half = c >> 6;
    const int chunk = (c & 63) >> 3;
    return tile + half * (kStageTok * 128) + r * 128 + ((chunk ^ (r & 7)) << 4) + ((c & 7) << 1);
}

// Byte address of e4m3 element (row r, column c) of an FP8 stage tile: one
// 128-byte line per row, 16-byte chunks XOR-swizzled with (r & 7).
__device__ __forceinline__ uint32_t tile_addr8(uint32_t tile, int r, int c) {
    return tile + r * 128 + ((((c >> 4) ^ (r & 7))) << 4) + (c & 15);
}

// The two code pairs of a word of four e4m3 codes as f16x2 words: lo from
// bytes 0-1, hi from bytes 2-3 (the halves are taken from the register as
// they are).
__device__ __forceinline__ void f16x2_from_e4m3x4(uint32_t w, uint32_t &lo, uint32_t &hi) {
    asm("{\n\t.reg .b16 l16, h16;\n\tmov.b32 {l16, h16}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l16;\n\tcvt.rn.f16x2.e4m3x2 %1, h16;\n\t}"
        : "=r"(lo), "=r"(hi) : "r"(w));
}

__device__ __forceinline__ uint32_t f16x2_from_f32(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// acc + a * b with f16 a, b (the low or high halves of f16x2 words) and an
// fp32 accumulator (mixed-precision FMA, sm_100).
__device__ __forceinline__ float fma_f16lo(uint32_t a, uint32_t b, float acc) {
    float r;
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.f16 %0, al, bl, %3;\n\t}"
        : "=f"(r) : "r"(a), "r"(b), "f"(acc));
    return r;
}
__device__ __forceinline__ float fma_f16hi(uint32_t a, uint32_t b, float acc) {
    float r;
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.f16 %0, ah, bh, %3;\n\t}"
        : "=f"(r) : "r"(a), "r"(b), "f"(acc));
    return r;
}

// ------------------------------------------------ CUDA-core path (g = 1) ----
// One query head per kv head (MHA).  A lane owns EPL = D/32 contiguous
// elements of every row.
// KV8: the stage tiles hold e4m3 codes.  q is kept as exact f16 pairs, K and V
// codes are converted to f16 (exactly) and multiplied in mixed precision with
// fp32 accumulation; the K scale times scale * log2 e multiplies each summed
// score, and the V scale is applied to the final output.
template <int D, bool KV8 = false>
struct SimtState {
    static constexpr int EPL = D / 32;  // elements per lane
    float q[EPL];
    uint32_t q16[EPL / 2];  // KV8: q as f16 pairs
    float kscale;           // KV8: scale * log2(e) * k_scale of the kv head
    float acc[EPL];
    float m;
    float l_part;  // this lane's share of l

    __device__ __forceinline__ void reset() {
        m = PKV_NEG_INF;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
        l_part = 0.f;
    }

    __device__ __forceinline__ void load_q(const __nv_bfloat16 *qs, int lane, float scale_log2) {
        kscale = scale_log2;
#pragma unroll
        for (int e = 0; e < EPL; e += 2) {
            const uint32_t pr = *reinterpret_cast<const uint32_t *>(qs + lane * EPL + e);
            if constexpr (KV8) {
                q16[e / 2] = f16x2_from_f32(bf16lo_to_f32(pr), bf16hi_to_f32(pr));
            } else {
                q[e] = bf16lo_to_f32(pr) * scale_log2;
                q[e + 1] = bf16hi_to_f32(pr) * scale_log2;
            }
        }
    }

    // KV8: this lane's 4 codes of row r as two f16 pairs.
    __device__ __forceinline__ void load_row8(uint32_t tile, int r, int lane, uint32_t (&h)[2]) {
        uint32_t w;
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w) : "r"(tile_addr8(tile, r, lane * EPL)));
        f16x2_from_e4m3x4(w, h[0], h[1]);
    }

    // Loads this lane's EPL elements of row r of a tile as fp32.
    __device__ __forceinline__ void load_row(uint32_t tile, int r, int lane, float (&x)[EPL]) {
        const uint32_t a = tile_addr(tile, r, lane * EPL);
        if constexpr (EPL == 4) {
            uint32_t w0, w1;
            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w0), "=r"(w1) : "r"(a));
            x[0] = bf16lo_to_f32(w0); x[1] = bf16hi_to_f32(w0);
            x[2] = bf16lo_to_f32(w1); x[3] = bf16hi_to_f32(w1);
        } else {
            uint32_t w0;
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w0) : "r"(a));
            x[0] = bf16lo_to_f32(w0); x[1] = bf16hi_to_f32(w0);
        }
    }

    // PARTIAL: fewer than 16 valid tokens in the stage (see MmaState::stage).
    template <bool PARTIAL>
    __device__ __forceinline__ void stage(uint32_t ktile, uint32_t vtile, int valid, int lane) {
        float v[16];
        // q.k partial sums v[r] of token r; tokens r and r+1 share one packed
        // fp32x2 FMA per element.
        if constexpr (KV8) {
            static_assert(EPL == 4, "FP8 stage tiles are 128-byte rows (head dim 128)");
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                uint32_t k16[2];
                load_row8(ktile, r, lane, k16);
                float d = fma_f16lo(q16[0], k16[0], 0.f);
                d = fma_f16hi(q16[0], k16[0], d);
                d = fma_f16lo(q16[1], k16[1], d);
                v[r] = fma_f16hi(q16[1], k16[1], d);
            }
        } else {
#pragma unroll
            for (int r = 0; r < 16; r += 2) {
                float x0[EPL], x1[EPL];
                load_row(ktile, r, lane, x0);
                load_row(ktile, r + 1, lane, x1);
                float d0 = 0.f, d1 = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; ++e) fma_f32x2(d0, d1, q[e], q[e], x0[e], x1[e]);
                v[r] = d0;
                v[r + 1] = d1;
            }
        }
        // Transposing butterfly: each step halves the values a lane keeps and
        // sums its half with the partner's; after it lanes 2t and 2t+1 both
        // hold the full 32-lane sum of token t.
        int n = 16;
#pragma unroll
        for (int mask = 16; mask >= 1; mask >>= 1) {
            if (n > 1) {
                const bool upper = (lane & mask) != 0;
                n >>= 1;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (i < n) {
                        const float send = upper ? v[i] : v[i + n];
                        const float keep = upper ? v[i + n] : v[i];
                        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
                    }
                }
            } else {
                v[0] += __shfl_xor_sync(0xffffffffu, v[0], mask);
            }
        }
        const int my_tok = lane >> 1;
        const float score = (!PARTIAL || my_tok < valid) ? (KV8 ? v[0] * kscale : v[0]) : PKV_NEG_INF;
        // stage max (one warp reduction), lazy rescale
        const float mx = warp_max_f32(score);
        if (mx > m + kRescaleSlack) {  // warp-uniform, rare after the first stage
            const float alpha = exp2f(m - mx);
            m = mx;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] *= alpha;
            l_part *= alpha;
        }
        const float pr = exp2f(score - m);
        l_part += pr;
        // KV8: p as an f16 pair, converted once here and shuffled as such
        const uint32_t pr16 = KV8 ? f16x2_from_f32(pr, pr) : 0u;
        // PV: broadcast p of each valid token (from lane 2r), accumulate its V
        // row (packed fp32x2 FMA over element pairs)
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            if (!PARTIAL || r < valid) {
                if constexpr (KV8) {
                    uint32_t v16[2];
                    load_row8(vtile, r, lane, v16);
                    const uint32_t p16 = __shfl_sync(0xffffffffu, pr16, 2 * r);
                    acc[0] = fma_f16lo(p16, v16[0], acc[0]);
                    acc[1] = fma_f16hi(p16, v16[0], acc[1]);
                    acc[2] = fma_f16lo(p16, v16[1], acc[2]);
                    acc[3] = fma_f16hi(p16, v16[1], acc[3]);
                } else {
                    float x[EPL];
                    load_row(vtile, r, lane, x);
                    const float pj = __shfl_sync(0xffffffffu, pr, 2 * r);
#pragma unroll
                    for (int e = 0; e < EPL; e += 2) fma_f32x2(acc[e], acc[e + 1], pj, pj, x[e], x[e + 1]);
                }
            }
        }
    }

    // Writes this warp's partial (m, l, acc) into the merge buffers.
    __device__ __forceinline__ void store_partial(float *mO, float *mM, float *mL, int w, int lane, int stride) {
        // lanes 2t and 2t+1 hold the same p: sum over one lane of each pair
        float l = l_part;
#pragma unroll
        for (int o = 2; o < 32; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
#pragma unroll
        for (int e = 0; e < EPL; ++e) mO[w * stride + lane * EPL + e] = acc[e];
        if (lane == 0) { mM[w] = m; mL[w] = l; }
    }
};

// ------------------------------------------- tensor-core path (2 <= g <= 16) --
// 8-bit transposing load of a 16 x 16 byte tile (rows from lanes 0-15): lane l
// receives rows 4(l%4) .. 4(l%4)+3 of byte column l/4 in r0 and of column
// l/4 + 8 in r1, row i of each group in byte i.
__device__ __forceinline__ void ldmatrix_b8_trans(uint32_t addr, uint32_t &r0, uint32_t &r1) {
    asm volatile("ldmatrix.sync.aligned.m16n16.x1.trans.shared.b8 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

// Token order of the FP8 tensor-core stage: A row (and k slot) r of the 16
// tokens holds token perm16(r) = 4j + {0, 1} for r = 2j + {0, 1} and
// 4j + 2 + {0, 1} for r = 8 + 2j + {0, 1}.  It makes the S^T rows that
// movmatrix turns into P^T's B fragment match the V^T A fragment that the
// 8-bit transposing load delivers (tokens 4j .. 4j+3 per lane).
__device__ __forceinline__ int perm16(int r) {
    return r < 8 ? 4 * (r >> 1) + (r & 1) : 4 * ((r - 8) >> 1) + 2 + (r & 1);
}

// H: an FP8 pool, f16 operands (the codes are exact in f16; q is converted to
// f16 and P packed as f16), otherwise bf16.  With H both operands come
// straight from the e4m3 stage tiles:
//   K: lane l (j = l % 4) loads the 4 codes of columns k0 + 4j .. 4j + 3 of
//      its two rows as one word each; the pairs (4j, 4j+1) and (4j+2, 4j+3)
//      fill the k slots (2j, 2j+1) and (2j+8, 2j+9) of the m16n8k16 A
//      fragment, and q's B fragment takes its columns in the same order (the
//      dot product does not depend on the order of k).  The rows are the
//      tokens in perm16 order.
//   V: one 8-bit transposing load per 16 head-dim columns gives lane l the
//      codes of tokens 4j .. 4j+3 at columns l/4 and l/4 + 8, which in perm16
//      order are exactly its A fragment of V^T.
template <int D, int NT, bool H = false>
struct MmaState {
    static constexpr int KS = D / 16;  // k-steps of QK^T
    static constexpr int MT = D / 16;  // m-tiles of O^T
    uint32_t qb[NT][KS][2];            // B fragments of Q^T
    float o[NT][MT][4];                // O^T accumulators
    float m[NT][2];                    // running max of heads nt*8 + 2*(lane%4) + {0,1}
    float l[NT][2];                    // this thread's share of the sums

    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int c = 0; c < 2; ++c) { m[nt][c] = PKV_NEG_INF; l[nt][c] = 0.f; }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int c = 0; c < 4; ++c) o[nt][mt][c] = 0.f;
        }
    }

    // B fragment of Q^T (k = head dim, n = head): b0 = Q[n][k0 + 2(l%4) + {0,1}],
    // b1 = the same 8 columns further; heads >= g are zero.
    __device__ __forceinline__ void load_q(const __nv_bfloat16 *qs, int lane, int g) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int head = nt * 8 + (lane >> 2);
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                // k slots 2j, 2j+1 and 2j+8, 2j+9; with H they hold columns
                // 4j, 4j+1 and 4j+2, 4j+3 (see above)
                const int col0 = H ? kk * 16 + 4 * (lane & 3) : kk * 16 + 2 * (lane & 3);
                const int col1 = H ? col0 + 2 : col0 + 8;
                uint32_t b0 = 0, b1 = 0;
                if (head < g) {
                    b0 = *reinterpret_cast<const uint32_t *>(qs + head * D + col0);
                    b1 = *reinterpret_cast<const uint32_t *>(qs + head * D + col1);
                    if constexpr (H) {
                        b0 = f16x2_from_f32(bf16lo_to_f32(b0), bf16hi_to_f32(b0));
                        b1 = f16x2_from_f32(bf16lo_to_f32(b1), bf16hi_to_f32(b1));
                    }
                }
                qb[nt][kk][0] = b0;
                qb[nt][kk][1] = b1;
            }
        }
    }

    // PARTIAL: the stage holds fewer than 16 valid tokens (a partition's last
    // stage); only then are scores past `valid` masked and the V operand's
    // rows of those tokens zeroed, so a full stage spends no instructions on it.
    template <bool PARTIAL>
    __device__ __forceinline__ void stage(uint32_t ktile, uint32_t vtile, int valid, int lane, float scale_log2) {
        // S^T[token][head] = K . Q^T
        // two independent accumulator chains (even / odd k-steps), summed after
        float s[NT][4], s2[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 4; ++c) { s[nt][c] = 0.f; s2[nt][c] = 0.f; }
        const int mi = lane >> 3, ri = lane & 7;
        uint32_t kw[4];  // H: K codes of two k-steps
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            // matrices: (rows 0-7, cols k0..+7), (rows 8-15, k0..), (rows 0-7, k0+8..), (rows 8-15, k0+8..)
            uint32_t a0, a1, a2, a3;
            if constexpr (H) {
                // one 8x8 matrix load per two k-steps: (rows perm16(0-7), bytes kk*16..+15),
                // (rows perm16(8-15), same), then the same for k-step kk + 1; lane l
                // receives codes 4(l%4) .. +3 of its rows, as one 32-bit load each would
                if ((kk & 1) == 0)
                    ldmatrix_x4(tile_addr8(ktile, perm16(ri + 8 * (mi & 1)), kk * 16 + 16 * (mi >> 1)), kw[0], kw[1],
                                kw[2], kw[3]);
                const uint32_t w0 = kw[2 * (kk & 1)], w1 = kw[2 * (kk & 1) + 1];
                f16x2_from_e4m3x4(w0, a0, a2);
                f16x2_from_e4m3x4(w1, a1, a3);
            } else {
                const int row = ri + 8 * (mi & 1);
                const int col = kk * 16 + 8 * (mi >> 1);
                ldmatrix_x4(tile_addr(ktile, row, col), a0, a1, a2, a3);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float *acc = (kk & 1) ? s2[nt] : s[nt];
                if constexpr (H) mma_f16_16816(acc[0], acc[1], acc[2], acc[3], a0, a1, a2, a3, qb[nt][kk][0], qb[nt][kk][1]);
                else mma_bf16_16816(acc[0], acc[1], acc[2], acc[3], a0, a1, a2, a3, qb[nt][kk][0], qb[nt][kk][1]);
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 4; ++c) s[nt][c] += s2[nt][c];
        const int t0 = lane >> 2;  // rows t0 and t0 + 8 (tokens, in perm16 order with H)
        const bool ok0 = !PARTIAL || (H ? perm16(t0) : t0) < valid;
        const bool ok1 = !PARTIAL || (H ? perm16(t0 + 8) : t0 + 8) < valid;
        uint32_t pb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float alpha[2], p[4], z[4];
            bool raise = false;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                z[c] = ok0 ? s[nt][c] * scale_log2 : PKV_NEG_INF;
                z[c + 2] = ok1 ? s[nt][c + 2] * scale_log2 : PKV_NEG_INF;
                float mx = fmaxf(z[c], z[c + 2]);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                // lazy rescale: raise the reference max only when exceeded by the slack
                const bool up = mx > m[nt][c] + kRescaleSlack;
                alpha[c] = up ? exp2f(m[nt][c] - mx) : 1.f;
                if (up) m[nt][c] = mx;
                raise |= up;
            }
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                p[c] = exp2f(z[c] - m[nt][c]);
                p[c + 2] = exp2f(z[c + 2] - m[nt][c]);
                l[nt][c] = l[nt][c] * alpha[c] + p[c] + p[c + 2];
            }
            // accumulator layout (token row, head pair) -> operand layout of P^T
            pb[nt][0] = movmatrix_trans(H ? f16x2_from_f32(p[0], p[1]) : pack_bf16x2(p[0], p[1]));
            pb[nt][1] = movmatrix_trans(H ? f16x2_from_f32(p[2], p[3]) : pack_bf16x2(p[2], p[3]));
            if (__any_sync(0xffffffffu, raise)) {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    o[nt][mt][0] *= alpha[0];
                    o[nt][mt][1] *= alpha[1];
                    o[nt][mt][2] *= alpha[0];
                    o[nt][mt][3] *= alpha[1];
                }
            }
        }
        // token masks of this thread's V^T operand halves: k slots 2(l%4)+{0,1}
        // and +8, i.e. tokens 2(l%4)+{0,1} and +8 (with H: 4(l%4)+{0,1} and +{2,3})
        uint32_t mask01 = 0xffffffffu, mask23 = 0xffffffffu;
        if constexpr (PARTIAL) {
            const int j0 = H ? 4 * (lane & 3) : 2 * (lane & 3);
            const int j2 = H ? j0 + 2 : j0 + 8;
            mask01 = (j0 < valid ? 0x0000ffffu : 0u) | (j0 + 1 < valid ? 0xffff0000u : 0u);
            mask23 = (j2 < valid ? 0x0000ffffu : 0u) | (j2 + 1 < valid ? 0xffff0000u : 0u);
        }
        // O^T[d][head] += V^T . P^T
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            uint32_t a0, a1, a2, a3;
            if constexpr (H) {
                uint32_t r0, r1;
                ldmatrix_b8_trans(tile_addr8(vtile, lane & 15, mt * 16), r0, r1);
                f16x2_from_e4m3x4(r0, a0, a2);  // d = l/4: tokens 4j, 4j+1 and 4j+2, 4j+3
                f16x2_from_e4m3x4(r1, a1, a3);  // d = l/4 + 8
            } else {
                // matrices (stored rows = tokens): (tok 0-7, d0..+7), (tok 0-7, d0+8..), (tok 8-15, d0..), (tok 8-15, d0+8..)
                const int row = ri + 8 * (mi >> 1);
                const int col = mt * 16 + 8 * (mi & 1);
                ldmatrix_x4_trans(tile_addr(vtile, row, col), a0, a1, a2, a3);
            }
            if constexpr (PARTIAL) { a0 &= mask01; a1 &= mask01; a2 &= mask23; a3 &= mask23; }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                if constexpr (H)
                    mma_f16_16816(o[nt][mt][0], o[nt][mt][1], o[nt][mt][2], o[nt][mt][3], a0, a1, a2, a3,
                                  pb[nt][0], pb[nt][1]);
                else
                    mma_bf16_16816(o[nt][mt][0], o[nt][mt][1], o[nt][mt][2], o[nt][mt][3], a0, a1, a2, a3,
                                   pb[nt][0], pb[nt][1]);
            }
        }
    }

    __device__ __forceinline__ void store_partial(float *mO, float *mM, float *mL, int w, int lane, int stride,
                                                  int GPn, int g) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float lsum = l[nt][c];
                lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
                lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
                lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
                const int head = nt * 8 + 2 * (lane & 3) + c;
                if (head < g) {
                    if (lane < 4) { mM[w * GPn + head] = m[nt][c]; mL[w * GPn + head] = lsum; }
                    float *row = mO + (w * GPn + head) * stride;
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        row[mt * 16 + (lane >> 2)] = o[nt][mt][c];
                        row[mt * 16 + (lane >> 2) + 8] = o[nt][mt][c + 2];
                    }
                }
            }
        }
    }
};

// PATH 0: CUDA cores, one query head per kv head (GSIMT = 1); PATH 1: tensor
// cores with query heads padded to GPAD in {4, 8, 16} (n-tiles of 8: GPAD/8
// rounded up).
// CTAs per SM the register budget must allow: the FP8 tensor-core instances
// with up to 8 padded heads take 44 KB of shared memory, so four CTAs fit
// and the registers must not cut that to three.
constexpr int decode_min_ctas(int PATH, int GPAD, bool KV8) { return (KV8 && PATH == 1 && GPAD <= 8) ? 4 : 1; }

template <int D, int PATH, int GSIMT, int GPAD, int NS, bool KV8 = false>
__global__ void __launch_bounds__(kDecodeThreads, decode_min_ctas(PATH, GPAD, KV8))
    paged_decode_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                        const DecodeParams p) {
    constexpr int W = kConsumerWarps;
    static_assert(PATH != 0 || GSIMT == 1, "the CUDA-core path serves one query head per kv head");
    constexpr int GP = PATH == 0 ? GSIMT : GPAD;
    constexpr int NT = (GPAD + 7) / 8;
    static_assert(!KV8 || D == 128, "FP8 stage tiles are 128-byte rows (head dim 128)");
    using L = DecodeSmem<D, GP, NS, KV8>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-B alignment: the 128-byte swizzle pattern repeats every 1 KB.
    // Everything below indexes the shared array itself, so accesses stay in
    // the shared window (ld.shared / st.shared, not generic loads).
    // The dynamic window starts 1 KB-aligned when the kernel has no static
    // shared variables (none here); the allocation has no slack for
    // realignment, so a misaligned base is reported and the CTA does nothing.
    if ((smem_u32(smem_raw) & 1023u) != 0) {
        if (threadIdx.x == 0) raise_error(PKV_DEVERR_LAYOUT);
        return;
    }
    uint8_t *smem = smem_raw;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::oBars);
    uint64_t *empty = full + NS;
    uint64_t *qfull = empty + NS;
    uint64_t *qempty = qfull + 2;
    uint64_t *mfull = qempty + 2;
    uint64_t *mempty = mfull + 1;
    StageInfo *info = reinterpret_cast<StageInfo *>(smem + L::oInfo);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::oAbort);
    int *grp_arrive = reinterpret_cast<int *>(smem + L::oAbort) + 1;  // warps done with a partition group
    const uint32_t tiles = smem_u32(smem + L::oTiles);
    __nv_bfloat16 *qbuf = reinterpret_cast<__nv_bfloat16 *>(smem + L::oQ);
    float *mO = reinterpret_cast<float *>(smem + L::oMergeO);
    float *mM = reinterpret_cast<float *>(smem + L::oMergeM);
    float *mL = reinterpret_cast<float *>(smem + L::oMergeL);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&qfull[i], 1); mbar_init(&qempty[i], W); }
        mbar_init(mfull, W);
        mbar_init(mempty, W);
        *abort_flag = 0;
        *grp_arrive = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
    }
    __syncthreads();
    // Everything below reads data written by earlier kernels on the stream.
    grid_dependency_wait();

    if (warp == W) {
        // ------------------------------------------------------ producer --
        // Items are claimed from a global counter (dynamic load balance).  The
        // next item's claim, entry, context length, first 32 table entries
        // and query tile are fetched while the current item streams, so the
        // ring does not drain at item boundaries.
        const int n_items = *reinterpret_cast<volatile int32_t *>(p.num_entries) * p.Hkv;
        uint32_t gc = 0;
        bool ok = true;
        // entry -> item geometry; n_raw is the sequence's context length as loaded
        auto describe = [&](int it, int2 sp, int n_raw) {
            ItemMeta m;
            const int e = it / p.Hkv;
            m.h = it - e * p.Hkv;
            m.s = sp.x;
            m.grp = (sp.y & kGroupFlag) ? 1 : 0;
            m.part = sp.y & ~kGroupFlag;
            m.n = clamp_context(p, n_raw, false);
            m.nparts = (m.n + p.PT - 1) / p.PT;
            if (m.grp) {
                m.npad = kConsumerWarps * (p.PT / kStageTok);
            } else {
                const int t0 = m.part * p.PT;
                const int nst = (min(m.n, t0 + p.PT) - t0 + kStageTok - 1) / kStageTok;
                m.npad = (nst + W - 1) / W * W;
            }
            return m;
        };
        // table entry of stage K of the item whose entry is sp (lane-parallel):
        // loaded whenever the index lies inside the row, checked only when the
        // stage holds tokens
        auto table_entry = [&](int2 sp, int K) {
            ItemMeta m;
            m.grp = (sp.y & kGroupFlag) ? 1 : 0;
            m.part = sp.y & ~kGroupFlag;
            const int idx = m.stage_token(K, p.PT) / p.bs;
            return idx < p.MBS ? __ldg(p.block_tables + (size_t)sp.x * p.MBS + idx) : -1;
        };
        int q_last = -1;  // ord of the last query tile load issued
        auto load_q = [&](int it, int2 sp, int ord) -> bool {
            bool r = true;
            if (lane == 0) {
                const int qb = ord & 1;
                r = wait_or_abort(&qempty[qb], ((ord >> 1) & 1) ^ 1, abort_flag);
                if (r) {
                    const int h = it - (it / p.Hkv) * p.Hkv;
                    const uint32_t bytes = (uint32_t)(p.g * D * 2);
                    mbar_arrive_expect_tx(&qfull[qb], bytes);
                    bulk_load(qbuf + qb * (L::kQBuf / 2), p.q + ((size_t)sp.x * p.Hq + (size_t)h * p.g) * D, bytes,
                              &qfull[qb]);
                    q_last = ord;
                }
            }
            return __shfl_sync(0xffffffffu, r, 0);
        };

        int claimed = 0;
        if (lane == 0) claimed = atomicAdd(p.work_counter, 1);
        int it = __shfl_sync(0xffffffffu, claimed, 0);
        int2 sp = make_int2(0, 0);
        int n_raw = 0, blk_first = -1;
        if (it < n_items) {
            sp = p.entries[it / p.Hkv];
            n_raw = __ldg(p.context_lens + sp.x);
            blk_first = table_entry(sp, lane);
            ok = load_q(it, sp, 0);
        }
        if (lane == 0) claimed = atomicAdd(p.work_counter, 1);  // the next item, one ahead
        for (int ord = 0; it < n_items && ok; ++ord) {
            const ItemMeta cur = describe(it, sp, n_raw);
            // The next item's fetch chain, one step per pass (each step uses
            // what the previous one loaded): claim -> entry -> context length,
            // table entries and query tile.
            int nxt = n_items, pf = 0, n_next = 0, blk_next = -1;
            int2 sp_next = make_int2(0, 0);
            auto prefetch_step = [&]() {
                if (pf == 0) {
                    nxt = __shfl_sync(0xffffffffu, claimed, 0);
                    if (nxt < n_items) sp_next = p.entries[nxt / p.Hkv];
                } else if (nxt < n_items) {
                    n_next = __ldg(p.context_lens + sp_next.x);
                    blk_next = table_entry(sp_next, lane);
                    ok = load_q(nxt, sp_next, ord + 1) && ok;
                }
                ++pf;
            };
            // Stages go out in groups of W, one per consumer warp: lane j < W
            // issues stage k0 + j into slot (gc + j) % NS, so one pass of the
            // warp issues W stages (waits, descriptors and TMA in lockstep).
            // Per 32 stages, lane l works out stage (k0 & ~31) + l once: its
            // valid tokens and its TMA row, from the table entry loaded a
            // chunk earlier; the issuing lanes take them by shuffle.
            int blk_chunk = blk_first, row_reg = 0, valid_reg = 0;
            for (int k0 = 0; k0 < cur.npad && ok; k0 += W) {
                if ((k0 & 31) == 0) {
                    const int K = k0 + lane;
                    valid_reg = K < cur.npad ? cur.stage_valid(K, p.PT) : 0;
                    row_reg = p.pool_rows;  // an invalid id reads the zero fill
                    if (valid_reg > 0) {
                        if (blk_chunk < 0 || blk_chunk >= p.NB) raise_error(PKV_DEVERR_BLOCK);
                        else row_reg = (blk_chunk * p.Hkv + cur.h) * p.bs + cur.stage_token(K, p.PT) % p.bs;
                    }
                    blk_chunk = k0 + 32 < cur.npad ? table_entry(sp, K + 32) : -1;  // the next chunk's
                }
                const int src = (k0 + lane) & 31;
                const int row = __shfl_sync(0xffffffffu, row_reg, src);
                const int valid = __shfl_sync(0xffffffffu, valid_reg, src);
                bool lane_ok = true;
                if (lane < W) {
                    const uint32_t g = gc + lane;
                    const uint32_t slot = g % NS;
                    lane_ok = wait_slot(&empty[slot], ((g / NS) & 1) ^ 1, abort_flag);
                    if (lane_ok) {
                        StageInfo si;
                        si.s = cur.s; si.h = cur.h; si.part = cur.part | (cur.grp ? kGroupFlag : 0);
                        si.nparts = cur.nparts; si.k = k0 + lane; si.npad = cur.npad; si.valid = valid; si.ord = ord;
                        info[slot] = si;
                        if (valid > 0) {
                            const uint32_t kt = tiles + slot * L::kStage;
                            mbar_arrive_expect_tx(&full[slot], (uint32_t)L::kStage);
#pragma unroll
                            for (int hf = 0; hf < L::kBoxes; ++hf) {
                                const int x = hf * (128 / L::kElem);  // box column in elements
                                tma_load_2d_u32(kt + hf * L::kHalfTile, &tmap_k, &full[slot], x, row);
                                tma_load_2d_u32(kt + L::kTile + hf * L::kHalfTile, &tmap_v, &full[slot], x, row);
                            }
                        } else {
                            mbar_arrive(&full[slot]);
                        }
                    }
                }
                ok = __all_sync(0xffffffffu, lane_ok) && ok;
                gc += W;
                if (pf < 2) prefetch_step();
            }
            while (ok && pf < 2) prefetch_step();  // a short item: finish the chain here
            if (lane == 0) claimed = atomicAdd(p.work_counter, 1);  // the item after next
            it = nxt;
            sp = sp_next;
            n_raw = n_next;
            blk_first = blk_next;
        }
        // end-of-stream marker for every consumer warp
        if (lane == 0) {
            for (int w = 0; w < W && ok; ++w) {
                const uint32_t slot = gc % NS;
                ok = wait_or_abort(&empty[slot], ((gc / NS) & 1) ^ 1, abort_flag);
                if (ok) {
                    info[slot].ord = -1;
                    mbar_arrive(&full[slot]);
                }
                ++gc;
            }
            // Drain: every TMA and bulk copy this CTA issued must have landed
            // before exit (the last two query tiles included).  In a normal run
            // the consumers already waited for all of them.
            if (!ok) {
                const uint32_t issued = gc;
                for (uint32_t c = (issued > (uint32_t)NS ? issued - NS : 0); c < issued; ++c)
                    mbar_wait_bounded(&full[c % NS], (c / NS) & 1, kWaitLimitNs);
                for (int o = max(0, q_last - 1); o <= q_last; ++o)
                    mbar_wait_bounded(&qfull[o & 1], (o >> 1) & 1, kWaitLimitNs);
            }
        }
        grid_launch_dependents();
    } else {
        // ------------------------------------------------------ consumer --
        const int w = warp;
        uint32_t gc = w;
        uint32_t mc = 0;   // merges done (each completes one phase of mempty)
        uint32_t mfc = 0;  // merges of single partitions (each completes one phase of mfull)
        float scale_log2 = p.scale_log2;
        SimtState<D, KV8> st0;
        MmaState<D, (PATH == 1 ? NT : 1), KV8> st1;
        while (true) {
            const uint32_t slot = gc % NS;
            if (!wait_or_abort(&full[slot], (gc / NS) & 1, abort_flag)) break;
            const StageInfo si = info[slot];
            if (si.ord < 0) break;
            if (si.k == w) {
                // first stage of this item for this warp: fresh state and q
                const int qb = si.ord & 1;
                if (!wait_or_abort(&qfull[qb], (si.ord >> 1) & 1, abort_flag)) break;
                const __nv_bfloat16 *qs = qbuf + qb * (L::kQBuf / 2);
                if constexpr (PATH == 0) {
                    st0.reset();
                    st0.load_q(qs, lane, KV8 ? scale_log2 * __ldg(p.k_scale + si.h) : scale_log2);
                } else {
                    st1.reset();
                    st1.load_q(qs, lane, p.g);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&qempty[qb]);
            }
            if (si.valid > 0) {
                const uint32_t kt = tiles + slot * L::kStage;
                const bool partial = si.valid < kStageTok;  // warp-uniform
                if constexpr (PATH == 0) {
                    if (partial) st0.template stage<true>(kt, kt + L::kTile, si.valid, lane);
                    else st0.template stage<false>(kt, kt + L::kTile, si.valid, lane);
                } else {
                    const float sl = KV8 ? scale_log2 * __ldg(p.k_scale + si.h) : scale_log2;
                    if (partial) st1.template stage<true>(kt, kt + L::kTile, si.valid, lane, sl);
                    else st1.template stage<false>(kt, kt + L::kTile, si.valid, lane, sl);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
            gc += W;
            const bool grp = (si.part & kGroupFlag) != 0;
            if (si.k + W >= si.npad) {
                // this warp's last stage of the item: its partial (m, l, acc)
                // goes to its merge buffer once the previous merge has read them
                if (!wait_or_abort(mempty, (mc & 1) ^ 1, abort_flag)) break;
                if constexpr (PATH == 0) st0.store_partial(mO, mM, mL, w, lane, L::kMergeStride);
                else st1.store_partial(mO, mM, mL, w, lane, L::kMergeStride, GP, p.g);
                __syncwarp();
                const int g = p.g;
                const size_t unit_head0 = (size_t)si.s * p.Hq + (size_t)si.h * g;
                const int part = si.part & ~kGroupFlag;
                // merged result of heads j0, j0 + step, ...: out (a single
                // partition sequence) or the split-K record `rec`
                auto combine = [&](int j0, int step, int rec) {
                    for (int j = j0; j < g; j += step) {
                        float M = PKV_NEG_INF;
#pragma unroll
                        for (int u = 0; u < W; ++u) M = fmaxf(M, mM[u * GP + j]);
                        float f[W], Lsum = 0.f;
#pragma unroll
                        for (int u = 0; u < W; ++u) {
                            const float mu = mM[u * GP + j];
                            f[u] = mu == PKV_NEG_INF ? 0.f : exp2f(mu - M);
                            Lsum = fmaf(mL[u * GP + j], f[u], Lsum);
                        }
                        float invL = Lsum > 0.f ? 1.f / Lsum : 0.f;
                        if constexpr (KV8) invL *= __ldg(p.v_scale + si.h);
#pragma unroll
                        for (int i = 0; i < D / 32; ++i) {
                            const int d = lane + 32 * i;
                            float O = 0.f;
#pragma unroll
                            for (int u = 0; u < W; ++u) O = fmaf(mO[(u * GP + j) * L::kMergeStride + d], f[u], O);
                            if (si.nparts == 1) {
                                p.out[(unit_head0 + j) * D + d] = __float2bfloat16_rn(O * invL);
                            } else {
                                const size_t pi = (unit_head0 + j) * p.maxP + rec;
                                p.part_acc[pi * D + d] = O;
                                if (d == 0) p.part_ml[pi] = make_float2(M, Lsum);
                            }
                        }
                    }
                };
                if (grp) {
                    // partition group: warp u walked partition part + u alone.
                    // The last warp to get here merges the W partitions into
                    // the group's record (an fp32 log-sum-exp merge); the
                    // others go on with the next item at once.
                    int last = 0;
                    if (lane == 0) {
                        __threadfence_block();
                        last = atomicAdd(grp_arrive, 1) == W - 1;
                    }
                    if (__shfl_sync(0xffffffffu, last, 0)) {
                        __threadfence_block();
                        combine(0, 1, part / W);
                        __syncwarp();
                        if (lane == 0) {
                            *grp_arrive = 0;
                            mbar_arrive_count(mempty, W);
                        }
                    }
                } else {
                    // the W warps shared the partition's stages: merge
                    // together, warp w taking heads w, w + W, ...; lanes on
                    // consecutive words (no bank conflicts)
                    if (lane == 0) mbar_arrive(mfull);
                    if (!wait_or_abort(mfull, mfc & 1, abort_flag)) break;
                    ++mfc;
                    combine(w, W, record_index(p, si.nparts, part));
                    __syncwarp();
                    if (lane == 0) mbar_arrive(mempty);
                }
                ++mc;
            }
        }
        grid_launch_dependents();
    }
}

// --------------------------------------------------------------- reduce ----
// Log-sum-exp merge of the split-K records of every (s, hq) with more than
// one partition (a record per partition group, then one per single
// partition): M = max_p m_p, L = sum_p l_p 2^(m_p - M),
// out = sum_p acc_p 2^(m_p - M) / L.  One CTA per (s, hq); warp w takes
// records w, w + 4, ...; lanes own D/32 consecutive elements.
template <int D>
__global__ void __launch_bounds__(kReduceWarps * 32) splitk_reduce_kernel(const DecodeParams p) {
    constexpr int EPL = D / 32;
    __shared__ float s_o[kReduceWarps][D];
    __shared__ float s_l[kReduceWarps];
    grid_dependency_wait();
    const int unit = blockIdx.x;  // s * Hq + hq
    const int s = unit / p.Hq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = clamped_context(p, s, false);
    const int parts = (n + p.PT - 1) / p.PT;
    if (parts <= 1) return;  // written directly by the attention kernel
    const int P = parts - (kConsumerWarps - 1) * group_count(p, parts);  // records
    const float2 *ml = p.part_ml + (size_t)unit * p.maxP;
    float M = PKV_NEG_INF;
    for (int i = lane; i < P; i += 32) M = fmaxf(M, ml[i].x);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float acc[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
    float lsum = 0.f;
    const float *base = p.part_acc + (size_t)unit * p.maxP * D + lane * EPL;
#pragma unroll 4
    for (int i = warp; i < P; i += kReduceWarps) {
        const float2 mli = ml[i];
        const float f = exp2f(mli.x - M);
        lsum = fmaf(mli.y, f, lsum);
        if constexpr (EPL == 4) {
            const float4 a = *reinterpret_cast<const float4 *>(base + (size_t)i * D);
            acc[0] = fmaf(a.x, f, acc[0]); acc[1] = fmaf(a.y, f, acc[1]);
            acc[2] = fmaf(a.z, f, acc[2]); acc[3] = fmaf(a.w, f, acc[3]);
        } else {
            const float2 a = *reinterpret_cast<const float2 *>(base + (size_t)i * D);
            acc[0] = fmaf(a.x, f, acc[0]); acc[1] = fmaf(a.y, f, acc[1]);
        }
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) s_o[warp][lane * EPL + e] = acc[e];
    if (lane == 0) s_l[warp] = lsum;
    __syncthreads();
    if (warp == 0) {
        float Lt = 0.f;
#pragma unroll
        for (int u = 0; u < kReduceWarps; ++u) Lt += s_l[u];
        float inv = Lt > 0.f ? 1.f / Lt : 0.f;
        if (p.v_scale) inv *= __ldg(p.v_scale + (unit % p.Hq) / p.g);  // FP8 pool: the kv head's V scale
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            float o = 0.f;
#pragma unroll
            for (int u = 0; u < kReduceWarps; ++u) o += s_o[u][lane * EPL + e];
            p.out[(size_t)unit * D + lane * EPL + e] = __float2bfloat16_rn(o * inv);
        }
    }
}

// ------------------------------------------------------------- self-test --
// Exercises the bounded waits of the attention kernel without a fault: warp 0
// waits on a barrier that nothing arrives on and gives up after limit_ns
// (setting PKV_DEVERR_TIMEOUT and the CTA's abort flag); warp 1 waits on
// another such barrier with the 2 s default limit and must return early
// because of the abort flag.  out[0] = warp 0's result, out[1] = warp 1's,
// out[2] = warp 1's wait time in microseconds.
__global__ void __launch_bounds__(64) selftest_wait_kernel(uint64_t limit_ns, int32_t *out) {
    __shared__ uint64_t bars[2];
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        if (warp == 0) {
            out[0] = wait_or_abort(&bars[0], 0, &abort_flag, limit_ns) ? 1 : 0;
        } else {
            const uint64_t t0 = global_timer_ns();
            out[1] = wait_or_abort(&bars[1], 0, &abort_flag) ? 1 : 0;
            out[2] = (int32_t)((global_timer_ns() - t0) / 1000);
        }
    }
}

}  // namespace pkv
