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
// Work decomposition: an item is (sequence, kv head h, query tile of QT tokens)
// with QT = 64 / g, so one item holds 64 query rows = (token, head of the GQA
// group) pairs.  The same producer warp as in decode streams the 16-token K/V
// stages of positions [0, last query position] into the ring; unlike decode,
// every consumer warp reads every stage: warp w owns rows 16w .. 16w+15 and
// computes S = Q K^T and O += P V with mma.sync m16n8k16 (bf16 in, fp32
// accumulate).  P is used straight from the S accumulator fragments as the A
// operand of the PV product.  Online softmax per row with the lazy rescale of
// decode; no split-K (each item walks its whole causal key range), items are
// claimed dynamically, longest tile of each sequence first.
#pragma once

#include "decode.cuh"

namespace pkv {

constexpr int kPrefillRows = 16 * kConsumerWarps;  // query rows per item

struct PrefillParams {
    const __nv_bfloat16 *q;       // [T][Hq][D]
    __nv_bfloat16 *out;           // [T][Hq][D]
    const int32_t *block_tables;  // [B][MBS]
    const int32_t *context_lens;  // [B]
    const int32_t *query_start;   // [B+1]
    int2 *entries;                // workspace: (seq, query tile)
    int32_t *num_entries;
    int32_t *work_counter;
    int B, Hq, Hkv, g, MBS, bs, NB, max_ctx, max_q, QT, T;
    int pool_rows;
    float scale_log2;
};

struct PrefillStage {
    int s, h, tile, q_len, prefix, q0;  // item: q0 = query_start[s]
    int k, nst, valid, ord;              // stage k of nst; valid keys in it; ord < 0 ends the stream
};

// Query length and cached prefix of sequence s, clamped to what the table, the
// workspace and the context allow (reported once, by the planner).
__device__ __forceinline__ void prefill_lengths(const PrefillParams &p, int s, bool report, int &q_len,
                                                int &prefix) {
    int ctx = __ldg(p.context_lens + s);
    const long long cap = min((long long)p.MBS * p.bs, (long long)p.max_ctx);
    const int q_begin = __ldg(p.query_start + s);
    int ql = __ldg(p.query_start + s + 1) - q_begin;
    bool bad = false;
    if (q_begin < 0 || q_begin > p.T) { bad = true; ql = 0; }
    else if (ql > p.T - q_begin) { bad = true; ql = p.T - q_begin; }
    if (ctx < 0 || ctx > cap) { bad = true; ctx = ctx < 0 ? 0 : (int)cap; }
    if (ql < 0 || ql > p.max_q || ql > ctx) { bad = true; ql = max(0, min(min(ql, p.max_q), ctx)); }
    if (bad && report) raise_error(PKV_DEVERR_CONTEXT);
    q_len = ql;
    prefix = ctx - ql;
}

// Planner: entries (s, tile) sequence-major, each sequence's last (longest)
// tile first; zeroes the work counter.
__global__ void __launch_bounds__(kPlanThreads) plan_prefill_kernel(PrefillParams p) {
    __shared__ int s_off[kPlanThreads + 1];
    __shared__ int s_warp[kPlanThreads / 32];
    __shared__ int s_carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    grid_launch_dependents();
    if (tid == 0) s_carry = 0;
    __syncthreads();
    for (int base = 0; base < p.B; base += kPlanThreads) {
        const int s = base + tid;
        int tiles = 0;
        if (s < p.B) {
            int ql, prefix;
            prefill_lengths(p, s, true, ql, prefix);
            tiles = (ql + p.QT - 1) / p.QT;
        }
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
            p.entries[carry + e] = make_int2(base + lo, n_tiles - 1 - (e - s_off[lo]));
        }
        __syncthreads();
        if (tid == 0) s_carry = carry + chunk_total;
        __syncthreads();
    }
    if (tid == 0) {
        *p.num_entries = s_carry;
        *p.work_counter = 0;
    }
}

template <int D, int NS>
struct PrefillSmem {
    static constexpr int kHalfTile = kStageTok * 64 * 2;
    static constexpr int kTile = kStageTok * D * 2;
    static constexpr int kStage = 2 * kTile;
    static constexpr int oTiles = 0;
    static constexpr int oBars = NS * kStage;
    static constexpr int oInfo = oBars + 2 * NS * 8;
    static constexpr int oAbort = oInfo + NS * (int)sizeof(PrefillStage);
    static constexpr int kBytes = oAbort + 16;
};

template <int D, int NS>
__global__ void __launch_bounds__(kDecodeThreads) paged_prefill_kernel(const __grid_constant__ CUtensorMap tmap_k,
                                                                       const __grid_constant__ CUtensorMap tmap_v,
                                                                       const PrefillParams p) {
    constexpr int W = kConsumerWarps;
    constexpr int KS = D / 16;  // k-steps of Q K^T
    constexpr int NTO = D / 8;  // n-tiles of O
    using L = PrefillSmem<D, NS>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if ((smem_u32(smem_raw) & 1023u) != 0) {
        if (threadIdx.x == 0) raise_error(PKV_DEVERR_LAYOUT);
        return;
    }
    uint8_t *smem = smem_raw;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::oBars);
    uint64_t *empty = full + NS;
    PrefillStage *info = reinterpret_cast<PrefillStage *>(smem + L::oInfo);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::oAbort);
    const uint32_t tiles = smem_u32(smem + L::oTiles);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], W); }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
    }
    __syncthreads();
    grid_dependency_wait();

    if (warp == W) {
        // ------------------------------------------------------ producer --
        const int n_items = *reinterpret_cast<volatile int32_t *>(p.num_entries) * p.Hkv;
        uint32_t gc = 0;
        bool ok = true;
        int claimed = 0;
        if (lane == 0) claimed = atomicAdd(p.work_counter, 1);
        int it = __shfl_sync(0xffffffffu, claimed, 0);
        for (int ord = 0; it < n_items && ok; ++ord) {
            if (lane == 0) claimed = atomicAdd(p.work_counter, 1);
            const int e = it / p.Hkv;
            const int h = it - e * p.Hkv;
            const int2 st = p.entries[e];
            const int s = st.x, tile = st.y;
            int q_len, prefix;
            prefill_lengths(p, s, false, q_len, prefix);
            const int q0 = __ldg(p.query_start + s);
            const int last_tok = min(q_len, (tile + 1) * p.QT) - 1;
            const int n_keys = prefix + last_tok + 1;
            const int nst = (n_keys + kStageTok - 1) / kStageTok;
            int blk_reg = -1;
            // groups of 4 stages, one per producer lane
            for (int k0 = 0; k0 < nst && ok; k0 += 4) {
                if ((k0 & 31) == 0) {
                    const int kk = k0 + lane;
                    int blk = -1;
                    if (kk < nst) {
                        blk = __ldg(p.block_tables + (size_t)s * p.MBS + (kk * kStageTok) / p.bs);
                        if (blk < 0 || blk >= p.NB) {
                            raise_error(PKV_DEVERR_BLOCK);
                            blk = -1;
                        }
                    }
                    blk_reg = blk;
                }
                const int k = k0 + lane;
                const int blk = __shfl_sync(0xffffffffu, blk_reg, k & 31);
                bool lane_ok = true;
                if (lane < 4 && k < nst) {
                    const uint32_t gg = gc + lane;
                    const uint32_t slot = gg % NS;
                    lane_ok = wait_or_abort(&empty[slot], ((gg / NS) & 1) ^ 1, abort_flag);
                    if (lane_ok) {
                        const int tok = k * kStageTok;
                        PrefillStage si;
                        si.s = s; si.h = h; si.tile = tile; si.q_len = q_len; si.prefix = prefix; si.q0 = q0;
                        si.k = k; si.nst = nst; si.valid = min(kStageTok, n_keys - tok); si.ord = ord;
                        info[slot] = si;
                        const int row = blk >= 0 ? (blk * p.Hkv + h) * p.bs + tok % p.bs : p.pool_rows;
                        const uint32_t kt = tiles + slot * L::kStage;
                        mbar_arrive_expect_tx(&full[slot], (uint32_t)L::kStage);
#pragma unroll
                        for (int hf = 0; hf < D / 64; ++hf) {
                            tma_load_2d_u32(kt + hf * L::kHalfTile, &tmap_k, &full[slot], hf * 64, row);
                            tma_load_2d_u32(kt + L::kTile + hf * L::kHalfTile, &tmap_v, &full[slot], hf * 64, row);
                        }
                    }
                }
                ok = __all_sync(0xffffffffu, lane_ok);
                gc += min(4, nst - k0);
            }
            it = __shfl_sync(0xffffffffu, claimed, 0);
        }
        if (lane == 0) {
            if (ok) {
                const uint32_t slot = gc % NS;
                ok = wait_or_abort(&empty[slot], ((gc / NS) & 1) ^ 1, abort_flag);
                if (ok) {
                    info[slot].ord = -1;
                    mbar_arrive(&full[slot]);
                }
                ++gc;
            }
            if (!ok) {
                for (uint32_t c = (gc > (uint32_t)NS ? gc - NS : 0); c < gc; ++c)
                    mbar_wait_bounded(&full[c % NS], (c / NS) & 1, kWaitLimitNs);
            }
        }
        grid_launch_dependents();
        return;
    }

    // ---------------------------------------------------------- consumer --
    // Thread (lane) holds rows r0 = 16w + lane/4 and r1 = r0 + 8 of the item.
    const int w = warp;
    const float scale_log2 = p.scale_log2;
    const int g = p.g;
    uint32_t qa[KS][4];
    float o[NTO][4];
    float m[2], l[2];
    int qpos[2], out_row[2];  // query position and out/q row index ([T][Hq] flattened), -1 = padding row
    const int mi = lane >> 3, ri = lane & 7;
    uint32_t gc = 0;
    while (true) {
        const uint32_t slot = gc % NS;
        if (!wait_or_abort(&full[slot], (gc / NS) & 1, abort_flag)) break;
        const PrefillStage si = info[slot];
        if (si.ord < 0) break;
        if (si.k == 0) {
            // new item: rows, query positions, Q fragments, fresh state
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int r = 16 * w + (lane >> 2) + 8 * i;
                const int tt = r / g, j = r - tt * g;
                const int tok = si.tile * p.QT + tt;
                const bool real = tt < p.QT && tok < si.q_len;
                qpos[i] = real ? si.prefix + tok : si.prefix + min(si.q_len, (si.tile + 1) * p.QT) - 1;
                out_row[i] = real ? (si.q0 + tok) * p.Hq + si.h * g + j : -1;
                m[i] = PKV_NEG_INF;
                l[i] = 0.f;
            }
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                const int c = kk * 16 + 2 * (lane & 3);
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const __nv_bfloat16 *qr = p.q + (size_t)(out_row[i] < 0 ? 0 : out_row[i]) * D;
                    const bool real = out_row[i] >= 0;
                    qa[kk][i] = real ? __ldg(reinterpret_cast<const uint32_t *>(qr + c)) : 0u;
                    qa[kk][2 + i] = real ? __ldg(reinterpret_cast<const uint32_t *>(qr + c + 8)) : 0u;
                }
            }
#pragma unroll
            for (int n = 0; n < NTO; ++n)
#pragma unroll
                for (int c = 0; c < 4; ++c) o[n][c] = 0.f;
        }
        const uint32_t kt = tiles + slot * L::kStage;
        const uint32_t vt = kt + L::kTile;
        // S[16 rows x 16 keys] = Q K^T (two n-tiles of 8 keys)
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            // matrices: (keys 0-7, d0..+7), (keys 0-7, d0+8..), (keys 8-15, d0..), (keys 8-15, d0+8..)
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(tile_addr(kt, ri + 8 * (mi >> 1), kk * 16 + 8 * (mi & 1)), b0, b1, b2, b3);
            mma_bf16_16816(sc[0][0], sc[0][1], sc[0][2], sc[0][3], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
            mma_bf16_16816(sc[1][0], sc[1][1], sc[1][2], sc[1][3], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b2, b3);
        }
        // scale, causal mask (a key is visible iff its position <= the row's)
        const int kbase = si.k * kStageTok;
        float z[2][4];
        bool raise = false;
        float alpha[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float mx = PKV_NEG_INF;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int kpos = kbase + nt * 8 + 2 * (lane & 3) + c;
                    const float v = (kpos <= qpos[i]) ? sc[nt][2 * i + c] * scale_log2 : PKV_NEG_INF;
                    z[nt][2 * i + c] = v;
                    mx = fmaxf(mx, v);
                }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const bool up = mx > m[i] + kRescaleSlack;
            alpha[i] = up ? exp2f(m[i] - mx) : 1.f;
            if (up) m[i] = mx;
            raise |= up;
        }
        float pr[2][4];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float sum = 0.f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    pr[nt][2 * i + c] = exp2f(z[nt][2 * i + c] - m[i]);
                    sum += pr[nt][2 * i + c];
                }
            l[i] = l[i] * alpha[i] + sum;
        }
        if (__any_sync(0xffffffffu, raise)) {
#pragma unroll
            for (int n = 0; n < NTO; ++n) {
                o[n][0] *= alpha[0];
                o[n][1] *= alpha[0];
                o[n][2] *= alpha[1];
                o[n][3] *= alpha[1];
            }
        }
        // P as the A operand (rows x 16 keys): the accumulator layout of the
        // two n-tiles is the m16k16 operand layout.
        const uint32_t pa0 = pack_bf16x2(pr[0][0], pr[0][1]);
        const uint32_t pa1 = pack_bf16x2(pr[0][2], pr[0][3]);
        const uint32_t pa2 = pack_bf16x2(pr[1][0], pr[1][1]);
        const uint32_t pa3 = pack_bf16x2(pr[1][2], pr[1][3]);
        // keys past the context (last stage) must not reach the MMA as NaN
        uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
        if (si.valid < 16) {
            const int j0 = 2 * (lane & 3);
            mlo = (j0 < si.valid ? 0x0000ffffu : 0u) | (j0 + 1 < si.valid ? 0xffff0000u : 0u);
            mhi = (j0 + 8 < si.valid ? 0x0000ffffu : 0u) | (j0 + 9 < si.valid ? 0xffff0000u : 0u);
        }
        // O[16 rows x D] += P V: V fragments by transposed ldmatrix, two d n-tiles per load
#pragma unroll
        for (int jp = 0; jp < NTO / 2; ++jp) {
            // matrices: (keys 0-7, d 16jp..+7), (keys 8-15, same), (keys 0-7, d 16jp+8..), (keys 8-15, same)
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(tile_addr(vt, ri + 8 * (mi & 1), 16 * jp + 8 * (mi >> 1)), b0, b1, b2, b3);
            b0 &= mlo; b1 &= mhi; b2 &= mlo; b3 &= mhi;
            mma_bf16_16816(o[2 * jp][0], o[2 * jp][1], o[2 * jp][2], o[2 * jp][3], pa0, pa1, pa2, pa3, b0, b1);
            mma_bf16_16816(o[2 * jp + 1][0], o[2 * jp + 1][1], o[2 * jp + 1][2], o[2 * jp + 1][3], pa0, pa1, pa2,
                           pa3, b2, b3);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        ++gc;
        if (si.k == si.nst - 1) {
            // item done: normalise and store this warp's rows
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                float lt = l[i];
                lt += __shfl_xor_sync(0xffffffffu, lt, 1);
                lt += __shfl_xor_sync(0xffffffffu, lt, 2);
                const float inv = lt > 0.f ? 1.f / lt : 0.f;
                if (out_row[i] >= 0) {
                    __nv_bfloat16 *orow = p.out + (size_t)out_row[i] * D;
#pragma unroll
                    for (int n = 0; n < NTO; ++n) {
                        const uint32_t v = pack_bf16x2(o[n][2 * i] * inv, o[n][2 * i + 1] * inv);
                        *reinterpret_cast<uint32_t *>(orow + n * 8 + 2 * (lane & 3)) = v;
                    }
                }
            }
        }
    }
    grid_launch_dependents();
}

}  // namespace pkv
