// prefill_tc.cuh -- chunked-prefill paged attention on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// Same operation as paged_prefill_kernel (prefill.cuh): query token i of a
// sequence's new chunk sits at position ctx - q_len + i and attends to positions
// [0, pos] read through the block table (wkbse.com "加速 LLM 推理：深入了解 vllm
// 引擎", section 3.1).  An item is (sequence, kv head, tile of 128 query rows),
// a row being (query token, head of the GQA group).
//
// One CTA per SM, warp-specialised (192 threads):
//   warp 0       producer: the item's Q tile (128 x D bf16) by a 3-D TMA load
//                into a double buffer, and 64-key K/V blocks of the paged cache
//                (4 stages of 16 keys, addressed through the block table) into
//                a ring; all 128-byte swizzled.
//   warp 1       MMA issuer (one thread) and tensor-memory owner:
//                S_j = Q K_j^T  (tcgen05.mma kind::f16, M 128, N 64, K-major
//                smem operands, fp32 into one of two TMEM S buffers), then
//                O += P_j V_j   (A = P_j in TMEM, B = V_j MN-major in smem,
//                N = D), each followed by tcgen05.commit onto an mbarrier.
//   warps 2-5    softmax: thread r owns row r (TMEM lane r).  It loads S_j,
//                applies the causal mask and scale, keeps the row's running
//                max (raised lazily, as in decode) and sum, writes P_j as bf16
//                into TMEM, rescales its O row when the max was raised (after
//                the previous PV product has completed), and at the end of the
//                item normalises O and stores the row.
// S_{j+1} runs on the tensor cores while the softmax works on S_j.
#pragma once

#include "prefill.cuh"

namespace pkv {

constexpr int kTcRows = 128;          // M: query rows per item
constexpr int kTcKeys = 64;           // N: keys per block (4 stages of 16)
constexpr int kTcThreads = 6 * 32;
constexpr uint32_t kTmemS = 0;        // two S buffers: columns [0, 64) and [64, 128)
constexpr uint32_t kTmemP = 128;      // two P buffers (bf16 pairs): [128, 160) and [160, 192)

// O follows the P buffers; the allocation is the next power of two (head dim
// 64 takes half of tensor memory, so two CTAs may share an SM).
template <int D>
struct TcTmem {
    static constexpr uint32_t kO = D == 64 ? 192 : 256;
    static constexpr uint32_t kCols = D == 64 ? 256 : 512;
};

struct TcItem {
    int s, h, tile, q_len, prefix, q0, n_keys, n_blocks;
};

template <int D, int NKV>
struct TcSmem {
    static constexpr int kHalves = D / 64;
    static constexpr int kQHalf = kTcRows * 128;          // 16 KB: 128 rows x 64 columns
    static constexpr int kQBuf = kHalves * kQHalf;
    static constexpr int kKVHalf = kTcKeys * 128;         // 8 KB: 64 keys x 64 columns
    static constexpr int kSlot = 2 * kHalves * kKVHalf;   // K halves then V halves
    static constexpr int oQ = 0;
    static constexpr int oKV = 2 * kQBuf;
    static constexpr int oBars = oKV + NKV * kSlot;
    // full[NKV], empty[NKV], qfull[2], qempty[2], sfull[2], sfree[2], pfull[2], odone, drain
    static constexpr int kNumBars = 2 * NKV + 12;
    static constexpr int oItem = oBars + kNumBars * 8;
    static constexpr int oTmemSlot = oItem + 2 * (int)sizeof(TcItem);
    static constexpr int oAbort = oTmemSlot + 16;
    static constexpr int kBytes = oAbort + 16;
};

// ------------------------------------------------------------ tcgen05 PTX --

// Shared-memory matrix descriptor, 128-byte swizzle (sm100 layout type 2),
// version 1; addresses and offsets in bytes (16-byte units in the fields).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulate, M x N.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn_major ? (1u << 16) : 0u) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 consecutive 32-bit TMEM columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
        "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
        "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::
            "r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// 3-D tiled TMA load (the Q tile: columns x heads x tokens).  No multicast.
__device__ __forceinline__ void tma_load_3d_u32(uint32_t smem_dst, const CUtensorMap *map, uint64_t *bar, int c0,
                                                int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// Item geometry shared by the three roles.
__device__ __forceinline__ TcItem tc_item(const PrefillParams &p, int it) {
    TcItem t;
    const int e = it / p.Hkv;
    t.h = it - e * p.Hkv;
    const int2 st = p.entries[e];
    t.s = st.x;
    t.tile = st.y;
    prefill_lengths(p, t.s, false, t.q_len, t.prefix);
    t.q0 = __ldg(p.query_start + t.s);
    const int last_tok = min(t.q_len, (t.tile + 1) * p.QT) - 1;
    t.n_keys = t.prefix + last_tok + 1;
    t.n_blocks = (t.n_keys + kTcKeys - 1) / kTcKeys;
    return t;
}

template <int D, int NKV>
__global__ void __launch_bounds__(kTcThreads, 1) paged_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                                                                         const __grid_constant__ CUtensorMap tmap_v,
                                                                         const __grid_constant__ CUtensorMap tmap_q,
                                                                         const PrefillParams p) {
    using L = TcSmem<D, NKV>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if ((smem_u32(smem_raw) & 1023u) != 0) {
        if (threadIdx.x == 0) raise_error(PKV_DEVERR_LAYOUT);
        return;
    }
    uint8_t *smem = smem_raw;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::oBars);
    uint64_t *full = bars, *empty = bars + NKV;
    uint64_t *qfull = bars + 2 * NKV, *qempty = qfull + 2;
    uint64_t *sfull = qempty + 2, *sfree = sfull + 2, *pfull = sfree + 2, *odone = pfull + 2, *drain = odone + 1;
    constexpr uint32_t kTmemO = TcTmem<D>::kO;
    constexpr uint32_t kTmemCols = TcTmem<D>::kCols;
    TcItem *items = reinterpret_cast<TcItem *>(smem + L::oItem);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::oTmemSlot);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::oAbort);
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NKV; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&qfull[i], 1);
            // released by the MMA's commit (Q read) and by every softmax
            // thread once it has taken the item description
            mbar_init(&qempty[i], 1 + kTcRows);
            mbar_init(&sfull[i], 1);
            mbar_init(&sfree[i], kTcRows);
            mbar_init(&pfull[i], kTcRows);
        }
        mbar_init(odone, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
        tma_prefetch_desc(&tmap_q);
    }
    // Q buffers start as zeros: rows a tile does not fill stay finite.
    for (int i = threadIdx.x; i < 2 * L::kQBuf / 16; i += kTcThreads)
        reinterpret_cast<uint4 *>(smem + L::oQ)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    grid_dependency_wait();
    const int n_items = *reinterpret_cast<volatile int32_t *>(p.num_entries) * p.Hkv;

    if (warp == 0) {
        // ------------------------------------------------------ producer --
        uint32_t gs = 0;  // KV slots filled
        int q_issued = -1;  // ord of the last Q tile load
        bool ok = true;
        int claimed = 0;
        if (lane == 0) claimed = atomicAdd(p.work_counter, 1);
        int it = __shfl_sync(0xffffffffu, claimed, 0);
        for (int ord = 0; ok; ++ord) {
            const int qb = ord & 1;
            if (lane == 0) {
                ok = wait_or_abort(&qempty[qb], ((ord >> 1) & 1) ^ 1, abort_flag);
                if (ok) {
                    TcItem t;
                    if (it < n_items) t = tc_item(p, it);
                    else t.n_blocks = -1;  // end of stream
                    items[qb] = t;
                    if (it < n_items) {
                        q_issued = ord;
                        mbar_arrive_expect_tx(&qfull[qb], (uint32_t)(L::kHalves * 128 * p.QT * p.g));
                        const uint32_t qdst = sbase + L::oQ + qb * L::kQBuf;
#pragma unroll
                        for (int hf = 0; hf < L::kHalves; ++hf)
                            tma_load_3d_u32(qdst + hf * L::kQHalf, &tmap_q, &qfull[qb], hf * 64, t.h * p.g,
                                            t.q0 + t.tile * p.QT);
                    } else {
                        mbar_arrive(&qfull[qb]);
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (it >= n_items || !ok) break;
            if (lane == 0) claimed = atomicAdd(p.work_counter, 1);
            const TcItem t = tc_item(p, it);
            for (int j = 0; j < t.n_blocks && ok; ++j) {
                const uint32_t slot = gs % NKV;
                if (lane == 0) {
                    ok = wait_or_abort(&empty[slot], ((gs / NKV) & 1) ^ 1, abort_flag);
                    if (ok) mbar_arrive_expect_tx(&full[slot], (uint32_t)L::kSlot);
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                __syncwarp();
                if (ok && lane < 4) {
                    // lane = stage of 16 keys within the block; stages past the
                    // keys read rows beyond the pool (zero fill)
                    const int tok = j * kTcKeys + lane * kStageTok;
                    int row = p.pool_rows;
                    if (tok < t.n_keys) {
                        const int blk = __ldg(p.block_tables + (size_t)t.s * p.MBS + tok / p.bs);
                        if (blk >= 0 && blk < p.NB) row = (blk * p.Hkv + t.h) * p.bs + tok % p.bs;
                        else raise_error(PKV_DEVERR_BLOCK);
                    }
                    const uint32_t kdst = sbase + L::oKV + slot * L::kSlot + lane * (kStageTok * 128);
#pragma unroll
                    for (int hf = 0; hf < L::kHalves; ++hf) {
                        tma_load_2d_u32(kdst + hf * L::kKVHalf, &tmap_k, &full[slot], hf * 64, row);
                        tma_load_2d_u32(kdst + (L::kHalves + hf) * L::kKVHalf, &tmap_v, &full[slot], hf * 64, row);
                    }
                }
                if (ok) ++gs;
            }
            it = __shfl_sync(0xffffffffu, claimed, 0);
        }
        // After an abort, loads this CTA issued must land before it exits.
        if (lane == 0 && *abort_flag) {
            for (uint32_t c = (gs > (uint32_t)NKV ? gs - NKV : 0); c < gs; ++c)
                mbar_wait_bounded(&full[c % NKV], (c / NKV) & 1, kWaitLimitNs);
            if (q_issued >= 0) mbar_wait_bounded(&qfull[q_issued & 1], (q_issued >> 1) & 1, kWaitLimitNs);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA --
        uint32_t gs = 0, gb = 0;  // KV slots consumed, blocks processed
        bool ok = true;
        const uint32_t idesc_s = umma_idesc_bf16(kTcRows, kTcKeys, false);
        const uint32_t idesc_o = umma_idesc_bf16(kTcRows, D, true);
        for (int ord = 0; ok; ++ord) {
            const int qb = ord & 1;
            ok = wait_or_abort(&qfull[qb], (ord >> 1) & 1, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            const int nb = items[qb].n_blocks;
            if (nb < 0) break;
            tc_fence_after();
            const uint32_t qaddr = sbase + L::oQ + qb * L::kQBuf;
            for (int j = 0; j <= nb && ok; ++j) {
                if (j < nb) {
                    // S_j = Q K_j^T into S buffer gb % 2
                    const uint32_t slot = gs % NKV;
                    const uint32_t sb = gb & 1;
                    if (lane == 0) {
                        ok = wait_or_abort(&full[slot], (gs / NKV) & 1, abort_flag) &&
                             wait_or_abort(&sfree[sb], ((gb >> 1) & 1) ^ 1, abort_flag);
                        if (ok) {
                            tc_fence_after();
                            const uint32_t kaddr = sbase + L::oKV + slot * L::kSlot;
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint32_t off = (kk >> 2) * L::kQHalf + (kk & 3) * 32;
                                const uint32_t koff = (kk >> 2) * L::kKVHalf + (kk & 3) * 32;
                                umma_ss(tmem + kTmemS + sb * kTcKeys, umma_desc_sw128(qaddr + off, 16, 1024),
                                        umma_desc_sw128(kaddr + koff, 16, 1024), idesc_s, kk > 0);
                            }
                            umma_commit(&sfull[sb]);
                            if (j == nb - 1) umma_commit(&qempty[qb]);  // Q no longer read
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                }
                if (j > 0 && ok) {
                    // O += P_{j-1} V_{j-1}
                    const uint32_t pg = gb - 1;
                    const uint32_t pb = pg & 1;
                    const uint32_t pslot = (gs - 1) % NKV;
                    if (lane == 0) {
                        ok = wait_or_abort(&pfull[pb], (pg >> 1) & 1, abort_flag);
                        if (ok) {
                            tc_fence_after();
                            const uint32_t vaddr = sbase + L::oKV + pslot * L::kSlot + L::kHalves * L::kKVHalf;
#pragma unroll
                            for (int kk = 0; kk < kTcKeys / 16; ++kk)
                                umma_ts(tmem + kTmemO, tmem + kTmemP + pb * (kTcKeys / 2) + kk * 8,
                                        umma_desc_sw128(vaddr + kk * 16 * 128, L::kKVHalf, 1024), idesc_o,
                                        (j > 1 || kk > 0) ? 1u : 0u);
                            umma_commit(odone);
                            umma_commit(&empty[pslot]);
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                }
                if (j < nb) { ++gs; ++gb; }
            }
        }
        // every MMA this thread issued has completed before tensor memory is freed
        if (lane == 0) {
            umma_commit(drain);
            mbar_wait_bounded(drain, 0, kWaitLimitNs);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ softmax --
        const int quarter = warp & 3;          // TMEM lane quarter of this warp
        const int r = quarter * 32 + lane;     // row = TMEM lane
        const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
        const float scale_log2 = p.scale_log2;
        uint32_t gb = 0;
        bool ok = true;
        for (int ord = 0; ok; ++ord) {
            const int qb = ord & 1;
            ok = __all_sync(0xffffffffu, wait_or_abort(&qfull[qb], (ord >> 1) & 1, abort_flag));
            if (!ok) break;
            const TcItem t = items[qb];
            mbar_arrive(&qempty[qb]);
            if (t.n_blocks < 0) break;
            const int tt = r / p.g, jh = r - tt * p.g;
            const int tok = t.tile * p.QT + tt;
            const bool real = tt < p.QT && tok < t.q_len;
            const int qpos = real ? t.prefix + tok : t.n_keys - 1;
            float m = PKV_NEG_INF, l = 0.f;
            for (int j = 0; j < t.n_blocks && ok; ++j, ++gb) {
                const uint32_t sb = gb & 1;
                ok = __all_sync(0xffffffffu, wait_or_abort(&sfull[sb], (gb >> 1) & 1, abort_flag));
                if (!ok) break;
                tc_fence_after();
                uint32_t sv[2][32];
                tmem_ld32(lane_addr + kTmemS + sb * kTcKeys, sv[0]);
                tmem_ld32(lane_addr + kTmemS + sb * kTcKeys + 32, sv[1]);
                tc_wait_ld();
                tc_fence_before();
                mbar_arrive(&sfree[sb]);
                // causal mask and scale; lazy running max
                const int kbase = j * kTcKeys;
                float mx = PKV_NEG_INF;
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int kpos = kbase + h2 * 32 + c;
                        const float z = kpos <= qpos ? __uint_as_float(sv[h2][c]) * scale_log2 : PKV_NEG_INF;
                        sv[h2][c] = __float_as_uint(z);
                        mx = fmaxf(mx, z);
                    }
                const bool up = mx > m + kRescaleSlack;
                const float alpha = up ? exp2f(m - mx) : 1.f;
                if (up) m = mx;
                float sum = 0.f;
                uint32_t pk[2][16];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const float p0 = exp2f(__uint_as_float(sv[h2][2 * c]) - m);
                        const float p1 = exp2f(__uint_as_float(sv[h2][2 * c + 1]) - m);
                        sum += p0 + p1;
                        pk[h2][c] = pack_bf16x2(p0, p1);
                    }
                l = l * alpha + sum;
                tmem_st16(lane_addr + kTmemP + sb * (kTcKeys / 2), pk[0]);
                tmem_st16(lane_addr + kTmemP + sb * (kTcKeys / 2) + 16, pk[1]);
                // The previous block's PV product (global index gb - 1) must be
                // complete before O is touched or P of this block is released;
                // observing every phase of odone in order keeps its parity
                // unambiguous (the next PV needs this block's P).
                if (gb > 0) ok = __all_sync(0xffffffffu, wait_or_abort(odone, (gb - 1) & 1, abort_flag));
                // rescale this row of O (the warp does it if any of its rows raised the max)
                if (j > 0 && __any_sync(0xffffffffu, up)) {
                    tc_fence_after();
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        uint32_t ov[32];
                        tmem_ld32(lane_addr + kTmemO + c0, ov);
                        tc_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
                        tmem_st32(lane_addr + kTmemO + c0, ov);
                    }
                }
                // keys past the context in the last block: zero their V rows so
                // stale (possibly NaN) data cannot reach the MMA (P is 0 there)
                if (j == t.n_blocks - 1 && (t.n_keys % kStageTok) != 0) {
                    const int first = t.n_keys - kbase;  // first invalid key of the block
                    const int last = (first / kStageTok + 1) * kStageTok;
                    const uint32_t slot = (uint32_t)(gb % NKV);
                    // gb counts blocks; KV slots advance one per block as well
                    uint8_t *vrow0 = smem + L::oKV + slot * L::kSlot + L::kHalves * L::kKVHalf;
                    for (int i = r; i < (last - first) * L::kHalves * 8; i += kTcRows) {
                        const int key = first + i / (L::kHalves * 8);
                        const int rest = i % (L::kHalves * 8);
                        *reinterpret_cast<uint4 *>(vrow0 + (rest / 8) * L::kKVHalf + key * 128 + (rest % 8) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                }
                tc_wait_st();
                tc_fence_before();
                mbar_arrive(&pfull[sb]);
            }
            if (!ok) break;
            // epilogue: O / l for this row
            ok = __all_sync(0xffffffffu, wait_or_abort(odone, (gb - 1) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *orow =
                real ? p.out + ((size_t)(t.q0 + tok) * p.Hq + (size_t)t.h * p.g + jh) * D : nullptr;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t ov[32];
                tmem_ld32(lane_addr + kTmemO + c0, ov);
                tc_wait_ld();
                if (real) {
#pragma unroll
                    for (int c = 0; c < 32; c += 8) {
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(ov[c]) * inv, __uint_as_float(ov[c + 1]) * inv);
                        v.y = pack_bf16x2(__uint_as_float(ov[c + 2]) * inv, __uint_as_float(ov[c + 3]) * inv);
                        v.z = pack_bf16x2(__uint_as_float(ov[c + 4]) * inv, __uint_as_float(ov[c + 5]) * inv);
                        v.w = pack_bf16x2(__uint_as_float(ov[c + 6]) * inv, __uint_as_float(ov[c + 7]) * inv);
                        *reinterpret_cast<uint4 *>(orow + c0 + c) = v;
                    }
                }
            }
            tc_fence_before();
        }
    }
    // Everyone is done with tensor memory before it is freed; a CTA that gave
    // up on a wait still frees it (the waits are bounded).
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
    grid_launch_dependents();
}

}  // namespace pkv
