// prefill_tc.cuh -- chunked-prefill paged attention on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// Chunked prefill (parameters and planner in prefill.cuh): query token i of a
// sequence's new chunk sits at position ctx - q_len + i and attends to positions
// [0, pos] read through the block table (wkbse.com "加速 LLM 推理：深入了解 vllm
// 引擎", section 3.1).  An item is (sequence, kv head, tile of 128 query rows),
// a row being (query token, head of the GQA group).
//
// Two CTAs per SM (each holds half of tensor memory and ~113 KB of shared
// memory), warp-specialised (224 threads):
//   warp 0       Q and K producer: the item's Q tile (128 x D bf16) by a 3-D
//                TMA load, and 64-key K blocks of the paged cache (4 stages of
//                16 keys each, addressed through the block table) into the K
//                ring; all 128-byte swizzled.  A K slot is released when its S
//                product completes.
//   warp 6       V producer: the same blocks' V into the V ring, a slot being
//                released when its PV product completes.  With its own warp
//                the K stream never waits behind a V slot that PV still holds.
//   warp 1       MMA issuer (one thread) and tensor-memory owner:
//                S_j = Q K_j^T  (tcgen05.mma kind::f16, M 128, N 64, K-major
//                smem operands, fp32 into TMEM S buffer j % 2), then
//                O += P_j V_j  (A = P in TMEM, B = V MN-major in smem,
//                N = D), each followed by tcgen05.commit onto an mbarrier.
//   warps 2-5    softmax: thread r owns row r (TMEM lane r).  It loads S_j,
//                masks the diagonal block, keeps the row's running max in
//                scaled log2 units (raised lazily, as in decode) and sum, writes
//                P_j as bf16 over the first half of S_j's own buffer, rescales
//                its O row when the max was raised (after the previous PV
//                product has completed), and at the end of the item normalises
//                O and stores the row.
// Two S buffers: the MMA thread issues P_j V_j as soon as P_j is ready and
// then S_{j+2} into S_j's buffer (the tensor core runs one thread's MMAs in
// order, so P_j has been read before S_{j+2} overwrites it).  S stays two
// blocks ahead of the softmax and no P·V queues behind an S issue.  The other
// CTA on the SM fills the gaps of this one.
#pragma once

#include "prefill.cuh"

namespace pkv {

constexpr int kTcRows = 128;          // M: query rows per item
constexpr int kTcKeys = 64;           // N: keys per block (4 stages of 16)
constexpr int kTcThreads = 7 * 32;
constexpr int kTcCtasPerSm = 2;
// Tensor memory of one CTA (256 of the SM's 512 columns):
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kTmemS = 0;        // S buffers: fp32, columns [0, 64) and [64, 128); P_j (bf16
                                      // pairs) over the first 32 columns of S_j's buffer
constexpr uint32_t kTmemO = 128;      // O: fp32, [128, 128 + D)

struct TcItem {
    int s, h, tile, q_len, prefix, q0, n_keys, n_blocks;
    int row0[4];  // TMA rows of the first 64-key block's four 16-key stages
};

// Shared memory of one CTA: NQ query buffers, an NK-slot K ring and an
// NV-slot V ring (two CTAs share an SM's 228 KB).
template <int D>
struct TcSmem {
    static constexpr int kHalves = D / 64;
    static constexpr int NQ = D == 128 ? 1 : 2;
    static constexpr int NK = D == 128 ? 2 : 4;
    static constexpr int NV = D == 128 ? 3 : 4;
    static constexpr int kQHalf = kTcRows * 128;          // 16 KB: 128 rows x 64 columns
    static constexpr int kQBuf = kHalves * kQHalf;
    static constexpr int kKVHalf = kTcKeys * 128;         // 8 KB: 64 keys x 64 columns
    static constexpr int kSlot = kHalves * kKVHalf;       // one K (or V) block
    static constexpr int oQ = 0;
    static constexpr int oK = NQ * kQBuf;
    static constexpr int oV = oK + NK * kSlot;
    static constexpr int oBars = oV + NV * kSlot;
    // kfull, kempty [NK]; vfull, vempty [NV]; qfull, qempty [NQ]; sfull[2],
    // pfull[2], odone, drain
    static constexpr int kNumBars = 2 * NK + 2 * NV + 2 * NQ + 6;
    static constexpr int oItem = oBars + kNumBars * 8;
    static constexpr int oTmemSlot = oItem + NQ * (int)sizeof(TcItem);
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

// 2^x on the special-function unit, flushing subnormal results to zero (a
// probability below 2^-126 of the row maximum contributes nothing in bf16).
__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed pair (a0, a1) = (b0 * c + d, b1 * c + d).
__device__ __forceinline__ void ffma2_bcast(float &a0, float &a1, float b0, float b1, float c, float d) {
    asm("{\n\t.reg .b64 pa, pb, pc, pd;\n\t"
        "mov.b64 pb, {%2, %3};\n\t"
        "mov.b64 pc, {%4, %4};\n\t"
        "mov.b64 pd, {%5, %5};\n\t"
        "fma.rn.f32x2 pa, pb, pc, pd;\n\t"
        "mov.b64 {%0, %1}, pa;\n\t}"
        : "=f"(a0), "=f"(a1)
        : "f"(b0), "f"(b1), "f"(c), "f"(d));
}

__device__ __forceinline__ float fmax3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Packed pair (a0, a1) += (b0, b1).
__device__ __forceinline__ void fadd2(float &a0, float &a1, float b0, float b1) {
    asm("{\n\t.reg .b64 pa, pb;\n\t"
        "mov.b64 pa, {%0, %1};\n\t"
        "mov.b64 pb, {%2, %3};\n\t"
        "add.rn.f32x2 pa, pa, pb;\n\t"
        "mov.b64 {%0, %1}, pa;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "f"(b0), "f"(b1));
}

// Item geometry from the item's planner entry `st` and its sequence's loaded
// lengths (ln = context_lens[s], query_start[s], query_start[s + 1]).
__device__ __forceinline__ TcItem tc_item(const PrefillParams &p, int it, int2 st, int3 ln) {
    TcItem t;
    const int e = it / p.Hkv;
    t.h = it - e * p.Hkv;
    t.s = st.x;
    t.tile = st.y;
    prefill_lengths_of(p, ln.x, ln.y, ln.z, false, t.q_len, t.prefix);
    t.q0 = ln.y;
    const int last_tok = min(t.q_len, (t.tile + 1) * p.QT) - 1;
    t.n_keys = t.prefix + last_tok + 1;
    t.n_blocks = (t.n_keys + kTcKeys - 1) / kTcKeys;
    return t;
}

__device__ __forceinline__ int3 tc_lengths(const PrefillParams &p, int s) {
    return make_int3(__ldg(p.context_lens + s), __ldg(p.query_start + s), __ldg(p.query_start + s + 1));
}

// Table entry of stage `lane` (< 4) of 64-key block j of item t (-1 for a
// stage past the keys, or a lane past 4).
__device__ __forceinline__ int tc_stage_block(const PrefillParams &p, const TcItem &t, int j, int lane) {
    const int tok = j * kTcKeys + (lane & 3) * kStageTok;
    return (lane < 4 && tok < t.n_keys) ? __ldg(p.block_tables + (size_t)t.s * p.MBS + tok / p.bs) : -1;
}

// TMA row of that stage from its table entry: an entry outside the pool, or a
// stage past the keys, reads rows beyond the pool (zero fill); the former is
// reported.
__device__ __forceinline__ int tc_stage_row_of(const PrefillParams &p, const TcItem &t, int j, int lane, int blk) {
    const int tok = j * kTcKeys + (lane & 3) * kStageTok;
    if (lane >= 4 || tok >= t.n_keys) return p.pool_rows;
    if (blk >= 0 && blk < p.NB) return (blk * p.Hkv + t.h) * p.bs + tok % p.bs;
    raise_error(PKV_DEVERR_BLOCK);
    return p.pool_rows;
}

__device__ __forceinline__ int tc_stage_row(const PrefillParams &p, const TcItem &t, int j, int lane) {
    return tc_stage_row_of(p, t, j, lane, tc_stage_block(p, t, j, lane));
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, kTcCtasPerSm)
    paged_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                            const __grid_constant__ CUtensorMap tmap_q, const PrefillParams p) {
    using L = TcSmem<D>;
    constexpr int NQ = L::NQ, NK = L::NK, NV = L::NV;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if ((smem_u32(smem_raw) & 1023u) != 0) {
        if (threadIdx.x == 0) raise_error(PKV_DEVERR_LAYOUT);
        return;
    }
    uint8_t *smem = smem_raw;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::oBars);
    uint64_t *kfull = bars, *kempty = bars + NK, *vfull = bars + 2 * NK, *vempty = bars + 2 * NK + NV;
    uint64_t *qfull = bars + 2 * NK + 2 * NV, *qempty = qfull + NQ;
    uint64_t *sfull = qempty + NQ, *pfull = sfull + 2, *odone = pfull + 2, *drain = odone + 1;
    TcItem *items = reinterpret_cast<TcItem *>(smem + L::oItem);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::oTmemSlot);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::oAbort);
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NK; ++i) {
            mbar_init(&kfull[i], 1);
            mbar_init(&kempty[i], 1);
        }
        for (int i = 0; i < NV; ++i) {
            mbar_init(&vfull[i], 1);
            mbar_init(&vempty[i], 1);
        }
        for (int i = 0; i < NQ; ++i) {
            mbar_init(&qfull[i], 1);
            // released by the MMA's commit (Q read), by every softmax thread
            // and by the V producer once they have taken the item description
            mbar_init(&qempty[i], 2 + kTcRows);
        }
        mbar_init(&sfull[0], 1);
        mbar_init(&sfull[1], 1);
        mbar_init(&pfull[0], kTcRows);
        mbar_init(&pfull[1], kTcRows);
        mbar_init(odone, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
        tma_prefetch_desc(&tmap_q);
    }
    // Q buffers start as zeros: rows a tile does not fill stay finite.
    for (int i = threadIdx.x; i < NQ * L::kQBuf / 16; i += kTcThreads)
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
        // ------------------------------------------------ Q and K producer --
        // The next item's claim, entry, lengths and first-block table entries
        // are fetched one step per K block while the current item streams, so
        // an item boundary waits on no dependent global load.
        uint32_t gk = 0;          // K blocks issued
        int q_issued = -1;        // ord of the last Q tile load
        bool ok = true;
        int claimed = 0;
        if (lane == 0) claimed = atomicAdd(p.work_counter, 1);
        int it = __shfl_sync(0xffffffffu, claimed, 0);
        TcItem cur;
        cur.n_blocks = -1;
        int row0 = p.pool_rows;
        if (it < n_items) {
            const int2 sp = p.entries[it / p.Hkv];
            cur = tc_item(p, it, sp, tc_lengths(p, sp.x));
            row0 = tc_stage_row(p, cur, 0, lane);
        }
        if (lane == 0) claimed = atomicAdd(p.work_counter, 1);  // the next item, one ahead
        for (int ord = 0; ok; ++ord) {
            const int qb = ord % NQ;
            // the first block's rows travel with the item (the V producer uses them)
#pragma unroll
            for (int i = 0; i < 4; ++i) cur.row0[i] = __shfl_sync(0xffffffffu, row0, i);
            if (lane == 0) {
                ok = wait_or_abort(&qempty[qb], ((ord / NQ) & 1) ^ 1, abort_flag);
                if (ok) {
                    TcItem t = cur;
                    if (it >= n_items) t.n_blocks = -1;  // end of stream
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
            // one step per K block, each using what the step before loaded:
            // claim -> entry -> lengths -> item geometry and first-block rows
            int nxt = n_items, pf = 0, nrow0 = p.pool_rows, nblk = -1;
            int2 nsp = make_int2(0, 0);
            int3 nln = make_int3(0, 0, 0);
            TcItem nt;
            nt.n_blocks = -1;
            auto prefetch_step = [&]() {
                if (pf == 0) {
                    nxt = __shfl_sync(0xffffffffu, claimed, 0);
                    if (nxt < n_items) nsp = p.entries[nxt / p.Hkv];
                } else if (pf == 1) {
                    if (nxt < n_items) nln = tc_lengths(p, nsp.x);
                } else if (pf == 2) {
                    if (nxt < n_items) {
                        nt = tc_item(p, nxt, nsp, nln);
                        nblk = tc_stage_block(p, nt, 0, lane);
                    }
                } else if (nxt < n_items) {
                    nrow0 = tc_stage_row_of(p, nt, 0, lane, nblk);
                }
                ++pf;
            };
            for (int j = 0; j < cur.n_blocks && ok; ++j) {
                // lane < 4: stage of 16 keys within the block
                const int row = j == 0 ? row0 : tc_stage_row(p, cur, j, lane);
                const uint32_t slot = gk % NK;
                if (lane == 0) {
                    ok = wait_or_abort(&kempty[slot], ((gk / NK) & 1) ^ 1, abort_flag);
                    if (ok) mbar_arrive_expect_tx(&kfull[slot], (uint32_t)L::kSlot);
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (ok && lane < 4) {
                    const uint32_t dst = sbase + L::oK + slot * L::kSlot + lane * (kStageTok * 128);
#pragma unroll
                    for (int hf = 0; hf < L::kHalves; ++hf)
                        tma_load_2d_u32(dst + hf * L::kKVHalf, &tmap_k, &kfull[slot], hf * 64, row);
                }
                if (ok) ++gk;
                if (pf < 4) prefetch_step();
            }
            while (ok && pf < 4) prefetch_step();  // a short item: finish the chain here
            if (lane == 0) claimed = atomicAdd(p.work_counter, 1);  // the item after next
            it = nxt;
            cur = nt;
            row0 = nrow0;
        }
        // After an abort, loads this CTA issued must land before it exits.
        if (lane == 0 && *abort_flag) {
            for (uint32_t c = (gk > (uint32_t)NK ? gk - NK : 0); c < gk; ++c)
                mbar_wait_bounded(&kfull[c % NK], (c / NK) & 1, kWaitLimitNs);
            if (q_issued >= 0) mbar_wait_bounded(&qfull[q_issued % NQ], ((q_issued / NQ) & 1), kWaitLimitNs);
        }
    } else if (warp == 6) {
        // ---------------------------------------------------- V producer --
        uint32_t gv = 0;
        bool ok = true;
        for (int ord = 0; ok; ++ord) {
            const int qb = ord % NQ;
            ok = __all_sync(0xffffffffu, wait_or_abort(&qfull[qb], (ord / NQ) & 1, abort_flag));
            if (!ok) break;
            const TcItem t = items[qb];
            __syncwarp();
            if (lane == 0) mbar_arrive(&qempty[qb]);
            if (t.n_blocks < 0) break;
            for (int j = 0; j < t.n_blocks && ok; ++j) {
                // lane < 4: stage of 16 keys, as in the K producer (the first
                // block's rows come with the item; the error, if any, was
                // reported there)
                int row = p.pool_rows;
                if (j == 0) {
                    row = lane == 0 ? t.row0[0] : lane == 1 ? t.row0[1] : lane == 2 ? t.row0[2] : t.row0[3];
                } else {
                    row = tc_stage_row(p, t, j, lane);
                }
                const uint32_t slot = gv % NV;
                if (lane == 0) {
                    ok = wait_or_abort(&vempty[slot], ((gv / NV) & 1) ^ 1, abort_flag);
                    if (ok) mbar_arrive_expect_tx(&vfull[slot], (uint32_t)L::kSlot);
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (ok && lane < 4) {
                    const uint32_t dst = sbase + L::oV + slot * L::kSlot + lane * (kStageTok * 128);
#pragma unroll
                    for (int hf = 0; hf < L::kHalves; ++hf)
                        tma_load_2d_u32(dst + hf * L::kKVHalf, &tmap_v, &vfull[slot], hf * 64, row);
                }
                if (ok) ++gv;
            }
        }
        if (lane == 0 && *abort_flag) {
            for (uint32_t c = (gv > (uint32_t)NV ? gv - NV : 0); c < gv; ++c)
                mbar_wait_bounded(&vfull[c % NV], (c / NV) & 1, kWaitLimitNs);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA --
        uint32_t gb = 0;  // blocks processed (K and V slots advance with it)
        bool ok = true;
        const uint32_t idesc_s = umma_idesc_bf16(kTcRows, kTcKeys, false);
        const uint32_t idesc_o = umma_idesc_bf16(kTcRows, D, true);
        for (int ord = 0; ok; ++ord) {
            const int qb = ord % NQ;
            ok = __all_sync(0xffffffffu, wait_or_abort(&qfull[qb], (ord / NQ) & 1, abort_flag));
            if (!ok) break;
            const int nb = items[qb].n_blocks;
            if (nb < 0) break;
            tc_fence_after();
            const uint32_t qaddr = sbase + L::oQ + qb * L::kQBuf;
            // Order: S_0, S_1, then for every block j: P_j V_j as soon as P_j is
            // ready, then S_{j+2} into the buffer P_j just vacated (the tensor
            // core runs this thread's MMAs in order, so P_j is read first).
            // S stays two blocks ahead of the softmax, and no P·V waits
            // behind an S issue.
            const uint32_t gb0 = gb;  // global index of the item's first block
            auto issue_s = [&](int jj) -> bool {
                const uint32_t g = gb0 + jj;
                const uint32_t slot = g % NK;
                if (!wait_or_abort(&kfull[slot], (g / NK) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t kaddr = sbase + L::oK + slot * L::kSlot;
                const uint32_t sbuf = tmem + kTmemS + (g & 1) * kTcKeys;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * L::kQHalf + (kk & 3) * 32;
                    const uint32_t koff = (kk >> 2) * L::kKVHalf + (kk & 3) * 32;
                    umma_ss(sbuf, umma_desc_sw128(qaddr + off, 16, 1024), umma_desc_sw128(kaddr + koff, 16, 1024),
                            idesc_s, kk > 0);
                }
                umma_commit(&sfull[g & 1]);
                umma_commit(&kempty[slot]);
                if (jj == nb - 1) umma_commit(&qempty[qb]);  // Q no longer read
                return true;
            };
            auto issue_pv = [&](int jj) -> bool {
                const uint32_t g = gb0 + jj;
                const uint32_t pb = g & 1;
                const uint32_t slot = g % NV;
                if (!wait_or_abort(&vfull[slot], (g / NV) & 1, abort_flag) ||
                    !wait_or_abort(&pfull[pb], (g >> 1) & 1, abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t vaddr = sbase + L::oV + slot * L::kSlot;
#pragma unroll
                for (int kk = 0; kk < kTcKeys / 16; ++kk)
                    umma_ts(tmem + kTmemO, tmem + kTmemS + pb * kTcKeys + kk * 8,
                            umma_desc_sw128(vaddr + kk * 16 * 128, L::kKVHalf, 1024), idesc_o,
                            (jj > 0 || kk > 0) ? 1u : 0u);
                umma_commit(odone);
                umma_commit(&vempty[slot]);
                return true;
            };
            if (lane == 0) {
                ok = issue_s(0) && (nb < 2 || issue_s(1));
                for (int jj = 0; jj < nb && ok; ++jj) {
                    ok = issue_pv(jj);
                    if (ok && jj + 2 < nb) ok = issue_s(jj + 2);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            gb += nb;
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
        const float c = p.scale_log2;          // > 0 (checked on the host)
        uint32_t gb = 0;
        bool ok = true;
        for (int ord = 0; ok; ++ord) {
            const int qb = ord % NQ;
            ok = __all_sync(0xffffffffu, wait_or_abort(&qfull[qb], (ord / NQ) & 1, abort_flag));
            if (!ok) break;
            const TcItem t = items[qb];
            mbar_arrive(&qempty[qb]);
            if (t.n_blocks < 0) break;
            const int tt = r / p.g, jh = r - tt * p.g;
            const int tok = t.tile * p.QT + tt;
            const bool real = tt < p.QT && tok < t.q_len;
            const int qpos = real ? t.prefix + tok : t.n_keys - 1;
            float m = PKV_NEG_INF, l0 = 0.f, l1 = 0.f;  // running max (scaled log2 units), sum
            for (int j = 0; j < t.n_blocks && ok; ++j, ++gb) {
                const uint32_t sbuf = kTmemS + (gb & 1) * kTcKeys;  // S_j, then P_j over it
                ok = __all_sync(0xffffffffu, wait_or_abort(&sfull[gb & 1], (gb >> 1) & 1, abort_flag));
                if (!ok) break;
                tc_fence_after();
                uint32_t sv[64];
                tmem_ld32(lane_addr + sbuf, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                tmem_ld32(lane_addr + sbuf + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                tc_wait_ld();
                // causal mask on the block the diagonal crosses; max of raw scores
                const int kbase = j * kTcKeys;
                if (__any_sync(0xffffffffu, kbase + kTcKeys - 1 > qpos)) {
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        if (kbase + i > qpos) sv[i] = __float_as_uint(PKV_NEG_INF);
                }
                // four independent chains of 3-input max
                float a0 = __uint_as_float(sv[0]), a1 = __uint_as_float(sv[1]);
                float a2 = __uint_as_float(sv[2]), a3 = __uint_as_float(sv[3]);
#pragma unroll
                for (int i = 4; i < 60; i += 8) {
                    a0 = fmax3f(a0, __uint_as_float(sv[i]), __uint_as_float(sv[i + 1]));
                    a1 = fmax3f(a1, __uint_as_float(sv[i + 2]), __uint_as_float(sv[i + 3]));
                    a2 = fmax3f(a2, __uint_as_float(sv[i + 4]), __uint_as_float(sv[i + 5]));
                    a3 = fmax3f(a3, __uint_as_float(sv[i + 6]), __uint_as_float(sv[i + 7]));
                }
                a0 = fmax3f(a0, __uint_as_float(sv[60]), __uint_as_float(sv[61]));
                a1 = fmax3f(a1, __uint_as_float(sv[62]), __uint_as_float(sv[63]));
                const float mxs = fmax3f(a0, a1, fmaxf(a2, a3)) * c;
                const bool up = mxs > m + kRescaleSlack;
                const float alpha = up ? ex2_ftz(m - mxs) : 1.f;
                if (up) m = mxs;
                const float nm = -m;
                float s0 = 0.f, s1 = 0.f;
                uint32_t pk[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float z0, z1;
                    ffma2_bcast(z0, z1, __uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1]), c, nm);
                    const float p0 = ex2_ftz(z0), p1 = ex2_ftz(z1);
                    fadd2(s0, s1, p0, p1);
                    pk[i] = pack_bf16x2(p0, p1);
                }
                l0 = l0 * alpha + s0;
                l1 = l1 * alpha + s1;
                tmem_st16(lane_addr + sbuf, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
                tmem_st16(lane_addr + sbuf + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
                // The previous block's PV product (global index gb - 1) must be
                // complete before O is touched or P of this block is released;
                // observing every phase of odone in order keeps its parity
                // unambiguous (the next PV needs this block's P).
                if (gb > 0) ok = __all_sync(0xffffffffu, wait_or_abort(odone, (gb - 1) & 1, abort_flag));
                // rescale this row of O (the warp does it if any of its rows raised the max)
                if (ok && j > 0 && __any_sync(0xffffffffu, up)) {
                    tc_fence_after();
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        uint32_t ov[32];
                        tmem_ld32(lane_addr + kTmemO + c0, ov);
                        tc_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                        tmem_st32(lane_addr + kTmemO + c0, ov);
                    }
                }
                // keys past the context in the last block: zero their V rows
                // (once the block has landed) so stale, possibly NaN, data
                // cannot reach the MMA (P is 0 there)
                if (ok && j == t.n_blocks - 1 && (t.n_keys % kStageTok) != 0) {
                    const uint32_t slot = gb % NV;
                    ok = __all_sync(0xffffffffu, wait_or_abort(&vfull[slot], (gb / NV) & 1, abort_flag));
                    const int first = t.n_keys - kbase;  // first invalid key of the block
                    const int last = (first / kStageTok + 1) * kStageTok;
                    uint8_t *vrow0 = smem + L::oV + slot * L::kSlot;
                    for (int i = r; ok && i < (last - first) * L::kHalves * 8; i += kTcRows) {
                        const int key = first + i / (L::kHalves * 8);
                        const int rest = i % (L::kHalves * 8);
                        *reinterpret_cast<uint4 *>(vrow0 + (rest / 8) * L::kKVHalf + key * 128 + (rest % 8) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                }
                tc_wait_st();
                tc_fence_before();
                mbar_arrive(&pfull[gb & 1]);
            }
            if (!ok) break;
            // epilogue: O / l for this row
            ok = __all_sync(0xffffffffu, wait_or_abort(odone, (gb - 1) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            const float l = l0 + l1;
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *orow =
                real ? p.out + ((size_t)(t.q0 + tok) * p.Hq + (size_t)t.h * p.g + jh) * D : nullptr;
            // A row is 2*D bytes, so with `out` 32-byte aligned every 16-column
            // piece of it is too, and it goes out in 32-byte stores (full
            // sectors, half the store instructions); 16-byte stores otherwise.
            const bool wide = (reinterpret_cast<uintptr_t>(p.out) & 31u) == 0;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t ov[32];
                tmem_ld32(lane_addr + kTmemO + c0, ov);
                tc_wait_ld();
                if (real) {
                    uint32_t lo[8], hi[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        lo[i] = pack_bf16x2(__uint_as_float(ov[2 * i]) * inv, __uint_as_float(ov[2 * i + 1]) * inv);
                        hi[i] = pack_bf16x2(__uint_as_float(ov[16 + 2 * i]) * inv,
                                            __uint_as_float(ov[16 + 2 * i + 1]) * inv);
                    }
                    if (wide) {
                        st_global_v8(orow + c0, lo);
                        st_global_v8(orow + c0 + 16, hi);
                    } else {
                        *reinterpret_cast<uint4 *>(orow + c0) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                        *reinterpret_cast<uint4 *>(orow + c0 + 8) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
                        *reinterpret_cast<uint4 *>(orow + c0 + 16) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                        *reinterpret_cast<uint4 *>(orow + c0 + 24) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
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
