// pkv_api.cu -- host side of the C ABI declared in include/pkv.h: argument
// validation, launch configuration, TMA descriptors and kernel launches.
// The device code lives in the headers included below (one translation unit,
// so the device error word is a single module global).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "block_manager.cuh"
#include "decode.cuh"
#include "pkv.h"
#include "prefill.cuh"
#include "prefill_tc.cuh"
#include "write_copy.cuh"

namespace {

constexpr int kMaxDevices = 64;
// NS: shared-memory ring slots per CTA (a multiple of the consumer warps)
constexpr int kStagesSimt = 8;
constexpr int kStagesMma = 8;
static_assert(kStagesSimt % pkv::kConsumerWarps == 0 && kStagesMma % pkv::kConsumerWarps == 0,
              "ring slots must be a multiple of the consumer warps");

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

// Per-device values computed on first use.  Several host threads may make
// their first call on a device at once: each slot is an atomic, and a value
// computed twice is the same value, so the last store is as good as the first.
using DeviceCache = std::atomic<int>[kMaxDevices];

int sm_count(int dev) {
    static DeviceCache cache{};
    if (dev < 0 || dev >= kMaxDevices) return 148;
    int n = cache[dev].load(std::memory_order_acquire);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev].store(n, std::memory_order_release);
    }
    return n;
}

pkv_status check_pool(const pkv_pool &pool) {
    if (pool.num_blocks <= 0 || pool.num_kv_heads <= 0 || pool.block_size <= 0 || pool.head_dim <= 0)
        return PKV_EINVAL;
    if (pool.kv_dtype != PKV_KV_BF16 && pool.kv_dtype != PKV_KV_E4M3) return PKV_EINVAL;
    if (pool.head_dim != 64 && pool.head_dim != 128) return PKV_EUNSUPPORTED;
    if (pool.block_size % 16 != 0 || pool.block_size > 1024) return PKV_EUNSUPPORTED;
    const long long rows = (long long)pool.num_blocks * pool.num_kv_heads * pool.block_size;
    if (rows >= (1ll << 31) - 1) return PKV_EUNSUPPORTED;  // TMA row coordinates are int32
    return PKV_OK;
}

// Bytes of one K/V element of the pool.
int elem_bytes(const pkv_pool &pool) { return pool.kv_dtype == PKV_KV_E4M3 ? 1 : 2; }

pkv_status launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PKV_OK : PKV_ECUDA;
}

// ------------------------------------------------------------ TMA maps ----

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// The pool viewed as a 2-D tensor: rows = (block, head, offset), columns =
// head_dim elements.  A box is 16 rows x 64 columns (128 B) with the 128-byte
// swizzle, so a K or V stage tile of one (block, head) is D/64 boxes.
bool encode_pool_map(CUtensorMap *map, const void *base, const pkv_pool &pool) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t rows = (cuuint64_t)pool.num_blocks * pool.num_kv_heads * pool.block_size;
    cuuint64_t dims[2] = {(cuuint64_t)pool.head_dim, rows};
    cuuint64_t strides[1] = {(cuuint64_t)pool.head_dim * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)pkv::kStageTok};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// An FP8 pool (e4m3 codes) as 2-D [rows][D] bytes; a box is 16 rows x 128
// bytes, the whole row at head dim 128.
bool encode_pool_map_u8(CUtensorMap *map, const void *base, const pkv_pool &pool) {
    auto fn = encode_fn();
    if (!fn || pool.head_dim != 128) return false;
    const cuuint64_t rows = (cuuint64_t)pool.num_blocks * pool.num_kv_heads * pool.block_size;
    cuuint64_t dims[2] = {(cuuint64_t)pool.head_dim, rows};
    cuuint64_t strides[1] = {(cuuint64_t)pool.head_dim};
    cuuint32_t box[2] = {128, (cuuint32_t)pkv::kStageTok};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The query tensor [T][Hq][D] viewed as 3-D (columns, heads, tokens); a box is
// 64 columns x g heads x QT tokens, so one tcgen05 prefill tile (rows = token x
// head of the group) lands as [QT][g][64] with the 128-byte swizzle.
bool encode_query_map(CUtensorMap *map, const void *base, int T, int Hq, int D, int g, int QT) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)T};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)g, (cuuint32_t)QT};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ----------------------------------------------------------- workspace ----

struct WorkspaceLayout {
    size_t off_count, off_entries, off_ml, off_acc, total;
};

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Library's choice of split-K partition: 512 tokens up to 16K-token contexts
// (short items keep a ragged batch balanced over the persistent CTAs), 2048
// beyond (fewer partitions per sequence: less per-item and reduce overhead).
int pick_partition_tokens(int32_t partition_tokens, int32_t max_context_len) {
    if (partition_tokens > 0) return partition_tokens;
    return max_context_len > 16384 ? 2048 : 512;
}

bool workspace_layout(int32_t B, int32_t Hq, int32_t D, int32_t max_ctx, int32_t PT, WorkspaceLayout *w) {
    if (B < 0 || Hq <= 0 || D <= 0 || max_ctx < 0 || PT <= 0) return false;
    const long long maxP = std::max<long long>(1, ((long long)max_ctx + PT - 1) / PT);
    size_t off = 0;
    w->off_count = off;
    off += 256;
    w->off_entries = off;
    off += round256((size_t)B * maxP * sizeof(int2));
    w->off_ml = off;
    if (maxP > 1) off += round256((size_t)B * Hq * maxP * sizeof(float2));
    w->off_acc = off;
    if (maxP > 1) off += round256((size_t)B * Hq * maxP * D * sizeof(float));
    w->total = off;
    return true;
}

// ---------------------------------------------------- decode dispatch ----

template <int D, int PATH, int GS, int GPAD, bool KV8 = false>
pkv_status launch_decode(const pkv::DecodeParams &prm, const CUtensorMap &mk, const CUtensorMap &mv,
                         cudaStream_t stream, int dev) {
    constexpr int NS = PATH == 0 ? kStagesSimt : kStagesMma;
    using L = pkv::DecodeSmem<D, (PATH == 0 ? GS : GPAD), NS, KV8>;
    auto kernel = pkv::paged_decode_kernel<D, PATH, GS, GPAD, NS, KV8>;
    // the shared-memory attribute is set before the occupancy query, so a
    // cached occupancy also means the attribute is set on this device
    static DeviceCache occ_cache{};
    int occ = (dev >= 0 && dev < kMaxDevices) ? occ_cache[dev].load(std::memory_order_acquire) : 0;
    if (occ == 0) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) != cudaSuccess)
            return PKV_ECUDA;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, pkv::kDecodeThreads, L::kAlloc) !=
                cudaSuccess ||
            occ <= 0)
            return PKV_ECUDA;
        if (dev >= 0 && dev < kMaxDevices) occ_cache[dev].store(occ, std::memory_order_release);
    }
    const long long items_upper = (long long)prm.B * prm.Hkv * prm.maxP;
    const long long grid = std::max<long long>(1, std::min<long long>(items_upper, (long long)sm_count(dev) * occ));

    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(pkv::kDecodeThreads);
    cfg.dynamicSmemBytes = L::kAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, mk, mv, prm) != cudaSuccess) return PKV_ECUDA;
    if (prm.maxP > 1) {
        cudaLaunchConfig_t rc = cfg;
        rc.gridDim = dim3((unsigned)((long long)prm.B * prm.Hq));
        rc.blockDim = dim3(pkv::kReduceWarps * 32);
        rc.dynamicSmemBytes = 0;
        if (cudaLaunchKernelEx(&rc, pkv::splitk_reduce_kernel<D>, prm) != cudaSuccess) return PKV_ECUDA;
    }
    return launch_status();
}

template <int D>
pkv_status dispatch_group(int g, const pkv::DecodeParams &prm, const CUtensorMap &mk, const CUtensorMap &mv,
                          cudaStream_t stream, int dev) {
    // g = 1 on CUDA cores; from g = 2 up the heads of a kv head share the
    // tensor-core tiles (measured faster than the two-head CUDA-core body)
    if (g == 1) return launch_decode<D, 0, 1, 1>(prm, mk, mv, stream, dev);
    if (g <= 4) return launch_decode<D, 1, 1, 4>(prm, mk, mv, stream, dev);
    if (g <= 8) return launch_decode<D, 1, 1, 8>(prm, mk, mv, stream, dev);
    return launch_decode<D, 1, 1, 16>(prm, mk, mv, stream, dev);
}

// -------------------------------------------------------- prefill ----

int prefill_query_tile(int g) { return pkv::kTcRows / g; }

// Workspace: entry count and work counter, the work list, and its staging
// copy in sequence order.
bool prefill_layout(int32_t B, int32_t g, int32_t max_q, size_t *off_entries, size_t *off_staged, size_t *total) {
    if (B < 0 || g <= 0 || max_q < 0) return false;
    const int QT = prefill_query_tile(g);
    const long long max_tiles = std::max<long long>(1, ((long long)max_q + QT - 1) / QT);
    const size_t list = round256((size_t)B * max_tiles * sizeof(int2));
    *off_entries = 256;
    *off_staged = 256 + list;
    *total = 256 + 2 * list;
    return true;
}

template <int D>
pkv_status launch_prefill_tc(const pkv::PrefillParams &prm, const CUtensorMap &mk, const CUtensorMap &mv,
                             const CUtensorMap &mq, cudaStream_t stream, int dev) {
    using L = pkv::TcSmem<D>;
    auto kernel = pkv::paged_prefill_tc_kernel<D>;
    static DeviceCache attr_set{};
    if (dev < 0 || dev >= kMaxDevices || attr_set[dev].load(std::memory_order_acquire) == 0) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes) != cudaSuccess)
            return PKV_ECUDA;
        if (dev >= 0 && dev < kMaxDevices) attr_set[dev].store(1, std::memory_order_release);
    }
    const long long tiles = std::max<long long>(1, ((long long)prm.max_q + prm.QT - 1) / prm.QT);
    const long long items_upper = (long long)prm.B * tiles * prm.Hkv;
    // persistent: two CTAs per SM, each holding half of tensor memory
    const long long grid = std::max<long long>(
        1, std::min<long long>(items_upper, (long long)pkv::kTcCtasPerSm * sm_count(dev)));
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(pkv::kTcThreads);
    cfg.dynamicSmemBytes = L::kBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, mk, mv, mq, prm) != cudaSuccess) return PKV_ECUDA;
    return launch_status();
}

// One copy launch of n <= CAP validated pairs (host int32 [n][2]), by value.
template <int CAP>
pkv_status copy_launch(const int32_t *pairs, int n, void *k_cache, void *v_cache, int64_t vec_per_block,
                       pkv_stream_t stream) {
    pkv::CopyParams<CAP> p;
    p.k_cache = static_cast<uint4 *>(k_cache);
    p.v_cache = static_cast<uint4 *>(v_cache);
    p.vec_per_block = vec_per_block;
    p.num_pairs = n;
    for (int i = 0; i < n; ++i) p.pairs[i] = make_int2(pairs[2 * i], pairs[2 * i + 1]);
    const long long per_cta = pkv::kCopyThreads * pkv::kCopyVecPerThread;
    const unsigned gx = (unsigned)((vec_per_block + per_cta - 1) / per_cta);
    pkv::copy_blocks_kernel<CAP><<<dim3(gx, n), pkv::kCopyThreads, 0, (cudaStream_t)stream>>>(p);
    return launch_status();
}

// Device address of host memory the GPU can reach (pinned; unified addressing
// makes it the host address), or nullptr for pageable or device memory.
void *mapped_host_pointer(const void *p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();  // clear the sticky-free error of an unknown pointer
        return nullptr;
    }
    if (a.type != cudaMemoryTypeHost || a.devicePointer == nullptr) return nullptr;
    return a.devicePointer;
}

template <bool OUT>
pkv_status swap_blocks(const int32_t *block_ids, int32_t n, void *k_cache, void *v_cache, const pkv_pool &pool,
                       const void *host_k, const void *host_v, pkv_stream_t stream) {
    const pkv_status ps = check_pool(pool);
    if (ps != PKV_OK) return ps;
    if (n < 0) return PKV_EINVAL;
    if (n == 0) return PKV_OK;
    if (!block_ids || !k_cache || !v_cache || !host_k || !host_v) return PKV_EINVAL;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(host_k, 16) || !aligned(host_v, 16))
        return PKV_EINVAL;
    for (int i = 0; i < n; ++i)
        if (block_ids[i] < 0 || block_ids[i] >= pool.num_blocks) return PKV_ERANGE;
    if (!OUT) {  // two copies into one block would leave it undefined
        std::vector<int32_t> ids(block_ids, block_ids + n);
        std::sort(ids.begin(), ids.end());
        for (int i = 1; i < n; ++i)
            if (ids[i] == ids[i - 1]) return PKV_EALIAS;
    }
    uint8_t *hk = static_cast<uint8_t *>(mapped_host_pointer(host_k));
    uint8_t *hv = static_cast<uint8_t *>(mapped_host_pointer(host_v));
    if (!hk || !hv) return PKV_EINVAL;
    const size_t block_bytes = (size_t)pool.num_kv_heads * pool.block_size * pool.head_dim * elem_bytes(pool);
    pkv::SwapParams p;
    p.pool_k = static_cast<uint4 *>(k_cache);
    p.pool_v = static_cast<uint4 *>(v_cache);
    p.vec_per_block = (int64_t)(block_bytes / 16);
    const long long per_cta = pkv::kSwapThreads * pkv::kSwapVecPerThread;
    const unsigned gx = (unsigned)((p.vec_per_block + per_cta - 1) / per_cta);
    for (int base = 0; base < n; base += pkv::kMaxSwapPerLaunch) {
        const int m = std::min(pkv::kMaxSwapPerLaunch, n - base);
        p.n = m;
        p.host_k = reinterpret_cast<uint4 *>(hk + (size_t)base * block_bytes);
        p.host_v = reinterpret_cast<uint4 *>(hv + (size_t)base * block_bytes);
        std::memcpy(p.ids, block_ids + base, sizeof(int32_t) * m);
        pkv::swap_blocks_kernel<OUT><<<dim3(gx, m), pkv::kSwapThreads, 0, (cudaStream_t)stream>>>(p);
        const pkv_status st = launch_status();
        if (st != PKV_OK) return st;
    }
    return PKV_OK;
}


// Block-manager state: a 256-byte header (top, error word, cached blocks,
// ring head and tail), then 256-byte-aligned arrays: free stack, reference
// counts and three scratch arrays (int32 [num_blocks] each), the prefix keys
// (uint64 [num_blocks]), the ring positions of cached blocks (uint32
// [num_blocks]), the eviction ring (int32 [2 num_blocks]) and the eviction
// scratch (int32 [num_blocks]).
size_t bm_array_bytes(int32_t nb) { return round256((size_t)nb * 4); }

bool bm_state(void *state, int32_t nb, pkv::BmState *s) {
    if (!state || nb <= 0 || nb > (1 << 29) || !aligned(state, 256)) return false;
    uint8_t *p = static_cast<uint8_t *>(state);
    const size_t a = bm_array_bytes(nb);
    const size_t h = round256((size_t)nb * 8);
    s->hdr = reinterpret_cast<int32_t *>(p);
    s->free_stack = reinterpret_cast<int32_t *>(p + 256);
    s->refcount = reinterpret_cast<int32_t *>(p + 256 + a);
    s->last_idx = reinterpret_cast<int32_t *>(p + 256 + 2 * a);
    s->zeroed = reinterpret_cast<int32_t *>(p + 256 + 3 * a);
    s->cow_rank = reinterpret_cast<int32_t *>(p + 256 + 4 * a);
    s->block_hash = reinterpret_cast<uint64_t *>(p + 256 + 5 * a);
    s->lru_pos = reinterpret_cast<uint32_t *>(p + 256 + 5 * a + h);
    s->ring = reinterpret_cast<int32_t *>(p + 256 + 6 * a + h);
    s->evicted = reinterpret_cast<int32_t *>(p + 256 + 6 * a + h + round256((size_t)nb * 8));
    return true;
}

// Prefix cache: keys (uint64), block ids and claims (int32), cap each.
bool prefix_cache(void *cache, int32_t cap, pkv::PrefixCache *c) {
    if (!cache || cap < 2 || (cap & (cap - 1)) != 0 || !aligned(cache, 256)) return false;
    uint8_t *p = static_cast<uint8_t *>(cache);
    c->keys = reinterpret_cast<unsigned long long *>(p);
    c->vals = reinterpret_cast<int32_t *>(p + round256((size_t)cap * 8));
    c->claim = reinterpret_cast<int32_t *>(p + round256((size_t)cap * 8) + round256((size_t)cap * 4));
    c->cap = cap;
    return true;
}

// Decode over a bf16 pool (scales null) or an FP8 (e4m3) pool with per-kv-head
// dequantisation scales (head dim 128, GQA group <= 2: the CUDA-core path).
pkv_status decode_impl(const void *q, const void *k_cache, const void *v_cache, const float *k_scale,
                       const float *v_scale, const int32_t *block_tables, int32_t max_blocks_per_seq,
                       const int32_t *context_lens, int32_t num_seqs, int32_t num_q_heads, float scale,
                       int32_t num_kv_heads, void *out, pkv_pool pool, int32_t max_context_len,
                       int32_t partition_tokens, void *workspace, size_t workspace_bytes, pkv_stream_t stream) {
    const bool kv8 = k_scale != nullptr;
    if (pool.kv_dtype != (kv8 ? PKV_KV_E4M3 : PKV_KV_BF16)) return PKV_EINVAL;
    const pkv_status ps = check_pool(pool);
    if (ps != PKV_OK) return ps;
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0)
        return PKV_EINVAL;
    if (num_kv_heads != pool.num_kv_heads || num_q_heads % num_kv_heads != 0) return PKV_EINVAL;
    const int g = num_q_heads / num_kv_heads;
    if (g > 16) return PKV_EUNSUPPORTED;
    if (kv8 && pool.head_dim != 128) return PKV_EUNSUPPORTED;
    if (partition_tokens < 0 || partition_tokens % 16 != 0 || partition_tokens > 65536) return PKV_EINVAL;
    if (num_seqs == 0) return PKV_OK;
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out || !workspace) return PKV_EINVAL;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(workspace, 256))
        return PKV_EINVAL;
    const int D = pool.head_dim;
    const int PT = pick_partition_tokens(partition_tokens, max_context_len);
    WorkspaceLayout wl;
    if (!workspace_layout(num_seqs, num_q_heads, D, max_context_len, PT, &wl) || workspace_bytes < wl.total)
        return PKV_EINVAL;

    pkv::DecodeParams prm;
    prm.q = static_cast<const __nv_bfloat16 *>(q);
    prm.out = static_cast<__nv_bfloat16 *>(out);
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    prm.num_entries = reinterpret_cast<int32_t *>(ws + wl.off_count);
    prm.work_counter = reinterpret_cast<int32_t *>(ws + wl.off_count) + 1;
    prm.entries = reinterpret_cast<int2 *>(ws + wl.off_entries);
    prm.part_ml = reinterpret_cast<float2 *>(ws + wl.off_ml);
    prm.part_acc = reinterpret_cast<float *>(ws + wl.off_acc);
    prm.B = num_seqs;
    prm.Hq = num_q_heads;
    prm.Hkv = num_kv_heads;
    prm.g = g;
    prm.MBS = max_blocks_per_seq;
    prm.bs = pool.block_size;
    prm.NB = pool.num_blocks;
    prm.max_ctx = max_context_len;
    prm.PT = PT;
    prm.maxP = (int)std::max<long long>(1, ((long long)max_context_len + PT - 1) / PT);
    prm.pool_rows = pool.num_blocks * pool.num_kv_heads * pool.block_size;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.k_scale = k_scale;
    prm.v_scale = v_scale;

    CUtensorMap mk, mv;
    if (kv8) {
        if (!encode_pool_map_u8(&mk, k_cache, pool) || !encode_pool_map_u8(&mv, v_cache, pool)) return PKV_ECUDA;
    } else if (!encode_pool_map(&mk, k_cache, pool) || !encode_pool_map(&mv, v_cache, pool)) {
        return PKV_ECUDA;
    }

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    pkv::plan_kernel<<<1, pkv::kPlanThreads, 0, st>>>(prm, D);
    pkv_status r = launch_status();
    if (r != PKV_OK) return r;
    const int dev = current_device();
    if (kv8) {
        // g = 2 runs on the tensor cores too: over e4m3 codes the CUDA-core body
        // is issue-bound (a conversion and four unpacked FMAs per code pair)
        if (g == 1) return launch_decode<128, 0, 1, 1, true>(prm, mk, mv, st, dev);
        if (g <= 4) return launch_decode<128, 1, 1, 4, true>(prm, mk, mv, st, dev);
        if (g <= 8) return launch_decode<128, 1, 1, 8, true>(prm, mk, mv, st, dev);
        return launch_decode<128, 1, 1, 16, true>(prm, mk, mv, st, dev);
    }
    return D == 128 ? dispatch_group<128>(g, prm, mk, mv, st, dev) : dispatch_group<64>(g, prm, mk, mv, st, dev);
}

}  // namespace

extern "C" {

int32_t pkv_version(void) { return 10100; }

const char *pkv_status_string(pkv_status s) {
    switch (s) {
        case PKV_OK: return "ok";
        case PKV_EINVAL: return "invalid argument (size, null or misaligned pointer, workspace)";
        case PKV_ERANGE: return "block id outside the pool";
        case PKV_EALIAS: return "copy pairs alias (repeated destination, or destination that is a source)";
        case PKV_ECUDA: return "CUDA call failed";
        case PKV_EDEVICE: return "device error word set";
        case PKV_EUNSUPPORTED: return "unsupported shape";
    }
    return "unknown status";
}

pkv_status pkv_write(const void *k, const void *v, const int64_t *slot_mapping, int32_t num_tokens, void *k_cache,
                     void *v_cache, pkv_pool pool, pkv_stream_t stream) {
    const pkv_status ps = check_pool(pool);
    if (ps != PKV_OK) return ps;
    if (pool.kv_dtype != PKV_KV_BF16) return PKV_EINVAL;
    if (num_tokens < 0) return PKV_EINVAL;
    if (num_tokens == 0) return PKV_OK;
    if (!k || !v || !slot_mapping || !k_cache || !v_cache) return PKV_EINVAL;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(slot_mapping, 8))
        return PKV_EINVAL;
    pkv::WriteParams p;
    p.k = static_cast<const uint4 *>(k);
    p.v = static_cast<const uint4 *>(v);
    p.slots = slot_mapping;
    p.k_cache = static_cast<uint4 *>(k_cache);
    p.v_cache = static_cast<uint4 *>(v_cache);
    p.vpr = pool.head_dim / 8;
    p.num_kv_heads = pool.num_kv_heads;
    p.block_size = pool.block_size;
    p.pool_slots = (int64_t)pool.num_blocks * pool.block_size;
    p.total = (int64_t)num_tokens * 2 * pool.num_kv_heads * p.vpr;
    const int dev = current_device();
    const long long blocks = std::min<long long>((p.total + 255) / 256, (long long)sm_count(dev) * 16);
    pkv::kv_write_kernel<<<(unsigned)std::max<long long>(blocks, 1), 256, 0, (cudaStream_t)stream>>>(p);
    return launch_status();
}

pkv_status pkv_copy_blocks(const int32_t *src_dst_pairs, int32_t num_pairs, void *k_cache, void *v_cache,
                           pkv_pool pool, pkv_stream_t stream) {
    const pkv_status ps = check_pool(pool);
    if (ps != PKV_OK) return ps;
    if (num_pairs < 0) return PKV_EINVAL;
    if (num_pairs == 0) return PKV_OK;
    if (!src_dst_pairs || !k_cache || !v_cache) return PKV_EINVAL;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16)) return PKV_EINVAL;
    std::vector<int32_t> src(num_pairs), dst(num_pairs);
    for (int i = 0; i < num_pairs; ++i) {
        src[i] = src_dst_pairs[2 * i];
        dst[i] = src_dst_pairs[2 * i + 1];
        if (src[i] < 0 || src[i] >= pool.num_blocks || dst[i] < 0 || dst[i] >= pool.num_blocks) return PKV_ERANGE;
    }
    std::sort(src.begin(), src.end());
    std::vector<int32_t> dsorted(dst);
    std::sort(dsorted.begin(), dsorted.end());
    for (int i = 1; i < num_pairs; ++i)
        if (dsorted[i] == dsorted[i - 1]) return PKV_EALIAS;
    for (int i = 0; i < num_pairs; ++i)
        if (std::binary_search(src.begin(), src.end(), dsorted[i])) return PKV_EALIAS;

    const int64_t vec = (int64_t)pool.num_kv_heads * pool.block_size * pool.head_dim * elem_bytes(pool) / 16;
    for (int base = 0; base < num_pairs; base += pkv::kMaxPairsPerLaunch) {
        const int n = std::min(pkv::kMaxPairsPerLaunch, num_pairs - base);
        const int32_t *pr = src_dst_pairs + 2 * base;
        const pkv_status st = n <= 32    ? copy_launch<32>(pr, n, k_cache, v_cache, vec, stream)
                              : n <= 256 ? copy_launch<256>(pr, n, k_cache, v_cache, vec, stream)
                                         : copy_launch<pkv::kMaxPairsPerLaunch>(pr, n, k_cache, v_cache, vec, stream);
        if (st != PKV_OK) return st;
    }
    return PKV_OK;
}

pkv_status pkv_swap_out(const void *k_cache, const void *v_cache, pkv_pool pool, const int32_t *block_ids,
                        int32_t n, void *host_k, void *host_v, pkv_stream_t stream) {
    return swap_blocks<true>(block_ids, n, const_cast<void *>(k_cache), const_cast<void *>(v_cache), pool, host_k,
                             host_v, stream);
}

pkv_status pkv_swap_in(const void *host_k, const void *host_v, const int32_t *block_ids, int32_t n, void *k_cache,
                       void *v_cache, pkv_pool pool, pkv_stream_t stream) {
    return swap_blocks<false>(block_ids, n, k_cache, v_cache, pool, host_k, host_v, stream);
}

pkv_status pkv_lru_victims(const int64_t *last_use, const uint8_t *evictable, int32_t num_blocks, int32_t k,
                           int32_t *victims, int32_t *count) {
    if (num_blocks < 0 || k < 0 || !count) return PKV_EINVAL;
    if (num_blocks > 0 && (!last_use || !evictable)) return PKV_EINVAL;
    if (k > 0 && !victims) return PKV_EINVAL;
    std::vector<int32_t> cand;
    cand.reserve(num_blocks);
    for (int32_t b = 0; b < num_blocks; ++b)
        if (evictable[b]) cand.push_back(b);
    const size_t m = std::min<size_t>((size_t)k, cand.size());
    auto older = [&](int32_t a, int32_t b) {
        return last_use[a] < last_use[b] || (last_use[a] == last_use[b] && a < b);
    };
    std::partial_sort(cand.begin(), cand.begin() + m, cand.end(), older);
    for (size_t i = 0; i < m; ++i) victims[i] = cand[i];
    *count = (int32_t)m;
    return PKV_OK;
}

size_t pkv_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                  int32_t max_context_len, int32_t partition_tokens) {
    if (num_kv_heads <= 0 || num_q_heads <= 0 || num_q_heads % num_kv_heads) return 0;
    if (partition_tokens < 0 || partition_tokens % 16) return 0;
    WorkspaceLayout w;
    if (!workspace_layout(num_seqs, num_q_heads, head_dim, max_context_len,
                          pick_partition_tokens(partition_tokens, max_context_len), &w))
        return 0;
    return w.total;
}

pkv_status paged_attn_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                             int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs,
                             int32_t num_q_heads, float scale, int32_t num_kv_heads, void *out, pkv_pool pool,
                             int32_t max_context_len, int32_t partition_tokens, void *workspace,
                             size_t workspace_bytes, pkv_stream_t stream) {
    return decode_impl(q, k_cache, v_cache, nullptr, nullptr, block_tables, max_blocks_per_seq, context_lens,
                       num_seqs, num_q_heads, scale, num_kv_heads, out, pool, max_context_len, partition_tokens,
                       workspace, workspace_bytes, stream);
}

pkv_status paged_attn_decode_fp8(const void *q, const void *k_cache, const void *v_cache, const float *k_scale,
                                 const float *v_scale, const int32_t *block_tables, int32_t max_blocks_per_seq,
                                 const int32_t *context_lens, int32_t num_seqs, int32_t num_q_heads, float scale,
                                 int32_t num_kv_heads, void *out, pkv_pool pool, int32_t max_context_len,
                                 int32_t partition_tokens, void *workspace, size_t workspace_bytes,
                                 pkv_stream_t stream) {
    if (!k_scale || !v_scale || !aligned(k_scale, 4) || !aligned(v_scale, 4)) return PKV_EINVAL;
    return decode_impl(q, k_cache, v_cache, k_scale, v_scale, block_tables, max_blocks_per_seq, context_lens,
                       num_seqs, num_q_heads, scale, num_kv_heads, out, pool, max_context_len, partition_tokens,
                       workspace, workspace_bytes, stream);
}

pkv_status pkv_write_fp8(const void *k, const void *v, const int64_t *slot_mapping, int32_t num_tokens,
                         const float *k_scale, const float *v_scale, void *k_cache, void *v_cache, pkv_pool pool,
                         pkv_stream_t stream) {
    const pkv_status ps = check_pool(pool);
    if (ps != PKV_OK) return ps;
    if (pool.kv_dtype != PKV_KV_E4M3) return PKV_EINVAL;
    if (num_tokens < 0) return PKV_EINVAL;
    if (num_tokens == 0) return PKV_OK;
    if (!k || !v || !slot_mapping || !k_cache || !v_cache || !k_scale || !v_scale) return PKV_EINVAL;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(slot_mapping, 8) || !aligned(k_scale, 4) || !aligned(v_scale, 4))
        return PKV_EINVAL;
    pkv::WriteFp8Params p;
    p.k = static_cast<const uint4 *>(k);
    p.v = static_cast<const uint4 *>(v);
    p.slots = slot_mapping;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.k_cache = static_cast<uint2 *>(k_cache);
    p.v_cache = static_cast<uint2 *>(v_cache);
    p.vpr = pool.head_dim / 8;
    p.num_kv_heads = pool.num_kv_heads;
    p.block_size = pool.block_size;
    p.pool_slots = (int64_t)pool.num_blocks * pool.block_size;
    p.total = (int64_t)num_tokens * 2 * pool.num_kv_heads * p.vpr;
    const int dev = current_device();
    const long long blocks = std::min<long long>((p.total + 255) / 256, (long long)sm_count(dev) * 16);
    pkv::kv_write_fp8_kernel<<<(unsigned)std::max<long long>(blocks, 1), 256, 0, (cudaStream_t)stream>>>(p);
    return launch_status();
}

size_t pkv_prefill_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                   int32_t max_query_len) {
    if (num_kv_heads <= 0 || num_q_heads <= 0 || num_q_heads % num_kv_heads) return 0;
    size_t off, off_staged, total;
    if (!prefill_layout(num_seqs, num_q_heads / num_kv_heads, max_query_len, &off, &off_staged, &total)) return 0;
    return total;
}

pkv_status paged_attn_prefill(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                              int32_t max_blocks_per_seq, const int32_t *context_lens, const int32_t *query_start,
                              int32_t num_seqs, int32_t num_tokens, int32_t num_q_heads, float scale,
                              int32_t num_kv_heads, void *out, pkv_pool pool, int32_t max_query_len,
                              int32_t max_context_len, void *workspace, size_t workspace_bytes, pkv_stream_t stream) {
    const pkv_status ps = check_pool(pool);
    if (ps != PKV_OK) return ps;
    if (pool.kv_dtype != PKV_KV_BF16) return PKV_EINVAL;
    if (num_seqs < 0 || num_tokens < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0 ||
        max_context_len < 0 || max_query_len < 0)
        return PKV_EINVAL;
    if (num_kv_heads != pool.num_kv_heads || num_q_heads % num_kv_heads != 0) return PKV_EINVAL;
    const int g = num_q_heads / num_kv_heads;
    if (g > 16) return PKV_EUNSUPPORTED;
    if (!(scale > 0.f) || !std::isfinite(scale)) return PKV_EINVAL;
    if (num_seqs == 0 || max_query_len == 0 || num_tokens == 0) return PKV_OK;
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start || !out || !workspace)
        return PKV_EINVAL;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(query_start, 4) || !aligned(workspace, 256))
        return PKV_EINVAL;
    size_t off_entries, off_staged, total;
    if (!prefill_layout(num_seqs, g, max_query_len, &off_entries, &off_staged, &total) || workspace_bytes < total)
        return PKV_EINVAL;
    pkv::PrefillParams prm;
    prm.q = static_cast<const __nv_bfloat16 *>(q);
    prm.out = static_cast<__nv_bfloat16 *>(out);
    prm.block_tables = block_tables;
    prm.context_lens = context_lens;
    prm.query_start = query_start;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    prm.num_entries = reinterpret_cast<int32_t *>(ws);
    prm.work_counter = reinterpret_cast<int32_t *>(ws) + 1;
    prm.entries = reinterpret_cast<int2 *>(ws + off_entries);
    prm.staged = reinterpret_cast<int2 *>(ws + off_staged);
    prm.B = num_seqs;
    prm.Hq = num_q_heads;
    prm.Hkv = num_kv_heads;
    prm.g = g;
    prm.MBS = max_blocks_per_seq;
    prm.bs = pool.block_size;
    prm.NB = pool.num_blocks;
    prm.max_ctx = max_context_len;
    prm.max_q = max_query_len;
    prm.QT = prefill_query_tile(g);
    prm.T = num_tokens;
    prm.pool_rows = pool.num_blocks * pool.num_kv_heads * pool.block_size;
    prm.scale_log2 = scale * 1.4426950408889634f;
    CUtensorMap mk, mv;
    if (!encode_pool_map(&mk, k_cache, pool) || !encode_pool_map(&mv, v_cache, pool)) return PKV_ECUDA;
    CUtensorMap mq;
    if (!encode_query_map(&mq, q, num_tokens, num_q_heads, pool.head_dim, g, prm.QT)) return PKV_ECUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    pkv::plan_prefill_kernel<<<1, pkv::kPlanThreads, 0, st>>>(prm);
    const pkv_status r = launch_status();
    if (r != PKV_OK) return r;
    const int dev = current_device();
    return pool.head_dim == 128 ? launch_prefill_tc<128>(prm, mk, mv, mq, st, dev)
                                : launch_prefill_tc<64>(prm, mk, mv, mq, st, dev);
}

size_t pkv_bm_state_bytes(int32_t num_blocks) {
    if (num_blocks <= 0 || num_blocks > (1 << 29)) return 0;
    return 256 + 7 * bm_array_bytes(num_blocks) + 2 * round256((size_t)num_blocks * 8);
}

size_t pkv_prefix_cache_bytes(int32_t capacity) {
    if (capacity < 2 || (capacity & (capacity - 1)) != 0) return 0;
    return round256((size_t)capacity * 8) + 2 * round256((size_t)capacity * 4);
}

pkv_status pkv_prefix_cache_init(void *cache, int32_t capacity, pkv_stream_t stream) {
    pkv::PrefixCache c;
    if (!prefix_cache(cache, capacity, &c)) return PKV_EINVAL;
    const int grid = std::max(1, std::min(1024, (capacity + 255) / 256));
    pkv::prefix_cache_init_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(c);
    return launch_status();
}

static pkv_status prefix_params(void *state, int32_t num_blocks, void *cache, int32_t capacity,
                                const int32_t *tokens, const int32_t *query_start, int32_t num_seqs,
                                int32_t block_size, int32_t *block_tables, int32_t max_blocks_per_seq,
                                pkv::PrefixParams *p) {
    if (!bm_state(state, num_blocks, &p->s) || !prefix_cache(cache, capacity, &p->c)) return PKV_EINVAL;
    if (num_seqs < 0 || block_size <= 0 || max_blocks_per_seq <= 0) return PKV_EINVAL;
    if (num_seqs > 0 && (!tokens || !query_start || !block_tables)) return PKV_EINVAL;
    if (!aligned(tokens, 4) || !aligned(query_start, 4) || !aligned(block_tables, 4)) return PKV_EINVAL;
    p->tokens = tokens;
    p->query_start = query_start;
    p->tables = block_tables;
    p->nb = num_blocks;
    p->B = num_seqs;
    p->bs = block_size;
    p->mbs = max_blocks_per_seq;
    p->num_cached = nullptr;
    return PKV_OK;
}

pkv_status pkv_prefix_lookup(void *state, int32_t num_blocks, void *cache, int32_t capacity, const int32_t *tokens,
                             const int32_t *query_start, int32_t num_seqs, int32_t block_size,
                             int32_t *block_tables, int32_t max_blocks_per_seq, int32_t *num_cached,
                             pkv_stream_t stream) {
    pkv::PrefixParams p;
    const pkv_status st = prefix_params(state, num_blocks, cache, capacity, tokens, query_start, num_seqs,
                                        block_size, block_tables, max_blocks_per_seq, &p);
    if (st != PKV_OK) return st;
    if (num_seqs == 0) return PKV_OK;
    if (!num_cached || !aligned(num_cached, 4)) return PKV_EINVAL;
    p.num_cached = num_cached;
    pkv::prefix_lookup_kernel<<<(num_seqs + 7) / 8, 256, 0, (cudaStream_t)stream>>>(p);  // a warp per sequence
    return launch_status();
}

pkv_status pkv_prefix_insert(void *state, int32_t num_blocks, void *cache, int32_t capacity, const int32_t *tokens,
                             const int32_t *query_start, int32_t num_seqs, int32_t block_size,
                             const int32_t *block_tables, int32_t max_blocks_per_seq, pkv_stream_t stream) {
    pkv::PrefixParams p;
    const pkv_status st = prefix_params(state, num_blocks, cache, capacity, tokens, query_start, num_seqs,
                                        block_size, const_cast<int32_t *>(block_tables), max_blocks_per_seq, &p);
    if (st != PKV_OK) return st;
    if (num_seqs == 0) return PKV_OK;
    const unsigned grid = (unsigned)((num_seqs + 7) / 8);  // a warp per sequence
    pkv::prefix_insert_kernel<0><<<grid, 256, 0, (cudaStream_t)stream>>>(p);
    pkv::prefix_insert_kernel<1><<<grid, 256, 0, (cudaStream_t)stream>>>(p);
    pkv::prefix_insert_kernel<2><<<grid, 256, 0, (cudaStream_t)stream>>>(p);
    return launch_status();
}

pkv_status pkv_bm_init(void *state, int32_t num_blocks, pkv_stream_t stream) {
    pkv::BmState s;
    if (!bm_state(state, num_blocks, &s)) return PKV_EINVAL;
    const int grid = std::max(1, std::min(1024, (num_blocks + 255) / 256));
    pkv::bm_init_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(s, num_blocks);
    return launch_status();
}

pkv_status pkv_bm_alloc(void *state, int32_t num_blocks, const int32_t *counts, int32_t n, int32_t *offsets,
                        int32_t *ids, int32_t capacity, pkv_stream_t stream) {
    pkv::BmState s;
    if (!bm_state(state, num_blocks, &s) || n < 0 || capacity < 0) return PKV_EINVAL;
    if (!offsets || (n > 0 && !counts) || (capacity > 0 && !ids)) return PKV_EINVAL;
    if (!aligned(counts, 4) || !aligned(offsets, 4) || !aligned(ids, 4)) return PKV_EINVAL;
    pkv::bm_alloc_kernel<<<1, pkv::kBmThreads, 0, (cudaStream_t)stream>>>(s, num_blocks, counts, n, offsets, ids,
                                                                         capacity);
    return launch_status();
}

pkv_status pkv_bm_free(void *state, int32_t num_blocks, const int32_t *block_ids, int32_t n, pkv_stream_t stream) {
    pkv::BmState s;
    if (!bm_state(state, num_blocks, &s) || n < 0) return PKV_EINVAL;
    if (n == 0) return PKV_OK;
    if (!block_ids || !aligned(block_ids, 4)) return PKV_EINVAL;
    pkv::bm_free_kernel<<<1, pkv::kBmThreads, 0, (cudaStream_t)stream>>>(s, num_blocks, block_ids, n);
    return launch_status();
}

pkv_status pkv_bm_share(void *state, int32_t num_blocks, const int32_t *block_ids, int32_t n, pkv_stream_t stream) {
    pkv::BmState s;
    if (!bm_state(state, num_blocks, &s) || n < 0) return PKV_EINVAL;
    if (n == 0) return PKV_OK;
    if (!block_ids || !aligned(block_ids, 4)) return PKV_EINVAL;
    const int grid = std::max(1, std::min(1024, (n + 255) / 256));
    pkv::bm_share_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(s, num_blocks, block_ids, n);
    return launch_status();
}

pkv_status pkv_bm_append_slots(void *state, int32_t num_blocks, int32_t *block_tables, int32_t max_blocks_per_seq,
                               int32_t *context_lens, const int32_t *num_new, int32_t num_seqs, int32_t block_size,
                               int64_t *slot_mapping, int64_t slot_capacity, int32_t *cow_pairs,
                               int32_t *num_cow_pairs, pkv_stream_t stream) {
    pkv::AppendParams p;
    if (slot_capacity < 0) return PKV_EINVAL;
    if (!bm_state(state, num_blocks, &p.s) || num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0)
        return PKV_EINVAL;
    if ((long long)max_blocks_per_seq * block_size >= (1ll << 31)) return PKV_EUNSUPPORTED;
    if (!num_cow_pairs ||
        (num_seqs > 0 && (!block_tables || !context_lens || !num_new || !cow_pairs || !slot_mapping)))
        return PKV_EINVAL;
    if (!aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(num_new, 4) || !aligned(slot_mapping, 8) ||
        !aligned(cow_pairs, 4) || !aligned(num_cow_pairs, 4))
        return PKV_EINVAL;
    p.tables = block_tables;
    p.ctx = context_lens;
    p.num_new = num_new;
    p.slots = slot_mapping;
    p.slot_cap = slot_capacity;
    p.pairs = cow_pairs;
    p.num_pairs = num_cow_pairs;
    p.nb = num_blocks;
    p.mbs = max_blocks_per_seq;
    p.B = num_seqs;
    p.bs = block_size;
    // One thread per sequence, and enough for the slot pass to write at most
    // four slots per thread (the output capacity bounds the slots), rounded up
    // to a warp: a 128-sequence decode step runs on four warps.
    const int64_t want = std::max<int64_t>((int64_t)num_seqs, slot_capacity / 4);
    const int threads = (int)std::min<int64_t>(pkv::kBmThreads, std::max<int64_t>(32, (want + 31) / 32 * 32));
    pkv::bm_append_slots_kernel<<<1, threads, 0, (cudaStream_t)stream>>>(p);
    return launch_status();
}

pkv_status pkv_copy_blocks_dev(const int32_t *cow_pairs, const int32_t *num_pairs, int32_t max_pairs, void *k_cache,
                               void *v_cache, pkv_pool pool, pkv_stream_t stream) {
    const pkv_status ps = check_pool(pool);
    if (ps != PKV_OK) return ps;
    if (max_pairs < 0) return PKV_EINVAL;
    if (max_pairs == 0) return PKV_OK;
    if (!cow_pairs || !num_pairs || !k_cache || !v_cache) return PKV_EINVAL;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(cow_pairs, 4) || !aligned(num_pairs, 4))
        return PKV_EINVAL;
    const int64_t vec = (int64_t)pool.num_kv_heads * pool.block_size * pool.head_dim * elem_bytes(pool) / 16;
    const long long per_cta = pkv::kCopyDevThreads * pkv::kCopyDevVec;
    const unsigned gx = (unsigned)((vec + per_cta - 1) / per_cta);
    for (int base = 0; base < max_pairs; base += 65535) {  // grid.y limit
        const int m = std::min(65535, max_pairs - base);
        pkv::copy_blocks_dev_kernel<<<dim3(gx, m), pkv::kCopyDevThreads, 0, (cudaStream_t)stream>>>(
            static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), cow_pairs + 2 * base, num_pairs, vec,
            pool.num_blocks, base);
        const pkv_status st = launch_status();
        if (st != PKV_OK) return st;
    }
    return PKV_OK;
}

pkv_status pkv_get_device_error(int32_t *code_out, pkv_stream_t stream) {
    if (!code_out) return PKV_EINVAL;
    void *dptr = nullptr;
    if (cudaGetSymbolAddress(&dptr, pkv::g_device_error) != cudaSuccess) return PKV_ECUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    unsigned int h = 0;
    if (cudaMemcpyAsync(&h, dptr, sizeof h, cudaMemcpyDeviceToHost, st) != cudaSuccess) return PKV_ECUDA;
    if (cudaMemsetAsync(dptr, 0, sizeof h, st) != cudaSuccess) return PKV_ECUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return PKV_ECUDA;
    *code_out = (int32_t)h;
    return h ? PKV_EDEVICE : PKV_OK;
}

pkv_status pkv_selftest_bounded_wait(int64_t limit_ns, int32_t *result_dev, pkv_stream_t stream) {
    if (limit_ns <= 0 || limit_ns > 1000000000ll || !result_dev || !aligned(result_dev, 4)) return PKV_EINVAL;
    pkv::selftest_wait_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>((uint64_t)limit_ns, result_dev);
    return launch_status();
}

}  // extern "C"

// ------------------------------------------------- no-allocation variant ----
// Scratch for paged_attn_decode_static_ws: a file-scope device array, so the
// call needs no allocator.  Host code must not use the name as an address;
// the device address is looked up once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_static_workspace[PKV_STATIC_WS_BYTES];

namespace {
std::mutex g_static_ws_mutex;
void *g_static_ws_ptr[kMaxDevices] = {nullptr};
}  // namespace

extern "C" pkv_status paged_attn_decode_static_ws(const void *q, const void *k_cache, const void *v_cache,
                                                  const int32_t *block_tables, int32_t max_blocks_per_seq,
                                                  const int32_t *context_lens, int32_t num_seqs,
                                                  int32_t num_q_heads, float scale, int32_t num_kv_heads,
                                                  void *out, pkv_pool pool, int32_t max_context_len,
                                                  int32_t partition_tokens, pkv_stream_t stream) {
    const size_t need = pkv_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, pool.head_dim,
                                                   max_context_len, partition_tokens);
    if (need == 0) return PKV_EINVAL;
    if (need > PKV_STATIC_WS_BYTES) return PKV_EUNSUPPORTED;
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return PKV_ECUDA;
    void *ws = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_static_ws_mutex);
        if (g_static_ws_ptr[dev] == nullptr) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr) return PKV_ECUDA;
            g_static_ws_ptr[dev] = p;
        }
        ws = g_static_ws_ptr[dev];
    }
    return paged_attn_decode(q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                             num_q_heads, scale, num_kv_heads, out, pool, max_context_len, partition_tokens, ws,
                             PKV_STATIC_WS_BYTES, stream);
}
