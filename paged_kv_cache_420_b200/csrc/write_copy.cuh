// write_copy.cuh -- the slot-mapped KV write and the copy-on-write block copy.
// Both are pure data movement in 16-byte vectors: bit-exact by construction.
#pragma once

#include "ptx.cuh"

namespace pkv {

// ---------------------------------------------------------------- write ----
// One thread per 16-byte vector of one token row of K or V.  Thread order is
// (token, K/V, head, vector), so a warp reads 512 contiguous bytes of k or v
// and writes whole 256-byte (head_dim 128) rows of the pool.
//   slot -> block = slot / bs, offset = slot % bs   (position -> block, offset
//   rule of the PagedAttention sketch, ruibaoantu.com section 1.1)
struct WriteParams {
    const uint4 *k;        // [T][Hkv][D/8] vectors
    const uint4 *v;
    const int64_t *slots;  // [T]
    uint4 *k_cache;        // [NB][Hkv][bs][D/8]
    uint4 *v_cache;
    int64_t total;         // T * 2 * Hkv * vpr
    int64_t pool_slots;    // NB * bs
    int num_kv_heads;
    int block_size;
    int vpr;               // vectors per row = D / 8
};

__global__ void __launch_bounds__(256) kv_write_kernel(WriteParams p) {
    const int per_token = 2 * p.num_kv_heads * p.vpr;
    const int per_kv = p.num_kv_heads * p.vpr;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / per_token;
        const int rem = (int)(i - t * per_token);
        const int is_v = rem >= per_kv;
        const int j = rem - is_v * per_kv;  // head * vpr + vector
        const int64_t slot = __ldg(p.slots + t);
        if (slot < 0) continue;  // padding token
        if (slot >= p.pool_slots) {
            if (j == 0 && !is_v) raise_error(PKV_DEVERR_SLOT);
            continue;
        }
        const int64_t block = slot / p.block_size;
        const int offset = (int)(slot - block * p.block_size);
        const int h = j / p.vpr;
        const int c = j - h * p.vpr;
        const uint4 val = __ldg((is_v ? p.v : p.k) + t * per_kv + j);
        const int64_t dst = ((block * p.num_kv_heads + h) * p.block_size + offset) * p.vpr + c;
        (is_v ? p.v_cache : p.k_cache)[dst] = val;
    }
}

// ------------------------------------------------------------ fp8 write ----
// The same slot-mapped write into an FP8 (e4m3) pool: each 16-byte vector of
// 8 bf16 elements becomes 8 codes of fp32(x) * fp32(1 / scale[h]) (IEEE
// round-to-nearest reciprocal and product), converted with round-to-nearest-
// even and saturation to +-448.
struct WriteFp8Params {
    const uint4 *k;        // [T][Hkv][D] bf16 as 16-B vectors
    const uint4 *v;
    const int64_t *slots;  // [T]
    const float *k_scale;  // [Hkv]
    const float *v_scale;
    uint2 *k_cache;        // [NB][Hkv][bs][D] e4m3 as 8-B vectors
    uint2 *v_cache;
    int64_t total;         // T * 2 * Hkv * vpr
    int64_t pool_slots;
    int num_kv_heads;
    int block_size;
    int vpr;               // vectors per row = D / 8
};

__global__ void __launch_bounds__(256) kv_write_fp8_kernel(WriteFp8Params p) {
    const int per_token = 2 * p.num_kv_heads * p.vpr;
    const int per_kv = p.num_kv_heads * p.vpr;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / per_token;
        const int rem = (int)(i - t * per_token);
        const int is_v = rem >= per_kv;
        const int j = rem - is_v * per_kv;  // head * vpr + vector
        const int64_t slot = __ldg(p.slots + t);
        if (slot < 0) continue;  // padding token
        if (slot >= p.pool_slots) {
            if (j == 0 && !is_v) raise_error(PKV_DEVERR_SLOT);
            continue;
        }
        const int64_t block = slot / p.block_size;
        const int offset = (int)(slot - block * p.block_size);
        const int h = j / p.vpr;
        const int c = j - h * p.vpr;
        const float inv = __frcp_rn(__ldg((is_v ? p.v_scale : p.k_scale) + h));
        const uint4 val = __ldg((is_v ? p.v : p.k) + t * per_kv + j);
        const uint32_t w[4] = {val.x, val.y, val.z, val.w};
        uint32_t code[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const float x0 = __fmul_rn(bf16lo_to_f32(w[2 * u]), inv), x1 = __fmul_rn(bf16hi_to_f32(w[2 * u]), inv);
            const float x2 = __fmul_rn(bf16lo_to_f32(w[2 * u + 1]), inv);
            const float x3 = __fmul_rn(bf16hi_to_f32(w[2 * u + 1]), inv);
            code[u] = e4m3x2_from_f32(x0, x1) | (e4m3x2_from_f32(x2, x3) << 16);
        }
        const int64_t dst = ((block * p.num_kv_heads + h) * p.block_size + offset) * p.vpr + c;
        (is_v ? p.v_cache : p.k_cache)[dst] = make_uint2(code[0], code[1]);
    }
}

// ----------------------------------------------------------------- copy ----
// Pairs travel by value in the kernel parameters (validated on the host),
// in a parameter block of CAP pairs: the host picks the smallest of 32, 256
// and 1024 that holds a launch's pairs (the launch latency grows with the
// parameter bytes: 8 KB cost about 1 us more than 2 KB for 256 pairs).
// grid.y = pair, grid.x = chunk of the block; each thread moves kVecPerThread
// vectors of K and of V, loads first, then stores.
constexpr int kMaxPairsPerLaunch = 1024;  // 8 KB of parameters
constexpr int kCopyThreads = 256;
constexpr int kCopyVecPerThread = 4;

template <int CAP>
struct CopyParams {
    uint4 *k_cache;
    uint4 *v_cache;
    int64_t vec_per_block;  // Hkv * bs * D / 8
    int num_pairs;
    int2 pairs[CAP];
};

template <int CAP>
__global__ void __launch_bounds__(kCopyThreads) copy_blocks_kernel(const __grid_constant__ CopyParams<CAP> p) {
    const int pair = blockIdx.y;
    const int64_t src = (int64_t)p.pairs[pair].x * p.vec_per_block;
    const int64_t dst = (int64_t)p.pairs[pair].y * p.vec_per_block;
    const int64_t base = (int64_t)blockIdx.x * (kCopyThreads * kCopyVecPerThread) + threadIdx.x;
    uint4 kv[kCopyVecPerThread], vv[kCopyVecPerThread];
#pragma unroll
    for (int u = 0; u < kCopyVecPerThread; ++u) {
        const int64_t e = base + u * kCopyThreads;
        if (e < p.vec_per_block) {
            kv[u] = p.k_cache[src + e];
            vv[u] = p.v_cache[src + e];
        }
    }
#pragma unroll
    for (int u = 0; u < kCopyVecPerThread; ++u) {
        const int64_t e = base + u * kCopyThreads;
        if (e < p.vec_per_block) {
            p.k_cache[dst + e] = kv[u];
            p.v_cache[dst + e] = vv[u];
        }
    }
}

// ----------------------------------------------------------------- swap ----
// Whole blocks (all heads, K and V) between the pool and host memory that the
// device can address (pinned, mapped through unified addressing).  Block ids
// travel by value; grid.y = list position, grid.x = chunk of the block.
// OUT gathers pool blocks into the packed host arrays [n][Hkv][bs][D]; IN
// scatters them back.  Each thread keeps kSwapVecPerThread 16-byte vectors of
// K and of V in flight (host memory is far: loads first, then stores).
constexpr int kMaxSwapPerLaunch = 2048;  // 8 KB of parameters
constexpr int kSwapThreads = 256;
constexpr int kSwapVecPerThread = 4;

struct SwapParams {
    uint4 *pool_k;
    uint4 *pool_v;
    uint4 *host_k;  // first block of this launch
    uint4 *host_v;
    int64_t vec_per_block;  // Hkv * bs * D / 8
    int n;
    int32_t ids[kMaxSwapPerLaunch];
};

template <bool OUT>
__global__ void __launch_bounds__(kSwapThreads) swap_blocks_kernel(const __grid_constant__ SwapParams p) {
    const int i = blockIdx.y;
    const int64_t pool_off = (int64_t)p.ids[i] * p.vec_per_block;
    const int64_t host_off = (int64_t)i * p.vec_per_block;
    const uint4 *sk = OUT ? p.pool_k + pool_off : p.host_k + host_off;
    const uint4 *sv = OUT ? p.pool_v + pool_off : p.host_v + host_off;
    uint4 *dk = OUT ? p.host_k + host_off : p.pool_k + pool_off;
    uint4 *dv = OUT ? p.host_v + host_off : p.pool_v + pool_off;
    const int64_t base = (int64_t)blockIdx.x * (kSwapThreads * kSwapVecPerThread) + threadIdx.x;
    uint4 kv[kSwapVecPerThread], vv[kSwapVecPerThread];
#pragma unroll
    for (int u = 0; u < kSwapVecPerThread; ++u) {
        const int64_t e = base + u * kSwapThreads;
        if (e < p.vec_per_block) {
            kv[u] = sk[e];
            vv[u] = sv[e];
        }
    }
#pragma unroll
    for (int u = 0; u < kSwapVecPerThread; ++u) {
        const int64_t e = base + u * kSwapThreads;
        if (e < p.vec_per_block) {
            dk[e] = kv[u];
            dv[e] = vv[u];
        }
    }
}

}  // namespace pkv
