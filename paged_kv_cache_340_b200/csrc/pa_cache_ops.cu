// Cache-side kernels: the slot write of new tokens and the copy-on-write
// block copy. Both are bit copies moved in 16-byte vectors; HBM-bound.
#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

// Slot write ([P3 "Ascend C ... PagedAttention融合算子", §3.1 and §4.2:
// block = slot / block_size, offset = slot % block_size]; [P4 "PagedAttention
// 实现细节", §3.4: each new token's K/V goes into its block).
// A token's K (or V) is num_kv_heads rows of 2^kVShift 16-byte vectors, in the
// source contiguous (per_token vectors) and in the pool one row per kv head.
// Thread t of a CTA always moves vector j of (token group member) tin, with
// (tin, j) fixed for the whole kernel, so no index is divided in the loop:
// CTAs of 256 threads take tpi = 256 / per_token tokens at a time when a
// token has at most 256 vectors, else one token in rounds of 256 vectors.
// Each thread keeps kU tokens' (or rounds') loads in flight before storing.
template <int kVShift>
__global__ void __launch_bounds__(256)
    reshape_and_cache_kernel(const uint4 *__restrict__ key, const uint4 *__restrict__ value,
                             uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                             const int32_t *__restrict__ slot_mapping, int num_tokens,
                             int num_blocks, int num_kv_heads, int bs_shift, unsigned int *err) {
    constexpr int kU = 4;
    const int per_token = num_kv_heads << kVShift;
    const long long slots = (long long)num_blocks << bs_shift;
    // one 16-byte vector: source index, token, vector j within the token
    auto move_one = [&](int token, int j, uint4 &kr, uint4 &vr, long long &dst) {
        dst = -1;
        if (token >= num_tokens) return;
        const int slot = __ldg(slot_mapping + token);
        if (slot < 0) return;
        if (slot >= slots) {
            if (j == 0) record_error(err, PA_DEVERR_SLOT);
            return;
        }
        const int h = j >> kVShift;
        const int v = j & ((1 << kVShift) - 1);
        const long long block = slot >> bs_shift;
        const int offset = slot & ((1 << bs_shift) - 1);
        dst = ((((block * num_kv_heads + h) << bs_shift) + offset) << kVShift) + v;
        const size_t src = (size_t)token * per_token + j;
        kr = __ldg(key + src);
        vr = __ldg(value + src);
    };
    if (per_token <= 256) {
        const int tpi = 256 / per_token;  // tokens per CTA round
        const int tin = threadIdx.x / per_token;
        const int j = threadIdx.x - tin * per_token;
        if (tin >= tpi) return;
        const int step = gridDim.x * tpi;
        for (int t0 = blockIdx.x * tpi + tin; t0 < num_tokens; t0 += kU * step) {
            uint4 kr[kU], vr[kU];
            long long dst[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) move_one(t0 + u * step, j, kr[u], vr[u], dst[u]);
#pragma unroll
            for (int u = 0; u < kU; ++u)
                if (dst[u] >= 0) {
                    k_cache[dst[u]] = kr[u];
                    v_cache[dst[u]] = vr[u];
                }
        }
    } else {
        for (int token = blockIdx.x; token < num_tokens; token += gridDim.x) {
            for (int j0 = threadIdx.x; j0 < per_token; j0 += kU * 256) {
                uint4 kr[kU], vr[kU];
                long long dst[kU];
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    dst[u] = -1;
                    if (j0 + u * 256 < per_token) move_one(token, j0 + u * 256, kr[u], vr[u], dst[u]);
                }
#pragma unroll
                for (int u = 0; u < kU; ++u)
                    if (dst[u] >= 0) {
                        k_cache[dst[u]] = kr[u];
                        v_cache[dst[u]] = vr[u];
                    }
            }
        }
    }
}

// Copy-on-write block copy ([P4 "PagedAttention 实现细节", §3.3]): grid.x walks
// the pairs, grid.y picks K (0) or V (1), grid.z splits a block into chunks.
__global__ void __launch_bounds__(256)
    copy_blocks_kernel(uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                       const int64_t *__restrict__ pairs, const int32_t *__restrict__ pair_count,
                       int num_blocks, long long vecs_per_block, unsigned int *err) {
    if (pair_count && (int)blockIdx.x >= __ldg(pair_count)) return;  // past the device-side count
    const int64_t src = __ldg(pairs + 2 * blockIdx.x);
    const int64_t dst = __ldg(pairs + 2 * blockIdx.x + 1);
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) record_error(err, PA_DEVERR_PAIR);
        return;
    }
    uint4 *pool = blockIdx.y == 0 ? k_cache : v_cache;
    const uint4 *s = pool + src * vecs_per_block;
    uint4 *d = pool + dst * vecs_per_block;
    const long long chunk = (vecs_per_block + gridDim.z - 1) / gridDim.z;
    const long long begin = blockIdx.z * chunk;
    const long long end = min(begin + chunk, vecs_per_block);
    // kU loads in flight per thread before their stores (the read-only path
    // is safe: within a call no block is both copied from and written to)
    constexpr int kU = 8;
    long long i = begin + threadIdx.x;
    for (; i + (kU - 1) * (long long)blockDim.x < end; i += kU * (long long)blockDim.x) {
        uint4 r[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) r[u] = __ldg(s + i + u * blockDim.x);
#pragma unroll
        for (int u = 0; u < kU; ++u) d[i + u * blockDim.x] = r[u];
    }
    for (; i < end; i += blockDim.x) d[i] = s[i];
}

cudaError_t launch_reshape_and_cache(const void *key, const void *value, void *k_cache,
                                     void *v_cache, const int32_t *slot_mapping, int num_tokens,
                                     int num_blocks, int num_kv_heads, int row_bytes,
                                     int block_size, unsigned int *err, cudaStream_t stream) {
    if (num_tokens == 0) return cudaSuccess;
    const int vecs_per_row = row_bytes / 16;  // 8, 16 or 32
    const int bs_shift = block_size == 16 ? 4 : 5;
    if ((long long)num_kv_heads * vecs_per_row > INT_MAX / 2) return cudaErrorInvalidValue;
    const int per_token = num_kv_heads * vecs_per_row;
    const long long tpi = per_token <= 256 ? 256 / per_token : 1;
    long long blocks = (num_tokens + tpi - 1) / tpi;  // one token (or one token's rounds) a thread, up to the cap
    const long long cap = (long long)sm_count() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    const uint4 *k = static_cast<const uint4 *>(key), *v = static_cast<const uint4 *>(value);
    uint4 *kc = static_cast<uint4 *>(k_cache), *vc = static_cast<uint4 *>(v_cache);
    switch (vecs_per_row) {
        case 8:
            reshape_and_cache_kernel<3><<<(unsigned)blocks, 256, 0, stream>>>(k, v, kc, vc, slot_mapping, num_tokens,
                                                                              num_blocks, num_kv_heads, bs_shift, err);
            break;
        case 16:
            reshape_and_cache_kernel<4><<<(unsigned)blocks, 256, 0, stream>>>(k, v, kc, vc, slot_mapping, num_tokens,
                                                                              num_blocks, num_kv_heads, bs_shift, err);
            break;
        case 32:
            reshape_and_cache_kernel<5><<<(unsigned)blocks, 256, 0, stream>>>(k, v, kc, vc, slot_mapping, num_tokens,
                                                                              num_blocks, num_kv_heads, bs_shift, err);
            break;
        default:
            return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_copy_blocks(void *k_cache, void *v_cache, const int64_t *pairs, int num_pairs,
                               const int32_t *pair_count, int num_blocks, size_t block_bytes,
                               unsigned int *err, cudaStream_t stream) {
    if (num_pairs == 0) return cudaSuccess;
    const long long vecs = (long long)(block_bytes / 16);
    // about 32 KiB per CTA
    long long chunks = (vecs + 2047) / 2048;
    if (chunks < 1) chunks = 1;
    if (chunks > 65535) chunks = 65535;
    dim3 grid((unsigned)num_pairs, 2, (unsigned)chunks);
    copy_blocks_kernel<<<grid, 256, 0, stream>>>(static_cast<uint4 *>(k_cache),
                                                 static_cast<uint4 *>(v_cache), pairs, pair_count,
                                                 num_blocks, vecs, err);
    return cudaGetLastError();
}

}  // namespace pa

namespace pa {

// Slot write into an int8 cache: one warp per (token, kv head) row. The row's
// largest magnitude sets the scale; codes are round-half-even(x * (127 /
// amax)), clamped to +-127, every step one IEEE fp32 operation (the same
// arithmetic wherever it runs); scale = amax / 127; a zero row gives codes 0
// and scale 0. The pages name int8 KV storage without a scheme; this is the
// library's (symmetric, per token and kv head).
template <typename TS, int D>
__global__ void __launch_bounds__(256)
    reshape_and_cache_q8_kernel(const TS *__restrict__ key, const TS *__restrict__ value, int8_t *__restrict__ k_cache,
                                int8_t *__restrict__ v_cache, float *__restrict__ k_scale, float *__restrict__ v_scale,
                                const int32_t *__restrict__ slot_mapping, int num_tokens, int num_blocks,
                                int num_kv_heads, int block_size, unsigned int *err) {
    constexpr int kPer = D / 32;  // values per lane
    const int lane = threadIdx.x & 31;
    const long long rows = (long long)num_tokens * num_kv_heads;
    const long long slots = (long long)num_blocks * block_size;
    for (long long row = (blockIdx.x * (long long)blockDim.x + threadIdx.x) / 32; row < rows;
         row += (long long)gridDim.x * blockDim.x / 32) {
        const int token = (int)(row / num_kv_heads);
        const int h = (int)(row - (long long)token * num_kv_heads);
        const int slot = __ldg(slot_mapping + token);
        if (slot < 0) continue;
        if (slot >= slots) {
            if (h == 0 && lane == 0) record_error(err, PA_DEVERR_SLOT);
            continue;
        }
        const int block = slot / block_size;
        const int offset = slot - block * block_size;
        const size_t srow = ((size_t)block * num_kv_heads + h) * block_size + offset;
#pragma unroll
        for (int kv = 0; kv < 2; ++kv) {
            const TS *src = (kv == 0 ? key : value) + row * D + lane * kPer;
            float x[kPer];
#pragma unroll
            for (int e = 0; e < kPer; ++e) x[e] = static_cast<float>(src[e]);
            float amax = 0.f;
#pragma unroll
            for (int e = 0; e < kPer; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
            for (int mk = 16; mk >= 1; mk >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, mk));
            uint32_t packed = 0;
            if (amax > 0.f) {
                const float inv = __fdiv_rn(127.f, amax);
#pragma unroll
                for (int e = 0; e < kPer; ++e) {
                    int qv = __float2int_rn(__fmul_rn(x[e], inv));
                    qv = max(-127, min(127, qv));
                    packed |= (uint32_t)(qv & 0xff) << (8 * e);
                }
            }
            int8_t *dst = (kv == 0 ? k_cache : v_cache) + srow * D + lane * kPer;
            if constexpr (kPer == 4)
                *reinterpret_cast<uint32_t *>(dst) = packed;
            else
                *reinterpret_cast<uint16_t *>(dst) = (uint16_t)packed;
            if (lane == 0) (kv == 0 ? k_scale : v_scale)[srow] = amax > 0.f ? __fdiv_rn(amax, 127.f) : 0.f;
        }
    }
}

template <typename TS>
static cudaError_t launch_q8_t(const void *key, const void *value, int8_t *k_cache, int8_t *v_cache, float *k_scale,
                               float *v_scale, const int32_t *slot_mapping, int num_tokens, int num_blocks,
                               int num_kv_heads, int head_dim, int block_size, unsigned int *err, cudaStream_t stream) {
    const long long rows = (long long)num_tokens * num_kv_heads;
    long long blocks = (rows * 32 + 255) / 256;
    const long long cap = (long long)sm_count() * 8;
    if (blocks > cap) blocks = cap;
    if (head_dim == 128)
        reshape_and_cache_q8_kernel<TS, 128><<<(unsigned)blocks, 256, 0, stream>>>(
            static_cast<const TS *>(key), static_cast<const TS *>(value), k_cache, v_cache, k_scale, v_scale,
            slot_mapping, num_tokens, num_blocks, num_kv_heads, block_size, err);
    else
        reshape_and_cache_q8_kernel<TS, 64><<<(unsigned)blocks, 256, 0, stream>>>(
            static_cast<const TS *>(key), static_cast<const TS *>(value), k_cache, v_cache, k_scale, v_scale,
            slot_mapping, num_tokens, num_blocks, num_kv_heads, block_size, err);
    return cudaGetLastError();
}

cudaError_t launch_reshape_and_cache_q8(const void *key, const void *value, pa_dtype src_dtype, int8_t *k_cache,
                                        int8_t *v_cache, float *k_scale, float *v_scale,
                                        const int32_t *slot_mapping, int num_tokens, int num_blocks,
                                        int num_kv_heads, int head_dim, int block_size, unsigned int *err,
                                        cudaStream_t stream) {
    if (num_tokens == 0) return cudaSuccess;
    switch (src_dtype) {
        case PA_F32: return launch_q8_t<float>(key, value, k_cache, v_cache, k_scale, v_scale, slot_mapping, num_tokens, num_blocks, num_kv_heads, head_dim, block_size, err, stream);
        case PA_F16: return launch_q8_t<__half>(key, value, k_cache, v_cache, k_scale, v_scale, slot_mapping, num_tokens, num_blocks, num_kv_heads, head_dim, block_size, err, stream);
        case PA_BF16: return launch_q8_t<__nv_bfloat16>(key, value, k_cache, v_cache, k_scale, v_scale, slot_mapping, num_tokens, num_blocks, num_kv_heads, head_dim, block_size, err, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pa
