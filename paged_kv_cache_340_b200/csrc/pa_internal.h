// Internal interfaces between the C-ABI layer (pa_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "pa.h"

namespace pa {

struct DecodeParams {
    void *out;          // unpartitioned: [num_seqs, num_heads, head_dim] of out_dtype
    float *ws_ml;       // split-K: [num_seqs, num_heads, max_parts, 2] (m, l)
    float *ws_acc;      // split-K: [num_seqs, num_heads, max_parts, head_dim]
    const void *query;  // [num_seqs, num_heads, head_dim]
    const void *k_cache;
    const void *v_cache;
    const float *k_scale;  // int8 caches: [num_blocks, num_kv_heads, block_size] per-row scales
    const float *v_scale;
    const int32_t *block_tables;
    const int32_t *context_lens;
    const int32_t *seq_order;  // nullable: CTA row z serves sequence seq_order[z]
    int max_blocks_per_seq;
    int num_heads;
    int num_kv_heads;
    int num_blocks;
    // head group: query heads per kv head (num_heads / num_kv_heads). A CTA
    // serves up to the kernel's compiled group size G of them (a power of two
    // >= the group, padded with zero queries whose outputs are not written);
    // a group larger than G is served by sub_groups CTAs of G heads each,
    // adjacent along gridDim.y (kv head = blockIdx.y / sub_groups).
    int group = 1;
    int sub_groups = 1;
    float scale_log2;    // scale * log2(e)
    int partition_size;  // 0: one CTA covers the whole sequence
    int max_parts;
    int max_context_len;
    pa_dtype out_dtype;
    unsigned int *err;   // device error word
    // nullable (16-bit and fp32 caches): the newest token of every sequence
    // (position context_len - 1), [num_seqs, num_kv_heads, head_dim] each,
    // written into the slot its table gives and used in place of the pool's
    // copy (pa_decode_append)
    const void *new_key;
    const void *new_value;
    // Prefill on the CUDA cores (pa_prefill over an fp32 cache): when q_start
    // (device int32 [num_seqs + 1]) is set, blockIdx.x is a query token t
    // (the grid has one CTA column per token and no partitions); its sequence
    // s has q_start[s] <= t < q_start[s + 1], and it attends to cache tokens
    // 0 .. context_lens[s] - q_len_s + (t - q_start[s]). query and out rows
    // are tokens; the table row and context are the sequence's.
    const int32_t *q_start = nullptr;
    int num_seqs = 0;
    // Test hook of the bounded waits (pa_decode_withhold_stage): the CTA of
    // sequence withhold_seq, kv head withhold_kvh (partition 0) never issues
    // the copy of its 16-token stage withhold_stage, so that stage's wait runs
    // out; every wait of the launch gives up after wait_limit_ns (0: the
    // default bound). withhold_seq = -1 withholds nothing.
    int withhold_seq = -1;
    int withhold_kvh = -1;
    int withhold_stage = -1;
    unsigned long long wait_limit_ns = 0;
    // The tensor-core consumers (int8 caches with head_dim 128; 16-bit caches
    // with head groups of two or more, set by launch_decode): the V pool as
    // 2-D rows, boxes of 128 bytes x 16 rows in the 128-byte swizzled layout
    // (the kernel's V fragment loads are then free of shared-memory bank
    // conflicts)
    alignas(64) CUtensorMap v_map;
    // The 16-bit tensor-core consumer: the K pool the same way (set by
    // launch_decode)
    alignas(64) CUtensorMap k_map;
};

cudaError_t launch_decode(const DecodeParams &p, pa_dtype kv_dtype, int head_dim, int block_size,
                          int group, int grid_x, int num_kv_heads, int num_seqs,
                          cudaStream_t stream);

// int8 caches (codes plus per-row scales in p.k_scale / p.v_scale); q_dtype is
// the query's type (PA_F16 or PA_BF16).
cudaError_t launch_decode_q8(const DecodeParams &p, pa_dtype q_dtype, int head_dim, int block_size, int group,
                             int grid_x, int num_kv_heads, int num_seqs, cudaStream_t stream);

cudaError_t launch_reshape_and_cache_q8(const void *key, const void *value, pa_dtype src_dtype, int8_t *k_cache,
                                        int8_t *v_cache, float *k_scale, float *v_scale,
                                        const int32_t *slot_mapping, int num_tokens, int num_blocks,
                                        int num_kv_heads, int head_dim, int block_size, unsigned int *err,
                                        cudaStream_t stream);

cudaError_t launch_splitk_reduce(void *out, const float *ws_ml, const float *ws_acc,
                                 const int32_t *context_lens, int num_seqs, int num_heads,
                                 int head_dim, int partition_size, int max_parts,
                                 int max_context_len, pa_dtype out_dtype, cudaStream_t stream);

cudaError_t launch_reshape_and_cache(const void *key, const void *value, void *k_cache,
                                     void *v_cache, const int32_t *slot_mapping, int num_tokens,
                                     int num_blocks, int num_kv_heads, int row_bytes,
                                     int block_size, unsigned int *err, cudaStream_t stream);

// pair_count (nullable, device): only the first *pair_count of num_pairs pairs are copied.
cudaError_t launch_copy_blocks(void *k_cache, void *v_cache, const int64_t *pairs, int num_pairs,
                               const int32_t *pair_count, int num_blocks, size_t block_bytes,
                               unsigned int *err, cudaStream_t stream);

cudaError_t launch_dpool_init(int32_t *state, int num_blocks, int block_size, int policy,
                              const int32_t *free_order, unsigned int *err, cudaStream_t stream);

cudaError_t launch_dpool_load(int32_t *state, int num_blocks, int block_size, int policy, const int32_t *ref_counts,
                              const int32_t *free_list, int num_free, unsigned int *err, cudaStream_t stream);

// withhold_cta >= 0: the test hook (pa_beam_step_withhold_arrival), one-launch form only.
cudaError_t launch_beam_step(int32_t *state, const int32_t *old_tables, const int32_t *old_ctx, int num_old,
                             const int32_t *parents, int num_new, int32_t *new_tables, int32_t *new_ctx,
                             int max_blocks, int32_t *slots, int64_t *cow_pairs, int32_t *num_cow,
                             int num_blocks, int block_size, unsigned int *err, cudaStream_t stream,
                             int withhold_cta = -1, unsigned long long barrier_limit_ns = 0);

// A rank-2 TMA tensor map over `rows` rows of `inner` elements (row stride in
// bytes), box box_inner x box_rows, zero fill. False if the encoder is
// unavailable or refuses the shape.
bool encode_rows_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, unsigned long long inner,
                    unsigned long long rows, unsigned long long row_stride_bytes, unsigned box_inner,
                    unsigned box_rows, CUtensorMapSwizzle swizzle);

// Per-device caches of the host side (symbol addresses, kernel attributes)
// are keyed by the device's current CUDA context, so that a context torn down
// and made again (cudaDeviceReset) is noticed and the entry refreshed.
constexpr int kCacheDevices = 64;

struct SymbolCache {
    std::atomic<void *> ctx[kCacheDevices];
    std::atomic<void *> addr[kCacheDevices];
};

struct AttrCache {
    std::atomic<void *> ctx[kCacheDevices];
};

// The calling thread's current CUDA context (driver handle), or nullptr.
void *current_context();

// Device address of a __device__ variable (its host-side stand-in `symbol`)
// on the current device, looked up once per context.
cudaError_t symbol_address(const void *symbol, SymbolCache *cache, void **addr);

// Device address of the current device's error word.
cudaError_t device_error_word(unsigned int **word);

// pa_prefill over an fp32 cache: the decode kernel with one CTA column per
// query token (see DecodeParams::q_start). Arguments as pa_prefill.
int prefill_cuda_cores(void *out, const void *query, const int32_t *q_start, int num_tokens, const void *k_cache,
                       const void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                       const int32_t *context_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                       float scale, int block_size, int num_blocks, cudaStream_t stream);

// Number of SMs of the current device.
int sm_count();

// Sets the dynamic shared memory limit of `func` once per device context.
cudaError_t ensure_smem_attr(const void *func, int bytes, AttrCache *done);

}  // namespace pa
