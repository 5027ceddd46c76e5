// C-ABI entry points of the device operations: host-side argument checks,
// dispatch, the device error word and the split-K workspace layout.
#include <atomic>
#include <climits>
#include <cmath>
#include <mutex>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

__device__ unsigned int g_device_errors = 0;

static constexpr int kMaxDevices = 64;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

void *current_context() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(f);
    });
    CUcontext c = nullptr;
    if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

cudaError_t symbol_address(const void *symbol, SymbolCache *cache, void **addr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    void *ctx = current_context();
    if (ctx != nullptr && cache->ctx[dev].load(std::memory_order_acquire) == ctx) {
        *addr = cache->addr[dev].load(std::memory_order_relaxed);
        return cudaSuccess;
    }
    void *a = nullptr;
    e = cudaGetSymbolAddress(&a, symbol);  // loads the module on its first use in this context
    if (e != cudaSuccess) return e;
    ctx = current_context();
    // address first, then the context it belongs to (readers check the context)
    cache->addr[dev].store(a, std::memory_order_relaxed);
    cache->ctx[dev].store(ctx, std::memory_order_release);
    *addr = a;
    return cudaSuccess;
}

cudaError_t device_error_word(unsigned int **word) {
    static SymbolCache cache;
    void *a = nullptr;
    cudaError_t e = symbol_address(&g_device_errors, &cache, &a);
    if (e == cudaSuccess) *word = static_cast<unsigned int *>(a);
    return e;
}

int sm_count() {
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

cudaError_t ensure_smem_attr(const void *func, int bytes, AttrCache *done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    void *ctx = current_context();
    if (ctx != nullptr && done->ctx[dev].load(std::memory_order_acquire) == ctx) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    done->ctx[dev].store(current_context(), std::memory_order_release);
    return cudaSuccess;
}

static int elt_bytes(pa_dtype dt) {
    switch (dt) {
        case PA_F32: return 4;
        case PA_F16: return 2;
        case PA_BF16: return 2;
    }
    return 0;
}

static bool aligned(const void *p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

// Checks shared by the decode entry points.
static int check_decode_args(const void *query, const void *k_cache, const void *v_cache,
                             const int32_t *block_tables, int max_blocks_per_seq,
                             const int32_t *context_lens, int num_seqs, int num_heads,
                             int num_kv_heads, int head_dim, float scale, int block_size,
                             int num_blocks, pa_dtype kv_dtype) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_blocks < 0 ||
        max_blocks_per_seq < 0 || num_seqs > 65535 || num_kv_heads > 65535 || !std::isfinite(scale))
        return PA_ERR_SHAPE;
    if (elt_bytes(kv_dtype) == 0) return PA_ERR_DTYPE;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_HEAD_DIM;
    if (block_size != 16 && block_size != 32) return PA_ERR_BLOCK_SIZE;
    if (num_heads % num_kv_heads != 0) return PA_ERR_HEADS;
    const int group = num_heads / num_kv_heads;
    // a group above 8 runs as sub-groups of 8 query heads, one CTA each along gridDim.y
    if ((long long)num_kv_heads * ((group + 7) / 8) > 65535) return PA_ERR_SHAPE;
    if (max_blocks_per_seq > INT_MAX / block_size) return PA_ERR_SHAPE;
    if (num_seqs == 0) return PA_OK;
    if (!query || !k_cache || !v_cache || !block_tables || !context_lens) return PA_ERR_NULL;
    if (!aligned(query, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4))
        return PA_ERR_ALIGN;
    return PA_OK;
}

static int max_parts_of(int max_context_len, int partition_size) {
    return (max_context_len + partition_size - 1) / partition_size;
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static size_t ml_bytes(int num_seqs, int num_heads, int max_parts) {
    return (size_t)num_seqs * num_heads * max_parts * 2 * sizeof(float);
}

}  // namespace pa

using namespace pa;

extern "C" {

const char *pa_status_string(int status) {
    switch (status) {
        case PA_OK: return "ok";
        case PA_ERR_NULL: return "a required pointer is NULL";
        case PA_ERR_DTYPE: return "unsupported element or output type";
        case PA_ERR_SHAPE: return "a size is negative, too large or inconsistent";
        case PA_ERR_HEADS: return "num_heads must be a multiple of num_kv_heads";
        case PA_ERR_HEAD_DIM: return "head_dim must be 64 or 128";
        case PA_ERR_BLOCK_SIZE: return "block_size must be 16 or 32";
        case PA_ERR_ALIGN: return "a device pointer is not 16-byte aligned";
        case PA_ERR_PARTITION: return "partition_size must be a positive multiple of block_size";
        case PA_ERR_WORKSPACE: return "workspace is missing or smaller than pa_splitk_workspace_bytes()";
        case PA_ERR_CUDA: return "a CUDA call or kernel launch failed";
        case PA_ERR_POOL_EXHAUSTED: return "block pool has no free block";
        case PA_ERR_POOL_STATE: return "block id out of range or block already free";
        case PA_ERR_CAPACITY: return "table row or output array too small";
    }
    return "unknown status";
}

int pa_read_device_errors(uint32_t *flags, cudaStream_t stream) {
    if (!flags) return PA_ERR_NULL;
    unsigned int *word = nullptr;
    if (device_error_word(&word) != cudaSuccess) return PA_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return PA_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpy(&v, word, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return PA_ERR_CUDA;
    if (cudaMemset(word, 0, sizeof(v)) != cudaSuccess) return PA_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return PA_ERR_CUDA;
    *flags = v;
    return PA_OK;
}

int pa_reshape_and_cache(const void *key, const void *value, void *k_cache, void *v_cache,
                         const int32_t *slot_mapping, int num_tokens, int num_blocks,
                         int num_kv_heads, int head_dim, int block_size, pa_dtype kv_dtype,
                         cudaStream_t stream) {
    if (num_tokens < 0 || num_blocks < 0 || num_kv_heads <= 0) return PA_ERR_SHAPE;
    const int eb = elt_bytes(kv_dtype);
    if (eb == 0) return PA_ERR_DTYPE;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_HEAD_DIM;
    if (block_size != 16 && block_size != 32) return PA_ERR_BLOCK_SIZE;
    if ((long long)num_blocks * block_size > INT_MAX) return PA_ERR_SHAPE;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_NULL;
    if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(slot_mapping, 4))
        return PA_ERR_ALIGN;
    unsigned int *err = nullptr;
    if (device_error_word(&err) != cudaSuccess) return PA_ERR_CUDA;
    cudaError_t e = launch_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, num_tokens,
                                             num_blocks, num_kv_heads, head_dim * eb, block_size,
                                             err, stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// The test hook of pa_decode_withhold_stage (none by default).
struct WithholdHook {
    int seq = -1, kv_head = -1, stage = -1;
    unsigned long long wait_limit_ns = 0;
};

static int decode_unsplit(void *out, const void *query, const void *new_key, const void *new_value,
                          const void *k_cache, const void *v_cache, const int32_t *block_tables,
                          int max_blocks_per_seq, const int32_t *context_lens, int num_seqs, int num_heads,
                          int num_kv_heads, int head_dim, float scale, int block_size, int num_blocks,
                          pa_dtype kv_dtype, pa_dtype out_dtype, const int32_t *seq_order, cudaStream_t stream,
                          const WithholdHook &hook = WithholdHook()) {
    int rc = check_decode_args(query, k_cache, v_cache, block_tables, max_blocks_per_seq,
                               context_lens, num_seqs, num_heads, num_kv_heads, head_dim, scale,
                               block_size, num_blocks, kv_dtype);
    if (rc != PA_OK) return rc;
    if (out_dtype != kv_dtype && out_dtype != PA_F32) return PA_ERR_DTYPE;
    if (num_seqs == 0) return PA_OK;
    if (!aligned(seq_order, 4)) return PA_ERR_ALIGN;
    if (!out) return PA_ERR_NULL;
    if (!aligned(out, 16) || !aligned(new_key, 16) || !aligned(new_value, 16)) return PA_ERR_ALIGN;
    unsigned int *err = nullptr;
    if (device_error_word(&err) != cudaSuccess) return PA_ERR_CUDA;
    DecodeParams p{};
    p.out = out;
    p.query = query;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.seq_order = seq_order;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.num_blocks = num_blocks;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.partition_size = 0;
    p.max_parts = 1;
    p.max_context_len = INT_MAX;
    p.out_dtype = out_dtype;
    p.err = err;
    p.new_key = new_key;
    p.new_value = new_value;
    p.withhold_seq = hook.seq;
    p.withhold_kvh = hook.kv_head;
    p.withhold_stage = hook.stage;
    p.wait_limit_ns = hook.wait_limit_ns;
    cudaError_t e = launch_decode(p, kv_dtype, head_dim, block_size, num_heads / num_kv_heads, 1,
                                  num_kv_heads, num_seqs, stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_decode(void *out, const void *query, const void *k_cache, const void *v_cache,
              const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
              int num_seqs, int num_heads, int num_kv_heads, int head_dim, float scale,
              int block_size, int num_blocks, pa_dtype kv_dtype, pa_dtype out_dtype,
              const int32_t *seq_order, cudaStream_t stream) {
    return decode_unsplit(out, query, nullptr, nullptr, k_cache, v_cache, block_tables, max_blocks_per_seq,
                          context_lens, num_seqs, num_heads, num_kv_heads, head_dim, scale, block_size,
                          num_blocks, kv_dtype, out_dtype, seq_order, stream);
}

int pa_decode_append(void *out, const void *query, const void *new_key, const void *new_value, void *k_cache,
                     void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                     const int32_t *context_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                     float scale, int block_size, int num_blocks, pa_dtype kv_dtype, pa_dtype out_dtype,
                     const int32_t *seq_order, cudaStream_t stream) {
    if (num_seqs > 0 && (!new_key || !new_value)) return PA_ERR_NULL;
    return decode_unsplit(out, query, new_key, new_value, k_cache, v_cache, block_tables, max_blocks_per_seq,
                          context_lens, num_seqs, num_heads, num_kv_heads, head_dim, scale, block_size,
                          num_blocks, kv_dtype, out_dtype, seq_order, stream);
}

}  // extern "C"

namespace pa {

int prefill_cuda_cores(void *out, const void *query, const int32_t *q_start, int num_tokens, const void *k_cache,
                       const void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                       const int32_t *context_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                       float scale, int block_size, int num_blocks, cudaStream_t stream) {
    int rc = check_decode_args(query, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                               num_heads, num_kv_heads, head_dim, scale, block_size, num_blocks, PA_F32);
    if (rc != PA_OK) return rc;
    if (num_tokens < 0) return PA_ERR_SHAPE;
    if (num_seqs == 0 || num_tokens == 0) return PA_OK;
    if (!out || !q_start) return PA_ERR_NULL;
    if (!aligned(out, 16) || !aligned(q_start, 4)) return PA_ERR_ALIGN;
    if ((long long)num_tokens * num_heads >= INT_MAX) return PA_ERR_SHAPE;
    unsigned int *err = nullptr;
    if (device_error_word(&err) != cudaSuccess) return PA_ERR_CUDA;
    DecodeParams p{};
    p.out = out;
    p.query = query;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.q_start = q_start;
    p.num_seqs = num_seqs;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.num_blocks = num_blocks;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.partition_size = 0;
    p.max_parts = 1;
    p.max_context_len = INT_MAX;
    p.out_dtype = PA_F32;
    p.err = err;
    cudaError_t e = launch_decode(p, PA_F32, head_dim, block_size, num_heads / num_kv_heads, num_tokens,
                                  num_kv_heads, 1, stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa

extern "C" {

int pa_decode_withhold_stage(void *out, const void *query, const void *k_cache, const void *v_cache,
                             const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                             int num_seqs, int num_heads, int num_kv_heads, int head_dim, float scale,
                             int block_size, int num_blocks, pa_dtype kv_dtype, pa_dtype out_dtype,
                             const int32_t *seq_order, int seq, int kv_head, int stage,
                             unsigned long long wait_limit_ns, cudaStream_t stream) {
    if (seq < 0 || seq >= num_seqs || kv_head < 0 || kv_head >= num_kv_heads || stage < 0) return PA_ERR_SHAPE;
    if (wait_limit_ns < 100000ull || wait_limit_ns > 1000000000ull) return PA_ERR_SHAPE;
    WithholdHook hook;
    hook.seq = seq;
    hook.kv_head = kv_head;
    hook.stage = stage;
    hook.wait_limit_ns = wait_limit_ns;
    return decode_unsplit(out, query, nullptr, nullptr, k_cache, v_cache, block_tables, max_blocks_per_seq,
                          context_lens, num_seqs, num_heads, num_kv_heads, head_dim, scale, block_size,
                          num_blocks, kv_dtype, out_dtype, seq_order, stream, hook);
}

size_t pa_splitk_acc_offset(int num_seqs, int num_heads, int max_context_len, int partition_size) {
    if (num_seqs < 0 || num_heads <= 0 || max_context_len < 0 || partition_size <= 0) return 0;
    const int mp = max_parts_of(max_context_len, partition_size);
    return align_up(ml_bytes(num_seqs, num_heads, mp), 256);
}

size_t pa_splitk_workspace_bytes(int num_seqs, int num_heads, int head_dim, int max_context_len,
                                 int partition_size) {
    if (num_seqs < 0 || num_heads <= 0 || head_dim <= 0 || max_context_len < 0 ||
        partition_size <= 0)
        return 0;
    const int mp = max_parts_of(max_context_len, partition_size);
    return pa_splitk_acc_offset(num_seqs, num_heads, max_context_len, partition_size) +
           (size_t)num_seqs * num_heads * mp * head_dim * sizeof(float);
}

int pa_decode_splitk(void *workspace, size_t workspace_bytes, const void *query,
                     const void *k_cache, const void *v_cache, const int32_t *block_tables,
                     int max_blocks_per_seq, const int32_t *context_lens, int num_seqs,
                     int num_heads, int num_kv_heads, int head_dim, float scale, int block_size,
                     int num_blocks, int max_context_len, int partition_size, pa_dtype kv_dtype,
                     const int32_t *seq_order, cudaStream_t stream) {
    int rc = check_decode_args(query, k_cache, v_cache, block_tables, max_blocks_per_seq,
                               context_lens, num_seqs, num_heads, num_kv_heads, head_dim, scale,
                               block_size, num_blocks, kv_dtype);
    if (rc != PA_OK) return rc;
    if (max_context_len < 0) return PA_ERR_SHAPE;
    if (partition_size <= 0 || partition_size % block_size != 0) return PA_ERR_PARTITION;
    if (num_seqs == 0 || max_context_len == 0) return PA_OK;
    if (!aligned(seq_order, 4)) return PA_ERR_ALIGN;
    const size_t need = pa_splitk_workspace_bytes(num_seqs, num_heads, head_dim, max_context_len,
                                                  partition_size);
    if (!workspace || workspace_bytes < need) return PA_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return PA_ERR_ALIGN;
    unsigned int *err = nullptr;
    if (device_error_word(&err) != cudaSuccess) return PA_ERR_CUDA;
    const int mp = max_parts_of(max_context_len, partition_size);
    DecodeParams p{};
    p.ws_ml = static_cast<float *>(workspace);
    p.ws_acc = reinterpret_cast<float *>(
        static_cast<unsigned char *>(workspace) +
        pa_splitk_acc_offset(num_seqs, num_heads, max_context_len, partition_size));
    p.query = query;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.seq_order = seq_order;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.num_blocks = num_blocks;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.partition_size = partition_size;
    p.max_parts = mp;
    p.max_context_len = max_context_len;
    p.out_dtype = PA_F32;
    p.err = err;
    cudaError_t e = launch_decode(p, kv_dtype, head_dim, block_size, num_heads / num_kv_heads, mp,
                                  num_kv_heads, num_seqs, stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_splitk_reduce(void *out, const void *workspace, size_t workspace_bytes,
                     const int32_t *context_lens, int num_seqs, int num_heads, int head_dim,
                     int max_context_len, int partition_size, pa_dtype out_dtype,
                     cudaStream_t stream) {
    if (num_seqs < 0 || num_heads <= 0 || max_context_len < 0 || num_seqs > 65535 ||
        num_heads > INT_MAX / 2)
        return PA_ERR_SHAPE;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_HEAD_DIM;
    if (partition_size <= 0) return PA_ERR_PARTITION;
    if (elt_bytes(out_dtype) == 0) return PA_ERR_DTYPE;
    if (num_seqs == 0) return PA_OK;
    if (!out || !context_lens) return PA_ERR_NULL;
    if (!aligned(out, 16) || !aligned(context_lens, 4)) return PA_ERR_ALIGN;
    const int mp = max_parts_of(max_context_len, partition_size);
    const size_t need = pa_splitk_workspace_bytes(num_seqs, num_heads, head_dim, max_context_len,
                                                  partition_size);
    if (mp > 0 && (!workspace || workspace_bytes < need)) return PA_ERR_WORKSPACE;
    const float *ml = static_cast<const float *>(workspace);
    const float *acc = workspace == nullptr
                           ? nullptr
                           : reinterpret_cast<const float *>(
                                 static_cast<const unsigned char *>(workspace) +
                                 pa_splitk_acc_offset(num_seqs, num_heads, max_context_len,
                                                      partition_size));
    cudaError_t e = launch_splitk_reduce(out, ml, acc, context_lens, num_seqs, num_heads, head_dim,
                                         partition_size, mp > 0 ? mp : 1, max_context_len,
                                         out_dtype, stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_choose_partition(int num_seqs, int num_kv_heads, int max_context_len, int block_size,
                        int head_dim, pa_dtype kv_dtype) {
    (void)head_dim;
    (void)kv_dtype;
    if (num_seqs <= 0 || num_kv_heads <= 0 || max_context_len <= 0 || block_size <= 0) return 0;
    const long long items = (long long)num_seqs * num_kv_heads;
    const long long target = 4LL * sm_count();  // work items that keep every SM busy
    if (items >= target) return 0;
    // Enough partitions of the longest sequence to reach the target, in
    // powers of two of at least 512 tokens.
    long long want = (long long)max_context_len * items / target;
    int P = 512;
    while (P < want && P < (1 << 20)) P <<= 1;
    P = (P + block_size - 1) / block_size * block_size;
    return P >= max_context_len ? 0 : P;
}

int pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *src_dst_pairs, int num_pairs,
                   int num_blocks, int num_kv_heads, int head_dim, int block_size,
                   pa_dtype kv_dtype, cudaStream_t stream) {
    if (num_pairs < 0 || num_blocks < 0 || num_kv_heads <= 0) return PA_ERR_SHAPE;
    const int eb = elt_bytes(kv_dtype);
    if (eb == 0) return PA_ERR_DTYPE;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_HEAD_DIM;
    if (block_size != 16 && block_size != 32) return PA_ERR_BLOCK_SIZE;
    if (num_pairs == 0) return PA_OK;
    if (!k_cache || !v_cache || !src_dst_pairs) return PA_ERR_NULL;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(src_dst_pairs, 8))
        return PA_ERR_ALIGN;
    unsigned int *err = nullptr;
    if (device_error_word(&err) != cudaSuccess) return PA_ERR_CUDA;
    const size_t block_bytes = (size_t)num_kv_heads * block_size * head_dim * eb;
    cudaError_t e = launch_copy_blocks(k_cache, v_cache, src_dst_pairs, num_pairs, nullptr, num_blocks,
                                       block_bytes, err, stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_copy_blocks_counted(void *k_cache, void *v_cache, const int64_t *src_dst_pairs,
                           const int32_t *num_pairs, int max_pairs, int num_blocks, int num_kv_heads,
                           int head_dim, int block_size, pa_dtype kv_dtype, cudaStream_t stream) {
    if (max_pairs < 0 || num_blocks < 0 || num_kv_heads <= 0) return PA_ERR_SHAPE;
    const int eb = elt_bytes(kv_dtype);
    if (eb == 0) return PA_ERR_DTYPE;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_HEAD_DIM;
    if (block_size != 16 && block_size != 32) return PA_ERR_BLOCK_SIZE;
    if (max_pairs == 0) return PA_OK;
    if (!k_cache || !v_cache || !src_dst_pairs || !num_pairs) return PA_ERR_NULL;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(src_dst_pairs, 8) || !aligned(num_pairs, 4))
        return PA_ERR_ALIGN;
    unsigned int *err = nullptr;
    if (device_error_word(&err) != cudaSuccess) return PA_ERR_CUDA;
    const size_t block_bytes = (size_t)num_kv_heads * block_size * head_dim * eb;
    cudaError_t e = launch_copy_blocks(k_cache, v_cache, src_dst_pairs, max_pairs, num_pairs, num_blocks,
                                       block_bytes, err, stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// ------------------------------------------------------------ int8 caches

int pa_reshape_and_cache_q8(const void *key, const void *value, pa_dtype src_dtype, int8_t *k_cache,
                            int8_t *v_cache, float *k_scale, float *v_scale, const int32_t *slot_mapping,
                            int num_tokens, int num_blocks, int num_kv_heads, int head_dim, int block_size,
                            cudaStream_t stream) {
    if (num_tokens < 0 || num_blocks < 0 || num_kv_heads <= 0) return PA_ERR_SHAPE;
    if (elt_bytes(src_dtype) == 0) return PA_ERR_DTYPE;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_HEAD_DIM;
    if (block_size != 16 && block_size != 32) return PA_ERR_BLOCK_SIZE;
    if ((long long)num_blocks * block_size > INT_MAX) return PA_ERR_SHAPE;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !k_cache || !v_cache || !k_scale || !v_scale || !slot_mapping) return PA_ERR_NULL;
    if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(k_scale, 16) || !aligned(v_scale, 16) || !aligned(slot_mapping, 4))
        return PA_ERR_ALIGN;
    unsigned int *err = nullptr;
    if (device_error_word(&err) != cudaSuccess) return PA_ERR_CUDA;
    cudaError_t e = launch_reshape_and_cache_q8(key, value, src_dtype, k_cache, v_cache, k_scale, v_scale,
                                                slot_mapping, num_tokens, num_blocks, num_kv_heads, head_dim,
                                                block_size, err, stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// The V pool of an int8 cache with head_dim 128 as 2-D rows for the decode
// kernel's swizzled TMA loads (see DecodeParams::v_map).
static int q8_v_map(DecodeParams &p, const int8_t *v_cache, int num_blocks, int num_kv_heads, int head_dim,
                    int block_size) {
    if (head_dim != 128) return PA_OK;
    const long long rows = (long long)num_blocks * num_kv_heads * block_size;
    if (rows <= 0) return PA_OK;
    if (rows >= INT_MAX) return PA_ERR_SHAPE;  // TMA row coordinates are 32-bit
    return encode_rows_2d(&p.v_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, v_cache, 128, (unsigned long long)rows, 128, 128,
                          16, CU_TENSOR_MAP_SWIZZLE_128B)
               ? PA_OK
               : PA_ERR_CUDA;
}

// Shared by the int8 decode entries: query type, scale pools, then the common checks.
static int check_q8_args(const void *query, pa_dtype q_dtype, const int8_t *k_cache, const int8_t *v_cache,
                         const float *k_scale, const float *v_scale, const int32_t *block_tables,
                         int max_blocks_per_seq, const int32_t *context_lens, int num_seqs, int num_heads,
                         int num_kv_heads, int head_dim, float scale, int block_size, int num_blocks) {
    if (q_dtype != PA_F16 && q_dtype != PA_BF16) return PA_ERR_DTYPE;
    int rc = check_decode_args(query, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                               num_heads, num_kv_heads, head_dim, scale, block_size, num_blocks, q_dtype);
    if (rc != PA_OK || num_seqs == 0) return rc;
    if (!k_scale || !v_scale) return PA_ERR_NULL;
    if (!aligned(k_scale, 16) || !aligned(v_scale, 16)) return PA_ERR_ALIGN;
    return PA_OK;
}

int pa_decode_q8(void *out, const void *query, pa_dtype q_dtype, const int8_t *k_cache, const int8_t *v_cache,
                 const float *k_scale, const float *v_scale, const int32_t *block_tables, int max_blocks_per_seq,
                 const int32_t *context_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                 float scale, int block_size, int num_blocks, pa_dtype out_dtype, const int32_t *seq_order,
                 cudaStream_t stream) {
    int rc = check_q8_args(query, q_dtype, k_cache, v_cache, k_scale, v_scale, block_tables, max_blocks_per_seq,
                           context_lens, num_seqs, num_heads, num_kv_heads, head_dim, scale, block_size, num_blocks);
    if (rc != PA_OK) return rc;
    if (out_dtype != q_dtype && out_dtype != PA_F32) return PA_ERR_DTYPE;
    if (num_seqs == 0) return PA_OK;
    if (!aligned(seq_order, 4)) return PA_ERR_ALIGN;
    if (!out) return PA_ERR_NULL;
    if (!aligned(out, 16)) return PA_ERR_ALIGN;
    unsigned int *err = nullptr;
    if (device_error_word(&err) != cudaSuccess) return PA_ERR_CUDA;
    DecodeParams p{};
    p.out = out;
    p.query = query;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.seq_order = seq_order;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.num_blocks = num_blocks;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.partition_size = 0;
    p.max_parts = 1;
    p.max_context_len = INT_MAX;
    p.out_dtype = out_dtype;
    p.err = err;
    rc = q8_v_map(p, v_cache, num_blocks, num_kv_heads, head_dim, block_size);
    if (rc != PA_OK) return rc;
    cudaError_t e = launch_decode_q8(p, q_dtype, head_dim, block_size, num_heads / num_kv_heads, 1, num_kv_heads,
                                     num_seqs, stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_decode_splitk_q8(void *workspace, size_t workspace_bytes, const void *query, pa_dtype q_dtype,
                        const int8_t *k_cache, const int8_t *v_cache, const float *k_scale, const float *v_scale,
                        const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                        int num_seqs, int num_heads, int num_kv_heads, int head_dim, float scale, int block_size,
                        int num_blocks, int max_context_len, int partition_size, const int32_t *seq_order,
                        cudaStream_t stream) {
    int rc = check_q8_args(query, q_dtype, k_cache, v_cache, k_scale, v_scale, block_tables, max_blocks_per_seq,
                           context_lens, num_seqs, num_heads, num_kv_heads, head_dim, scale, block_size, num_blocks);
    if (rc != PA_OK) return rc;
    if (max_context_len < 0) return PA_ERR_SHAPE;
    if (partition_size <= 0 || partition_size % block_size != 0) return PA_ERR_PARTITION;
    if (num_seqs == 0 || max_context_len == 0) return PA_OK;
    if (!aligned(seq_order, 4)) return PA_ERR_ALIGN;
    const size_t need = pa_splitk_workspace_bytes(num_seqs, num_heads, head_dim, max_context_len, partition_size);
    if (!workspace || workspace_bytes < need) return PA_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return PA_ERR_ALIGN;
    unsigned int *err = nullptr;
    if (device_error_word(&err) != cudaSuccess) return PA_ERR_CUDA;
    const int mp = max_parts_of(max_context_len, partition_size);
    DecodeParams p{};
    p.ws_ml = static_cast<float *>(workspace);
    p.ws_acc = reinterpret_cast<float *>(static_cast<unsigned char *>(workspace) +
                                         pa_splitk_acc_offset(num_seqs, num_heads, max_context_len, partition_size));
    p.query = query;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.seq_order = seq_order;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.num_blocks = num_blocks;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.partition_size = partition_size;
    p.max_parts = mp;
    p.max_context_len = max_context_len;
    p.out_dtype = PA_F32;
    p.err = err;
    rc = q8_v_map(p, v_cache, num_blocks, num_kv_heads, head_dim, block_size);
    if (rc != PA_OK) return rc;
    cudaError_t e = launch_decode_q8(p, q_dtype, head_dim, block_size, num_heads / num_kv_heads, mp, num_kv_heads,
                                     num_seqs, stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_copy_blocks_q8(int8_t *k_cache, int8_t *v_cache, float *k_scale, float *v_scale,
                      const int64_t *src_dst_pairs, int num_pairs, int num_blocks, int num_kv_heads, int head_dim,
                      int block_size, cudaStream_t stream) {
    if (num_pairs < 0 || num_blocks < 0 || num_kv_heads <= 0) return PA_ERR_SHAPE;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_HEAD_DIM;
    if (block_size != 16 && block_size != 32) return PA_ERR_BLOCK_SIZE;
    if (num_pairs == 0) return PA_OK;
    if (!k_cache || !v_cache || !k_scale || !v_scale || !src_dst_pairs) return PA_ERR_NULL;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(k_scale, 16) || !aligned(v_scale, 16) ||
        !aligned(src_dst_pairs, 8))
        return PA_ERR_ALIGN;
    unsigned int *err = nullptr;
    if (device_error_word(&err) != cudaSuccess) return PA_ERR_CUDA;
    cudaError_t e = launch_copy_blocks(k_cache, v_cache, src_dst_pairs, num_pairs, nullptr, num_blocks,
                                       (size_t)num_kv_heads * block_size * head_dim, err, stream);
    if (e == cudaSuccess)
        e = launch_copy_blocks(k_scale, v_scale, src_dst_pairs, num_pairs, nullptr, num_blocks,
                               (size_t)num_kv_heads * block_size * sizeof(float), err, stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

size_t pa_dpool_state_bytes(int num_blocks) {
    if (num_blocks <= 0) return 0;
    return (PA_DPOOL_HEADER_WORDS + (size_t)PA_DPOOL_ARRAYS * num_blocks + PA_DPOOL_TAIL_WORDS) * sizeof(int32_t);
}

int pa_dpool_init(void *state, int num_blocks, int block_size, int policy, const int32_t *free_order,
                  cudaStream_t stream) {
    if (num_blocks <= 0 || block_size <= 0 || num_blocks > INT_MAX / PA_DPOOL_ARRAYS) return PA_ERR_SHAPE;
    if (policy != PA_POOL_LIFO && policy != PA_POOL_FIFO) return PA_ERR_SHAPE;
    if (!state) return PA_ERR_NULL;
    if (!aligned(state, 16) || (free_order && !aligned(free_order, 4))) return PA_ERR_ALIGN;
    unsigned int *err = nullptr;
    if (device_error_word(&err) != cudaSuccess) return PA_ERR_CUDA;
    cudaError_t e = launch_dpool_init(static_cast<int32_t *>(state), num_blocks, block_size, policy, free_order,
                                      err, stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_dpool_load(void *state, int num_blocks, int block_size, int policy, const int32_t *ref_counts,
                  const int32_t *free_list, int num_free, cudaStream_t stream) {
    if (num_blocks <= 0 || block_size <= 0 || num_blocks > INT_MAX / PA_DPOOL_ARRAYS) return PA_ERR_SHAPE;
    if (num_free < 0 || num_free > num_blocks) return PA_ERR_SHAPE;
    if (policy != PA_POOL_LIFO && policy != PA_POOL_FIFO) return PA_ERR_SHAPE;
    if (!state || !ref_counts || (num_free > 0 && !free_list)) return PA_ERR_NULL;
    if (!aligned(state, 16) || !aligned(ref_counts, 4) || !aligned(free_list, 4)) return PA_ERR_ALIGN;
    unsigned int *err = nullptr;
    if (device_error_word(&err) != cudaSuccess) return PA_ERR_CUDA;
    cudaError_t e = launch_dpool_load(static_cast<int32_t *>(state), num_blocks, block_size, policy, ref_counts,
                                      free_list, num_free, err, stream);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // extern "C"

namespace {

// pa_beam_step, with the test hook's arguments (withhold_cta -1 for a normal call).
int beam_step_call(void *state, int num_blocks, int block_size, const int32_t *old_tables,
                   const int32_t *old_context_lens, int num_old, const int32_t *parents, int num_new,
                   int32_t *new_tables, int32_t *new_context_lens, int max_blocks_per_seq, int32_t *slot_mapping,
                   int64_t *cow_pairs, int32_t *num_cow, int withhold_cta, unsigned long long limit_ns,
                   cudaStream_t stream) {
    if (num_blocks <= 0 || block_size <= 0 || num_old < 0 || num_new < 0 || max_blocks_per_seq <= 0)
        return PA_ERR_SHAPE;
    if (((long long)num_old + num_new) * max_blocks_per_seq >= (1LL << 30) ||
        (long long)num_blocks * block_size >= INT_MAX || 3LL * num_old + num_new > PA_BEAM_MAX_STAGED)
        return PA_ERR_SHAPE;
    if (!state || !num_cow || (num_old > 0 && (!old_tables || !old_context_lens)) ||
        (num_new > 0 && (!parents || !new_tables || !new_context_lens || !slot_mapping || !cow_pairs)))
        return PA_ERR_NULL;
    if (num_new > 0 && num_old > 0 && (new_tables == old_tables || new_context_lens == old_context_lens))
        return PA_ERR_SHAPE;
    if (!aligned(state, 16) || !aligned(num_cow, 4) || !aligned(old_tables, 4) || !aligned(old_context_lens, 4) ||
        !aligned(parents, 4) || !aligned(new_tables, 4) || !aligned(new_context_lens, 4) ||
        !aligned(slot_mapping, 4) || !aligned(cow_pairs, 8))
        return PA_ERR_ALIGN;
    unsigned int *err = nullptr;
    if (device_error_word(&err) != cudaSuccess) return PA_ERR_CUDA;
    cudaError_t e = launch_beam_step(static_cast<int32_t *>(state), old_tables, old_context_lens, num_old, parents,
                                     num_new, new_tables, new_context_lens, max_blocks_per_seq, slot_mapping,
                                     cow_pairs, num_cow, num_blocks, block_size, err, stream, withhold_cta, limit_ns);
    if (withhold_cta >= 0 && e == cudaErrorNotSupported) {  // no one-launch form for this step
        (void)cudaGetLastError();
        return PA_ERR_SHAPE;
    }
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace

extern "C" {

int pa_beam_step(void *state, int num_blocks, int block_size, const int32_t *old_tables,
                 const int32_t *old_context_lens, int num_old, const int32_t *parents, int num_new,
                 int32_t *new_tables, int32_t *new_context_lens, int max_blocks_per_seq,
                 int32_t *slot_mapping, int64_t *cow_pairs, int32_t *num_cow, cudaStream_t stream) {
    return beam_step_call(state, num_blocks, block_size, old_tables, old_context_lens, num_old, parents, num_new,
                          new_tables, new_context_lens, max_blocks_per_seq, slot_mapping, cow_pairs, num_cow, -1, 0,
                          stream);
}

int pa_beam_step_withhold_arrival(void *state, int num_blocks, int block_size, const int32_t *old_tables,
                                  const int32_t *old_context_lens, int num_old, const int32_t *parents, int num_new,
                                  int32_t *new_tables, int32_t *new_context_lens, int max_blocks_per_seq,
                                  int32_t *slot_mapping, int64_t *cow_pairs, int32_t *num_cow, int cta,
                                  unsigned long long wait_limit_ns, cudaStream_t stream) {
    if (cta < 0 || wait_limit_ns < 100000ull || wait_limit_ns > 1000000000ull) return PA_ERR_SHAPE;
    return beam_step_call(state, num_blocks, block_size, old_tables, old_context_lens, num_old, parents, num_new,
                          new_tables, new_context_lens, max_blocks_per_seq, slot_mapping, cow_pairs, num_cow, cta,
                          wait_limit_ns, stream);
}

}  // extern "C"
