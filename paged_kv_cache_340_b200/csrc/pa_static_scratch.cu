// Split-K decode that needs no allocation from its caller: the partials live
// in a fixed scratch array owned by this library.
//
// Who needs this: code that must not allocate device memory while it runs --
// a serving loop that has handed nearly all of HBM to its KV-cache pool up
// front (a cudaMalloc at step time could fail, or fragment what is left),
// plug-in or callback code whose host framework forbids allocating inside its
// execute hook, and callers with no allocator of their own on the device.
// Such callers pass only inputs and the output; the workspace that
// pa_decode_splitk would need is taken from the array below instead.
//
// Cost and limits: the array is PA_STATIC_SCRATCH_BYTES of device memory. It
// lives in this file's own module, which CUDA's lazy module loading loads --
// and so allocates the array -- on the first call on each device (the address
// lookup below), not when the library is opened. A caller that gives nearly
// all of HBM to its KV pool makes that first call (an empty one, num_seqs ==
// 0, is enough) before sizing the pool, and before any stream capture; from
// then on the array stays until the process exits (or the context is reset,
// after which the next call loads it again). Every call on a device shares
// it, so calls whose kernels overlap on that device (two streams, or two host
// threads) race on it; serialise them. A call keeps the previous call's
// partials in the array; nothing in it needs to start at zero, because every
// partial the reduce reads is written first by the same call.
#include <climits>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

static __device__ __align__(256) unsigned char g_static_scratch[PA_STATIC_SCRATCH_BYTES];

// Device address of the array on the current device. Host code cannot use
// the symbol itself (on the host it names a stand-in, not device memory), so
// the address is looked up on the first call in each device context.
static cudaError_t static_scratch_address(unsigned char **addr) {
    static SymbolCache cache;
    void *a = nullptr;
    cudaError_t e = symbol_address(&g_static_scratch, &cache, &a);
    if (e == cudaSuccess) *addr = static_cast<unsigned char *>(a);
    return e;
}

}  // namespace pa

extern "C" int pa_decode_splitk_static(void *out, const void *query, const void *k_cache,
                                       const void *v_cache, const int32_t *block_tables,
                                       int max_blocks_per_seq, const int32_t *context_lens,
                                       int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                       float scale, int block_size, int num_blocks,
                                       int max_context_len, int partition_size, pa_dtype kv_dtype,
                                       pa_dtype out_dtype, cudaStream_t stream) {
    // Reject what the array cannot hold, and every argument the reduce would
    // refuse, before any device work.
    if (num_seqs < 0 || num_heads <= 0 || max_context_len < 0) return PA_ERR_SHAPE;
    if (partition_size <= 0 || (block_size > 0 && partition_size % block_size != 0))
        return PA_ERR_PARTITION;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_HEAD_DIM;
    if (out_dtype != PA_F32 && out_dtype != PA_F16 && out_dtype != PA_BF16) return PA_ERR_DTYPE;
    const size_t need = pa_splitk_workspace_bytes(num_seqs, num_heads, head_dim, max_context_len,
                                                  partition_size);
    if (need > (size_t)PA_STATIC_SCRATCH_BYTES) return PA_ERR_WORKSPACE;
    if (num_seqs > 0) {
        if (!out || !context_lens) return PA_ERR_NULL;
        if ((reinterpret_cast<uintptr_t>(out) & 15u) != 0 || (reinterpret_cast<uintptr_t>(context_lens) & 3u) != 0)
            return PA_ERR_ALIGN;
    }
    // Also on an empty call, so that one can load the array ahead of time.
    unsigned char *scratch = nullptr;
    if (pa::static_scratch_address(&scratch) != cudaSuccess) return PA_ERR_CUDA;
    if (num_seqs == 0) return PA_OK;
    int rc = pa_decode_splitk(scratch, (size_t)PA_STATIC_SCRATCH_BYTES, query, k_cache, v_cache,
                              block_tables, max_blocks_per_seq, context_lens, num_seqs, num_heads,
                              num_kv_heads, head_dim, scale, block_size, num_blocks,
                              max_context_len, partition_size, kv_dtype, nullptr, stream);
    if (rc != PA_OK) return rc;
    return pa_splitk_reduce(out, scratch, (size_t)PA_STATIC_SCRATCH_BYTES, context_lens, num_seqs,
                            num_heads, head_dim, max_context_len, partition_size, out_dtype,
                            stream);
}
