/*
 * pa.h -- C ABI of the paged KV-cache library for NVIDIA B200 (sm_100a):
 * decode, split-K decode, slot write fused with decode, prefill, slot writes
 * and block copies (16-bit, fp32 and int8 caches), the host block pool with
 * its prefix cache, and a device block pool with a beam-search step.
 *
 * A sequence's keys and values live in fixed-size blocks of a shared pool; a
 * per-sequence block table maps logical block i (tokens i*bs .. i*bs+bs-1) to
 * a physical block, so no sequence needs contiguous memory.
 *
 * Sources (web pages, cited by title and section):
 *   [P1] "PagedAttention 源码解析：KV Cache 怎么管理" (coreui.cn)
 *   [P2] "PagedAttention原理与KV Cache显存优化" (xdnf.cn)
 *   [P3] "Ascend C算子开发高阶实战：实现高性能KV Cache管理与PagedAttention融合算子" (cann.csdn.net)
 *   [P4] "PagedAttention 实现细节" (pyllm.pages.dev, vLLM series)
 *   [P5] "Ascend平台下的PageAttention优化实践" (jsqmd.com)
 *
 * Conventions for every device entry point:
 *   - Pointers named *_cache, query, out, key, value, new_key, new_value,
 *     block_tables, context_lens, slot_mapping, src_dst_pairs and workspace are DEVICE
 *     pointers owned by the caller. The library never allocates, frees or
 *     keeps them.
 *   - Layouts (row-major, contiguous):
 *       k_cache, v_cache  [num_blocks, num_kv_heads, block_size, head_dim]
 *       query, out        [num_seqs, num_heads, head_dim]
 *       key, value        [num_tokens, num_kv_heads, head_dim]
 *       block_tables      [num_seqs, max_blocks_per_seq] int32
 *       context_lens      [num_seqs] int32
 *       slot_mapping      [num_tokens] int32
 *     Token t of sequence s is row (block_tables[s][t / block_size], kv head,
 *     t % block_size) of the pools ([P2] §3.1; [P4] §3.1 index-based kernel).
 *   - Supported: head_dim 64 or 128; block_size 16 or 32; num_heads any
 *     multiple of num_kv_heads (query head h reads kv head
 *     h / (num_heads / num_kv_heads)); element types PA_F32, PA_F16,
 *     PA_BF16. Every device pointer must be 16-byte aligned.
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream)
 *     and return PA_OK once the work is enqueued. Arguments are checked on
 *     the host first; a violation returns a negative pa_status and enqueues
 *     nothing. A failed launch returns PA_ERR_CUDA.
 *   - Data errors that only the device can see (a table entry or slot out of
 *     range, a context longer than its table row) never fault: the kernel
 *     skips the offending block or token and records a PA_DEVERR_* bit in a
 *     device error word that pa_read_device_errors() returns.
 */
#ifndef PAGED_KV_CACHE_340_B200_PA_H
#define PAGED_KV_CACHE_340_B200_PA_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_dtype { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2 } pa_dtype;

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_NULL = -1,            /* a required pointer is NULL */
    PA_ERR_DTYPE = -2,           /* unsupported element type or output type */
    PA_ERR_SHAPE = -3,           /* a size is negative or inconsistent */
    PA_ERR_HEADS = -4,           /* num_heads % num_kv_heads != 0 */
    PA_ERR_HEAD_DIM = -5,        /* head_dim not in {64, 128} */
    PA_ERR_BLOCK_SIZE = -6,      /* block_size not in {16, 32} */
    PA_ERR_ALIGN = -7,           /* a device pointer is not 16-byte aligned */
    PA_ERR_PARTITION = -8,       /* partition_size not a positive multiple of block_size */
    PA_ERR_WORKSPACE = -9,       /* workspace smaller than pa_splitk_workspace_bytes() */
    PA_ERR_CUDA = -10,           /* a CUDA runtime call or launch failed */
    PA_ERR_POOL_EXHAUSTED = -11, /* host pool: no free block */
    PA_ERR_POOL_STATE = -12,     /* host pool: block id out of range or already free */
    PA_ERR_CAPACITY = -13        /* host pool: caller's table row or output array too small */
} pa_status;

/* Bits of the device error word (see pa_read_device_errors). */
#define PA_DEVERR_BLOCK_ID 0x1u  /* table entry outside [0, num_blocks): its tokens were skipped */
#define PA_DEVERR_SLOT 0x2u      /* slot >= num_blocks * block_size: the token was not written */
#define PA_DEVERR_CONTEXT 0x4u   /* context_len < 0, or longer than its table row / max_context_len: clamped */
#define PA_DEVERR_TIMEOUT 0x8u   /* an on-chip pipeline wait ran past its bound: output undefined */
#define PA_DEVERR_PAIR 0x10u     /* copy pair with an id outside [0, num_blocks): skipped */
#define PA_DEVERR_POOL 0x20u     /* device pool: exhausted, no table room, or state not initialised: step not applied */

/* Text for a pa_status value (static storage, never NULL). */
const char *pa_status_string(int status);

/* Waits for `stream`, then returns in *flags the PA_DEVERR_* bits recorded
 * by kernels on the current device since the last call, and clears them.
 * Returns PA_ERR_CUDA if the synchronisation or copy fails. */
int pa_read_device_errors(uint32_t *flags, cudaStream_t stream);

/*
 * pa_reshape_and_cache -- slot write of new tokens.
 * For each token i with slot = slot_mapping[i] >= 0 and every kv head h:
 *   k_cache[slot / block_size, h, slot % block_size, :] = key[i, h, :]
 *   v_cache[slot / block_size, h, slot % block_size, :] = value[i, h, :]
 * as a bit copy. Negative slots are skipped. Non-negative slots must be
 * distinct within one call (two writes to one slot race).
 * [P3] §3.1 and §4.2 (slot_mapping, block_id = slot / block_size,
 * offset = slot % block_size); [P4] §3.4 (the runner writes each new token's
 * K/V into its block).
 * key/value/k_cache/v_cache share dtype `kv_dtype`.
 */
int pa_reshape_and_cache(const void *key, const void *value, void *k_cache, void *v_cache,
                         const int32_t *slot_mapping, int num_tokens, int num_blocks,
                         int num_kv_heads, int head_dim, int block_size, pa_dtype kv_dtype,
                         cudaStream_t stream);

/*
 * pa_decode -- fused paged decode attention, one pass, no partitioning.
 * For each sequence s (L = context_lens[s] tokens) and query head h:
 *   out[s, h, :] = sum_t softmax_t(scale * query[s, h, :] . K_t) V_t,  t < L,
 * where K_t, V_t are read in place from the pools through block_tables[s]
 * (no gathered copy), with fp32 accumulation and a running max and sum.
 * L == 0 writes zeros. Entries of block_tables[s] past ceil(L / block_size)
 * are never read. query has dtype kv_dtype; out_dtype is kv_dtype or PA_F32.
 * [P3] §1.3 (softmax(QK^T / sqrt(d)) V over the gathered history) and §3
 * (gather and attention fused in one pass, no intermediate written back);
 * [P4] §3.1 (index-based kernel over key_cache/value_cache
 * [num_blocks, num_kv_heads, block_size, head_dim]); [P5] §3.2 (inputs
 * query, key_cache, value_cache, block_tables, context_lens, scale).
 *
 * seq_order (nullable device int32 [num_seqs], a permutation of
 * 0 .. num_seqs-1) is the order in which sequences are scheduled on the GPU;
 * it changes no result. Work is handed to SMs roughly in this order, so
 * listing sequences longest first keeps a long sequence from starting last
 * and finishing alone. Entries outside [0, num_seqs) are skipped
 * (PA_DEVERR_CONTEXT). NULL schedules 0, 1, 2, ...
 */
int pa_decode(void *out, const void *query, const void *k_cache, const void *v_cache,
              const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
              int num_seqs, int num_heads, int num_kv_heads, int head_dim, float scale,
              int block_size, int num_blocks, pa_dtype kv_dtype, pa_dtype out_dtype,
              const int32_t *seq_order, cudaStream_t stream);

/*
 * pa_decode_append -- pa_reshape_and_cache of each sequence's newest token
 * followed by pa_decode, in one launch. The newest token of sequence s is at
 * position L - 1 (L = context_lens[s] >= 1, the new token counted): its rows
 * new_key[s, :, :] and new_value[s, :, :] ([num_seqs, num_kv_heads,
 * head_dim], dtype kv_dtype, device, 16-byte aligned) are written into the
 * slot block_tables[s][(L - 1) / block_size] * block_size + (L - 1) %
 * block_size of k_cache / v_cache, and the attention uses them for t = L - 1.
 * The result (pools and out) is that of the two calls in sequence, provided no
 * other sequence of the call reads that block (true once copy-on-write has
 * given each sequence its own last block). L == 0 writes nothing and outputs
 * zeros; a table entry out of range skips the block (PA_DEVERR_BLOCK_ID) and
 * writes nothing for it. Arguments otherwise as pa_decode. [P4] §3.4 (the
 * runner writes each new token's K/V into its block, then attention reads the
 * cache); the fusion is this library's: the warp whose 16-token stage holds
 * position L - 1 puts the new row over its landed tile before using it.
 */
int pa_decode_append(void *out, const void *query, const void *new_key, const void *new_value, void *k_cache,
                     void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                     const int32_t *context_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                     float scale, int block_size, int num_blocks, pa_dtype kv_dtype, pa_dtype out_dtype,
                     const int32_t *seq_order, cudaStream_t stream);

/*
 * pa_decode_withhold_stage -- pa_decode with a fault planted on the host, for
 * testing the bounded waits; not for production use. The CTA of sequence
 * `seq` (its index in the call), kv head `kv_head` never issues the copy of
 * its 16-token stage `stage` (tokens 16 * stage .. 16 * stage + 15), so the
 * warp that owns the stage waits for data that never comes. After
 * wait_limit_ns (between 1e5 and 1e9; the library's own bound is 1 s) it
 * records PA_DEVERR_TIMEOUT, waits with the same bound for the copies it
 * still has in flight, and leaves its loop; the launch ends normally. That
 * (sequence, kv head)'s output is undefined, every other output is
 * pa_decode's. A stage past the sequence's end withholds nothing. Nothing
 * faults and nothing hangs: this runs the path that a copy which never lands
 * would take, so a test can check that it returns and reports. Other
 * arguments as pa_decode; seq and kv_head out of range, stage < 0 or the
 * limit out of range give PA_ERR_SHAPE.
 */
int pa_decode_withhold_stage(void *out, const void *query, const void *k_cache, const void *v_cache,
                             const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                             int num_seqs, int num_heads, int num_kv_heads, int head_dim, float scale,
                             int block_size, int num_blocks, pa_dtype kv_dtype, pa_dtype out_dtype,
                             const int32_t *seq_order, int seq, int kv_head, int stage,
                             unsigned long long wait_limit_ns, cudaStream_t stream);

/*
 * Split-K (partitioned) decode for few, long sequences ([P5] §2.3: the
 * partitioned kernel of the pair). Tokens of sequence s are cut into
 * partitions of `partition_size` tokens (a multiple of block_size); partition
 * p covers [p * P, min((p + 1) * P, L)). pa_decode_splitk writes, per
 * (s, h, p) with a non-empty range:
 *   m   = max_t scale * q . K_t                          (float)
 *   l   = sum_t exp(scale * q . K_t - m)                 (float)
 *   acc = sum_t exp(scale * q . K_t - m) V_t             (float[head_dim])
 * into `workspace`, laid out as
 *   ml  float [num_seqs, num_heads, max_parts, 2]   (m, l) at offset 0
 *   acc float [num_seqs, num_heads, max_parts, head_dim] at byte offset
 *       pa_splitk_acc_offset(...)
 * with max_parts = ceil(max_context_len / partition_size). Entries of empty
 * partitions are not written. max_context_len must bound every
 * context_lens[s]; longer contexts are clamped (PA_DEVERR_CONTEXT).
 * pa_splitk_reduce then merges them by log-sum-exp:
 *   M = max_p m_p,  out = sum_p e^(m_p - M) acc_p / sum_p e^(m_p - M) l_p
 * (the standard split of the softmax; the pages only name the partitioned
 * kernel). Both calls must get the same sizes. seq_order (nullable) is the
 * scheduling order of sequences, as for pa_decode.
 */
size_t pa_splitk_workspace_bytes(int num_seqs, int num_heads, int head_dim, int max_context_len,
                                 int partition_size);
size_t pa_splitk_acc_offset(int num_seqs, int num_heads, int max_context_len, int partition_size);

int pa_decode_splitk(void *workspace, size_t workspace_bytes, const void *query,
                     const void *k_cache, const void *v_cache, const int32_t *block_tables,
                     int max_blocks_per_seq, const int32_t *context_lens, int num_seqs,
                     int num_heads, int num_kv_heads, int head_dim, float scale, int block_size,
                     int num_blocks, int max_context_len, int partition_size, pa_dtype kv_dtype,
                     const int32_t *seq_order, cudaStream_t stream);

int pa_splitk_reduce(void *out, const void *workspace, size_t workspace_bytes,
                     const int32_t *context_lens, int num_seqs, int num_heads, int head_dim,
                     int max_context_len, int partition_size, pa_dtype out_dtype,
                     cudaStream_t stream);

/*
 * pa_decode_splitk_static -- split-K decode plus reduce for callers that
 * cannot allocate device memory. The source pages have no counterpart; this
 * is an interface choice of this library.
 *
 * Same inputs and result as pa_decode_splitk followed by pa_splitk_reduce
 * (out [num_seqs, num_heads, head_dim] of out_dtype), but the workspace is a
 * fixed array inside the library (PA_STATIC_SCRATCH_BYTES of device memory on
 * every GPU where it has been called, kept until the process exits), so the
 * caller passes only inputs and the output. It suits code that must not
 * allocate while it runs: a serving loop that gave nearly all of HBM to its
 * KV pool up front, a plug-in whose host framework forbids allocation inside
 * its execute callback, or a caller with no device allocator at all.
 *   - Returns PA_ERR_WORKSPACE, with no device work, when
 *     pa_splitk_workspace_bytes(num_seqs, num_heads, head_dim,
 *     max_context_len, partition_size) exceeds PA_STATIC_SCRATCH_BYTES
 *     (use a larger partition_size or fewer sequences per call).
 *   - Every other argument the split-K decode or the reduce would refuse
 *     (NULL or misaligned out, an out_dtype other than PA_F32, PA_F16 or
 *     PA_BF16, ...) is also refused before any device work.
 *   - The array belongs to a module that CUDA loads lazily: the first call on
 *     each device (and again after a cudaDeviceReset) loads it, which takes
 *     the PA_STATIC_SCRATCH_BYTES of device memory then, and looks up its
 *     device address (cudaGetSymbolAddress). A caller that gives nearly all
 *     of HBM to its KV pool therefore makes one call first -- an empty one,
 *     num_seqs == 0 with valid sizes, does only this -- before sizing the
 *     pool, and before any stream capture. Later calls allocate nothing and
 *     call no allocating routine.
 *   - All calls on a device share the array: calls whose kernels overlap on
 *     the GPU (other streams, other host threads) race and must be
 *     serialised. The array keeps the previous call's partials; none of it
 *     needs to start at zero.
 */
#define PA_STATIC_SCRATCH_BYTES (32u * 1024u * 1024u)

int pa_decode_splitk_static(void *out, const void *query, const void *k_cache, const void *v_cache,
                            const int32_t *block_tables, int max_blocks_per_seq,
                            const int32_t *context_lens, int num_seqs, int num_heads,
                            int num_kv_heads, int head_dim, float scale, int block_size,
                            int num_blocks, int max_context_len, int partition_size,
                            pa_dtype kv_dtype, pa_dtype out_dtype, cudaStream_t stream);

/*
 * pa_prefill -- paged prefill (chunked prefill) attention on the tensor cores.
 * Sequence s has q_len_s = q_start[s+1] - q_start[s] new query tokens, rows
 * q_start[s] .. of query [num_tokens, num_heads, head_dim] (q_start is a device
 * int32 [num_seqs + 1], non-decreasing, q_start[num_seqs] <= num_tokens),
 * whose K/V are already in the cache (written by pa_reshape_and_cache). Query
 * token i sits at position pos = context_lens[s] - q_len_s + i and attends
 * causally to cache tokens 0 .. pos:
 *   out[q_start[s] + i, h, :] = sum_{t <= pos} softmax_t(scale q . K_t) V_t.
 * q_len_s = 1 is decode. max_q_len bounds every q_len_s. Requires
 * q_len_s <= context_lens[s] (else PA_DEVERR_CONTEXT and that sequence is
 * skipped). head_dim 64 or 128, block_size 16 or 32, any head group
 * (num_heads a multiple of num_kv_heads). kv_dtype PA_F16 or PA_BF16
 * (out_dtype kv_dtype or PA_F32): QK^T and PV run as tcgen05 MMAs with
 * accumulators in tensor memory, K/V tiles gathered through the table by
 * TMA. kv_dtype PA_F32 (out_dtype PA_F32): exact fp32 arithmetic on the CUDA
 * cores, each query token a decode over its causal prefix (the tensor cores
 * take fp32 only as tf32). ([P4] §3.4: the forward pass over the step's new
 * tokens, each layer attending over the paged cache; [P3] §3.1: the
 * num_tokens axis of queries.)
 */
int pa_prefill(void *out, const void *query, const int32_t *q_start, int num_tokens, int max_q_len,
               const void *k_cache, const void *v_cache, const int32_t *block_tables,
               int max_blocks_per_seq, const int32_t *context_lens, int num_seqs, int num_heads,
               int num_kv_heads, int head_dim, float scale, int block_size, int num_blocks,
               pa_dtype kv_dtype, pa_dtype out_dtype, cudaStream_t stream);

/*
 * pa_prefill_withhold_tile -- pa_prefill (16-bit caches, the tensor-core
 * kernel) with a fault planted on the host, for testing the bounded waits;
 * not for production use. The CTA of sequence `seq`, kv head `kv_head` and
 * query tile `query_tile` (its 128 rows of (token, query head) pairs: tokens
 * query_tile * 128 / G' .. of the sequence's new tokens, G' the head group
 * rounded up to a power of two; a group above 128 withholds in its first
 * sub-group only) never issues the copy of its 64-token K tile `tile`
 * (cache tokens 64 * tile ..), so the MMA thread that needs it waits for data
 * that never comes. After wait_limit_ns (between 1e5 and 1e9; the library's
 * own bound is 1 s) it records PA_DEVERR_TIMEOUT and releases the CTA's other
 * warps, which leave their loops; the load warp waits, with the same bound,
 * for the copies it still has in flight; every product issued finishes
 * before tensor memory is freed, and the launch ends normally. That CTA's
 * output rows are undefined, every other output is pa_prefill's. A tile or
 * query tile past the CTA's work withholds nothing. Other arguments as
 * pa_prefill; PA_F32 caches give PA_ERR_DTYPE, head_dim other than 128
 * PA_ERR_HEAD_DIM (the hook is compiled into separate head_dim-128 instances
 * of the kernel, so pa_prefill's own carry none of it), and seq or kv_head
 * out of range, query_tile or tile < 0, or the limit out of range
 * PA_ERR_SHAPE.
 */
int pa_prefill_withhold_tile(void *out, const void *query, const int32_t *q_start, int num_tokens,
                             int max_q_len, const void *k_cache, const void *v_cache,
                             const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                             int num_seqs, int num_heads, int num_kv_heads, int head_dim, float scale,
                             int block_size, int num_blocks, pa_dtype kv_dtype, pa_dtype out_dtype, int seq,
                             int kv_head, int query_tile, int tile, unsigned long long wait_limit_ns,
                             cudaStream_t stream);

/*
 * Partition size this library would pick for a batch: 0 when the
 * unpartitioned pa_decode already fills the GPU, else a multiple of
 * block_size. Host-only arithmetic on the sizes given (occupancy rule:
 * split until there are enough work items for every SM).
 */
int pa_choose_partition(int num_seqs, int num_kv_heads, int max_context_len, int block_size,
                        int head_dim, pa_dtype kv_dtype);

/*
 * pa_copy_blocks -- copy-on-write block copy. For each pair
 * (src_dst_pairs[2i], src_dst_pairs[2i+1]) = (src, dst): physical block dst
 * of both pools becomes a bit copy of block src (all kv heads, all slots).
 * Preconditions: dst ids distinct, and no dst is also a src in the same call
 * (all pairs run in parallel). Pairs with an id outside [0, num_blocks) are
 * skipped (PA_DEVERR_PAIR). src_dst_pairs is a device int64 [num_pairs, 2].
 * [P4] §3.3 (copy the whole block, device to device, before writing the
 * copy); [P2] §3.4 (parallel sampling, beam search).
 */
int pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *src_dst_pairs, int num_pairs,
                   int num_blocks, int num_kv_heads, int head_dim, int block_size,
                   pa_dtype kv_dtype, cudaStream_t stream);

/* As pa_copy_blocks, but the pair count is read on the device from
 * *num_pairs (device int32, at most max_pairs): the form that follows
 * pa_beam_step without a host round trip. */
int pa_copy_blocks_counted(void *k_cache, void *v_cache, const int64_t *src_dst_pairs,
                           const int32_t *num_pairs, int max_pairs, int num_blocks, int num_kv_heads,
                           int head_dim, int block_size, pa_dtype kv_dtype, cudaStream_t stream);

/*
 * int8 KV caches. The pages list int8 among the paged backend's storage
 * types ([P4] §3.4, attention backends) and name KV quantization as a memory
 * saving with a precision cost ([P2] §2.3, §6.3), without a scheme. This
 * library's scheme: symmetric int8 per (token, kv head) row with one fp32
 * scale, decided at the slot write:
 *   amax = max_d |x_d|; q_d = round_half_even(x_d * (127 / amax)) clamped to
 *   [-127, 127]; scale = amax / 127 (a zero row: codes 0, scale 0);
 * every step one IEEE fp32 operation. The cache holds K_t = q_t * scale_t.
 * Layouts: k_cache/v_cache int8 [num_blocks, num_kv_heads, block_size,
 * head_dim]; k_scale/v_scale fp32 [num_blocks, num_kv_heads, block_size];
 * all device pointers 16-byte aligned. Half the bytes of an fp16 cache plus
 * 4 bytes per row.
 */

/* Quantizing slot write: key/value [num_tokens, num_kv_heads, head_dim] of
 * src_dtype (PA_F32, PA_F16 or PA_BF16) -> codes and scales at each token's
 * slot (slot < 0 skipped, out of range PA_DEVERR_SLOT). */
int pa_reshape_and_cache_q8(const void *key, const void *value, pa_dtype src_dtype, int8_t *k_cache,
                            int8_t *v_cache, float *k_scale, float *v_scale, const int32_t *slot_mapping,
                            int num_tokens, int num_blocks, int num_kv_heads, int head_dim, int block_size,
                            cudaStream_t stream);

/* pa_decode over an int8 cache: out = softmax(scale q . K_t) V_t with
 * K_t = kq_t * k_scale_t, V_t = vq_t * v_scale_t. query is q_dtype (PA_F16
 * or PA_BF16); out_dtype q_dtype or PA_F32. On the tensor cores q . kq_t is
 * an exact integer product of kq_t and the query held as 16-bit fixed point
 * per head (each q_d within 2^-16 of the head's largest |q_d|); P enters
 * P V in fp16. Other arguments, checks and device errors as pa_decode. */
int pa_decode_q8(void *out, const void *query, pa_dtype q_dtype, const int8_t *k_cache, const int8_t *v_cache,
                 const float *k_scale, const float *v_scale, const int32_t *block_tables, int max_blocks_per_seq,
                 const int32_t *context_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                 float scale, int block_size, int num_blocks, pa_dtype out_dtype, const int32_t *seq_order,
                 cudaStream_t stream);

/* pa_decode_splitk over an int8 cache (then pa_splitk_reduce as usual). */
int pa_decode_splitk_q8(void *workspace, size_t workspace_bytes, const void *query, pa_dtype q_dtype,
                        const int8_t *k_cache, const int8_t *v_cache, const float *k_scale, const float *v_scale,
                        const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                        int num_seqs, int num_heads, int num_kv_heads, int head_dim, float scale, int block_size,
                        int num_blocks, int max_context_len, int partition_size, const int32_t *seq_order,
                        cudaStream_t stream);

/* pa_copy_blocks for an int8 cache: codes and scales of each pair. */
int pa_copy_blocks_q8(int8_t *k_cache, int8_t *v_cache, float *k_scale, float *v_scale,
                      const int64_t *src_dst_pairs, int num_pairs, int num_blocks, int num_kv_heads, int head_dim,
                      int block_size, cudaStream_t stream);

/*
 * Host block pool (no device memory): free list, reference counts and the
 * copy-on-write decision. These are plain host calls on host memory.
 * [P2] §3.3-§3.4 and §4.2 (PhysicalBlockPool: allocate sets the count to 1,
 * free returns a block at count 0; append_token_kv takes a new block when the
 * cached token count is a multiple of the block size); [P4] §3.3 (write into
 * a block whose count is above 1: take a new block, copy, drop the old
 * block's count, give the copy count 1, repoint the table).
 * A pool is not thread-safe; callers serialise access.
 */
typedef struct pa_block_pool pa_block_pool;

enum { PA_POOL_LIFO = 0, PA_POOL_FIFO = 1 };

/* free_order: NULL for 0..num_blocks-1, else a permutation of the ids giving
 * the initial free list. PA_POOL_LIFO hands out the list's last entry
 * ([P2] §4.2), PA_POOL_FIFO its first ([P1] §3); freed blocks go to the end.
 * Returns NULL on bad arguments or if free_order is not a permutation. */
pa_block_pool *pa_pool_create(int num_blocks, int block_size, int policy,
                              const int32_t *free_order);
void pa_pool_destroy(pa_block_pool *pool);
int pa_pool_num_free(const pa_block_pool *pool);
/* Reference count of a block (0 = free), or PA_ERR_POOL_STATE for a bad id. */
int pa_pool_ref_count(const pa_block_pool *pool, int block);
int pa_pool_allocate(pa_block_pool *pool, int32_t *block_out);
int pa_pool_share(pa_block_pool *pool, int block);
int pa_pool_free(pa_block_pool *pool, int block);

/*
 * Appends n_new tokens to a sequence whose host table row `table` (capacity
 * max_blocks) and token count *num_tokens describe it. Token t = *num_tokens
 * goes to table[t / bs] at offset t % bs: a new block is taken when t % bs == 0;
 * otherwise, if that block's count is above 1, it is copied first (the pair
 * (old, new) is appended to cow_pairs as two int64, the row is repointed).
 * slots (nullable) receives each new token's slot. cow_pairs (nullable when
 * cow_capacity is 0) has room for cow_capacity pairs; *num_cow receives the
 * count. On an error the tokens appended before it stay appended and
 * *num_tokens says how many there are.
 */
int pa_pool_append(pa_block_pool *pool, int32_t *table, int max_blocks, int32_t *num_tokens,
                   int n_new, int32_t *slots, int64_t *cow_pairs, int cow_capacity, int *num_cow);

/* Makes dst_table share every block of table (first ceil(num_tokens / bs)
 * entries): each count goes up by one. */
int pa_pool_fork(pa_block_pool *pool, const int32_t *table, int num_tokens, int32_t *dst_table,
                 int max_blocks);

/* Drops the sequence's reference to each of its blocks. */
int pa_pool_release(pa_block_pool *pool, const int32_t *table, int num_tokens);

/* Copies the pool's state out: ref_counts [num_blocks] and the free list
 * front first (free_list has room for num_blocks; *num_free receives its
 * length). With pa_dpool_load this hands a host pool over to the device. */
int pa_pool_export(const pa_block_pool *pool, int32_t *ref_counts, int32_t *free_list, int *num_free);

/*
 * Prefix cache over a host block pool ([P4] §3.2, Prefix Caching): a prompt
 * prefix (e.g. a system prompt shared by many requests) gets its blocks, and
 * its KV, once; later requests with the same prefix reuse them.
 *   - pa_prefix_get_or_create: if this exact token list is cached, its use
 *     count goes up by one and its block ids are written to block_ids
 *     (*hit = 1). Otherwise ceil(num_tokens / block_size) blocks are taken
 *     from the pool (PA_ERR_POOL_EXHAUSTED and nothing taken if the pool has
 *     fewer free blocks), recorded with use count 1 and returned (*hit = 0);
 *     the caller then writes the prefix's K/V into them. block_ids has room
 *     for max_blocks ids (PA_ERR_CAPACITY, nothing changed, if too few);
 *     *num_ids receives the count.
 *   - pa_prefix_release: an unknown token list is ignored; otherwise the use
 *     count drops by one and at zero every block of the entry is freed
 *     (pa_pool_free) and the entry removed.
 *   - The entry holds one pool reference per block. A sequence that maps the
 *     prefix blocks into its own table row should take its own references
 *     (pa_pool_fork over them) so that pa_pool_append copies a shared block
 *     before writing into it.
 * Entries are found by a 64-bit FNV-1a hash of the token ids, of which the
 * low hash_bits bits are kept (0 = all 64; small values only make lookups
 * slower), and a hit also needs equal token lists, so a hash collision never
 * shares blocks. tokens: host int32 [num_tokens]. The cache keeps a pointer
 * to the pool, which must outlive it; pa_prefix_cache_destroy frees no
 * blocks. Not thread-safe.
 */
typedef struct pa_prefix_cache pa_prefix_cache;

pa_prefix_cache *pa_prefix_cache_create(pa_block_pool *pool, int hash_bits);
void pa_prefix_cache_destroy(pa_prefix_cache *cache);
int pa_prefix_num_entries(const pa_prefix_cache *cache);
int pa_prefix_get_or_create(pa_prefix_cache *cache, const int32_t *tokens, int num_tokens,
                            int32_t *block_ids, int max_blocks, int *num_ids, int *hit);
int pa_prefix_release(pa_prefix_cache *cache, const int32_t *tokens, int num_tokens);
/* The use count of this token list (0 if it is not cached). */
int pa_prefix_ref_count(pa_prefix_cache *cache, const int32_t *tokens, int num_tokens);

/*
 * Device block pool and the beam-search step on the GPU.
 *
 * The pool's state lives in one caller-allocated DEVICE buffer of
 * pa_dpool_state_bytes(num_blocks) bytes (16-byte aligned), int32 words:
 *   [0] num_blocks  [1] block_size  [2] policy  [3] head  [4] count
 *   [5] a marker set by pa_dpool_init  [6..7] the beam step's own
 *   bookkeeping (a step count and a grid-barrier base; every step advances
 *   them, also a step that applies nothing)
 *   ref   = words + PA_DPOOL_HEADER_WORDS          [num_blocks] reference counts
 *   ring  = ref + num_blocks                       [num_blocks] free list: entries
 *           ring[(head + k) % num_blocks], k < count, front first
 *   then four scratch arrays of num_blocks words each (all zero / -1 between
 *   calls), then PA_DPOOL_TAIL_WORDS words of beam-step scratch (status
 *   words, per-chunk totals, a grid-barrier count). The library keeps no
 *   pointer to it.
 * Same rules as the host pool: PA_POOL_FIFO takes the free list's front,
 * PA_POOL_LIFO its back; freed blocks go to the back.
 */
#define PA_DPOOL_HEADER_WORDS 8
#define PA_DPOOL_ARRAYS 6
#define PA_DPOOL_TAIL_WORDS 1024

size_t pa_dpool_state_bytes(int num_blocks);

/* Every block free, counts 0. free_order (device int32 [num_blocks],
 * nullable) gives the initial free list, else 0 .. num_blocks-1; if it is
 * not a permutation the state is left unusable and PA_DEVERR_POOL is set. */
int pa_dpool_init(void *state, int num_blocks, int block_size, int policy, const int32_t *free_order,
                  cudaStream_t stream);

/* Loads a pool state (e.g. from pa_pool_export): ref_counts [num_blocks]
 * and free_list [num_free] (front first) are device int32 arrays. The free
 * list must hold distinct ids of count 0, and every block of count 0 must be
 * on it; otherwise the state is left unusable and PA_DEVERR_POOL is set. */
int pa_dpool_load(void *state, int num_blocks, int block_size, int policy, const int32_t *ref_counts,
                  const int32_t *free_list, int num_free, cudaStream_t stream);

/*
 * pa_beam_step -- one beam-search step on the device ([P2] §3.4: beams share
 * blocks and copy one before writing into it; [P4] §3.3: the copy-on-write
 * rule). New beam i (i < num_new) continues old beam parents[i] and writes
 * one token. The result equals, run one after another: every new beam forks
 * its parent (counts up); every old beam is released, beams in order and each
 * table in order (a block reaching 0 goes to the back of the free list);
 * every new beam writes its token in beam order: at a block boundary it
 * takes a free block, else if its block's count is above 1 it takes a free
 * block, appends (old, new) to cow_pairs and drops the old count, else it
 * writes in place.
 * Inputs (device): old_tables [num_old, max_blocks_per_seq] and
 * old_context_lens [num_old] (entries past ceil(ctx / block_size) are not
 * read), parents [num_new] in [0, num_old). Outputs (device):
 * new_tables [num_new, max_blocks_per_seq] (-1 past the blocks in use; must
 * not overlap old_tables), new_context_lens [num_new] = parent's + 1 (must
 * not overlap old_context_lens),
 * slot_mapping [num_new] (the new tokens' slots, for pa_reshape_and_cache),
 * cow_pairs int64 [num_new, 2] and *num_cow (for pa_copy_blocks_counted).
 * A table row never lists a block twice (the pool never makes one).
 * Any error (a bad parent, context or block id, a free list too short, no
 * table room for the new token, an uninitialised state) applies nothing:
 * counts, free list and header words 0-5 are unchanged, every slot is -1,
 * *num_cow = 0 and a PA_DEVERR_* bit is set. Runs over chunks of the old
 * tables spread over the SMs: one cooperative launch (up to 1024 new beams
 * and 1024 table entries per SM; its grid barriers wait at most 200 ms, and a
 * wait that gives up marks the state unusable), else four launches. Calls on
 * one state must not overlap.
 * Limits (else PA_ERR_SHAPE): 3 * num_old + num_new <= PA_BEAM_MAX_STAGED
 * and (num_old + num_new) * max_blocks_per_seq < 2^30.
 */
#define PA_BEAM_MAX_STAGED 24576
int pa_beam_step(void *state, int num_blocks, int block_size, const int32_t *old_tables,
                 const int32_t *old_context_lens, int num_old, const int32_t *parents, int num_new,
                 int32_t *new_tables, int32_t *new_context_lens, int max_blocks_per_seq,
                 int32_t *slot_mapping, int64_t *cow_pairs, int32_t *num_cow, cudaStream_t stream);

/*
 * pa_beam_step_withhold_arrival -- pa_beam_step (its one-launch form) with a
 * fault planted on the host, for testing the bounded grid barrier; not for
 * production use. CTA `cta` of the cooperative launch (CTA c takes old-table
 * entries c * chunk ..) never counts itself at the first grid barrier, so
 * every CTA's wait there runs out after wait_limit_ns (between 1e5 and 1e9;
 * the library's own bound is 200 ms). The step then applies nothing, sets
 * PA_DEVERR_TIMEOUT, every slot is -1 and *num_cow = 0, and the state is
 * marked unusable (header word 5 cleared): later steps on it report
 * PA_DEVERR_POOL until pa_dpool_init or pa_dpool_load. A CTA index past the
 * launch withholds nothing. The hook is compiled into a separate instance of
 * the kernel, so pa_beam_step's own carries none of it. Other arguments as
 * pa_beam_step; a step too large for the one-launch form, cta < 0 or the
 * limit out of range give PA_ERR_SHAPE.
 */
int pa_beam_step_withhold_arrival(void *state, int num_blocks, int block_size, const int32_t *old_tables,
                                  const int32_t *old_context_lens, int num_old, const int32_t *parents, int num_new,
                                  int32_t *new_tables, int32_t *new_context_lens, int max_blocks_per_seq,
                                  int32_t *slot_mapping, int64_t *cow_pairs, int32_t *num_cow, int cta,
                                  unsigned long long wait_limit_ns, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_KV_CACHE_340_B200_PA_H */
