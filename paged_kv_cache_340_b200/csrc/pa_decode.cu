// Paged decode attention for sm_100a: the fused one-pass kernel (whole
// sequence or one split-K partition per CTA) and the log-sum-exp reduce.
//
// What is computed: for sequence s and query head h (kv head h / G),
//   out = sum_t softmax_t(scale * q . K_t) V_t over the sequence's tokens,
// with K_t, V_t read in place through the block table ([P4 "PagedAttention
// 实现细节", §3.1, index-based kernel]; [P3 "Ascend C ... PagedAttention融合算子",
// §3: gather, QK^T, softmax and PV fused in one pass, no intermediate written
// back; §6: fp16 storage, fp32 arithmetic]).
//
// How (B200 design, not the pages'):
//   * one CTA per (sequence, kv head[, partition]); all G query heads of the
//     GQA group share every K/V tile, so each tile crosses HBM once;
//   * warp 4 is the producer: it reads the table row 32 entries at a time
//     (coalesced, prefetched one chunk ahead) and streams each (block, kv head)
//     K tile and V tile -- contiguous block_size*head_dim runs in this layout --
//     into a ring of shared-memory stages with one-dimensional bulk copies
//     (cp.async.bulk, TMA engine) completing on per-stage mbarriers;
//   * warps 0-3 are consumers; warp w takes stages w, w+4, ... Each 16-byte
//     lane vector covers 8 (16-bit) or 4 (fp32) elements of a token row; a
//     warp instruction covers 32 / (head_dim / vec) token rows ("row
//     groups"). Scores are reduced across the lanes of a row with a
//     transposing butterfly (each step halves the values a lane holds), so a
//     lane ends with whole scores and runs one exp per score, not one per lane;
//   * each row group keeps its own running max / sum / accumulator in fp32
//     (log2 domain: q is pre-scaled by scale * log2 e); the CTA merges the
//     row groups at the end, by the same log-sum-exp rule as the split-K
//     reduce;
//   * every wait is bounded (PA_DEVERR_TIMEOUT), bad table entries skip their
//     block (PA_DEVERR_BLOCK_ID).
#include <math.h>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <typename T, int D, int BS, int G>
struct DecodeShape {
    static constexpr int kElt = sizeof(T);
    static constexpr int kVec = 16 / kElt;             // elements per 16-byte lane vector
    static constexpr int kLpt = D / kVec;              // lanes per token row
    static constexpr int kRows = 32 / kLpt;            // token rows per warp instruction
    static constexpr int kTS = 16;                     // tokens per pipeline stage
    static constexpr int kSubs = BS / kTS;             // stages per physical block
    static constexpr int kTpg = kTS / kRows;           // tokens of one stage per row group
    static constexpr int kTc = (G * kTpg <= 32) ? kTpg : (32 / G);  // tokens per softmax chunk
    static constexpr int kChunks = kTpg / kTc;
    static constexpr int kNv = G * kTc;                // scores per lane before the butterfly
    static constexpr int kNvl = kNv >= kLpt ? kNv / kLpt : 1;   // scores a lane keeps
    static constexpr int kDup = kNv >= kLpt ? 1 : kLpt / kNv;   // lanes keeping the same score
    static constexpr int kLanesPerG = kLpt / G;        // lanes whose scores belong to one head
    static constexpr int kConsumerWarps = 4;
    static constexpr int kThreads = (kConsumerWarps + 1) * 32;
    static constexpr int kTileBytes = kTS * D * kElt;  // 16 token rows of one kv head, K or V
    static constexpr int kStageBytes = 2 * kTileBytes;
    // Stage k is consumed by warp k % 4 and lives in buffer k % 8, so the
    // previous use of a buffer always belongs to the same warp: a parity
    // wait can never see a phase two behind.
    static constexpr int kStages = 8;
    static constexpr int kRowGroups = kConsumerWarps * kRows;
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kMergeBytes = kRowGroups * G * (D + 2) * 4;
    static constexpr int kDataBytes = kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes;
    static constexpr int kSmemBytes = 128 + kDataBytes + kStages * 16 + kStages * 4;

    static_assert(kStages % kConsumerWarps == 0, "buffer reuse must stay within one warp");
    static_assert(BS % kTS == 0, "block size is a multiple of the stage");
    static_assert(kLpt >= 1 && kLpt <= 32 && (32 % kLpt) == 0, "row width");
    static_assert(kTS % kRows == 0 && kTpg % kTc == 0, "stage split");
    static_assert(G <= kLpt, "a lane's kept scores must belong to one query head");
    static_assert(kNvl <= kTc, "kept scores within one head");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

// Butterfly over the lanes of a token row (xor masks MK, MK/2, .., 1): while a
// lane holds N > 1 partial sums it keeps half and sends half, so after the
// halving steps lane c holds whole sums for scores [c*N0/L, ...).
template <int N, int MK>
struct RowReduce {
    static __device__ __forceinline__ void run(float *x, int lane) {
        if constexpr (MK >= 1) {
            if constexpr (N > 1) {
                constexpr int H = N / 2;
                const bool upper = (lane & MK) != 0;
#pragma unroll
                for (int j = 0; j < H; ++j) {
                    const float send = upper ? x[j] : x[j + H];
                    const float keep = upper ? x[j + H] : x[j];
                    x[j] = keep + __shfl_xor_sync(0xffffffffu, send, MK);
                }
                RowReduce<H, MK / 2>::run(x, lane);
            } else {
                x[0] += __shfl_xor_sync(0xffffffffu, x[0], MK);
                RowReduce<1, MK / 2>::run(x, lane);
            }
        }
    }
};

template <typename T, int D, int BS, int G>
__global__ void __launch_bounds__(DecodeShape<T, D, BS, G>::kThreads)
    decode_kernel(const DecodeParams p) {
    using S = DecodeShape<T, D, BS, G>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *ring = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    uint64_t *full = reinterpret_cast<uint64_t *>(ring + S::kDataBytes);
    uint64_t *empty = full + S::kStages;
    int *bad = reinterpret_cast<int *>(empty + S::kStages);

    const int part = blockIdx.x;
    const int kvh = blockIdx.y;
    const int s = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const bool split = p.partition_size > 0;

    // ---- token range of this CTA
    int ctx = p.context_lens[s];
    bool ctx_bad = false;
    if (ctx < 0) { ctx = 0; ctx_bad = true; }
    if (ctx > p.max_blocks_per_seq * BS) { ctx = p.max_blocks_per_seq * BS; ctx_bad = true; }
    if (split && ctx > p.max_context_len) { ctx = p.max_context_len; ctx_bad = true; }
    if (ctx_bad && threadIdx.x == 0 && part == 0 && kvh == 0) record_error(p.err, PA_DEVERR_CONTEXT);
    int t_begin = 0, t_end = ctx;
    if (split) {
        t_begin = part * p.partition_size;
        if (t_begin >= ctx) return;  // empty partition: nothing written
        t_end = min(t_begin + p.partition_size, ctx);
    }
    const int nblk = (t_end - t_begin + BS - 1) / BS;           // table entries read
    const int nstage = (t_end - t_begin + S::kTS - 1) / S::kTS;  // 16-token stages
    const size_t head0 = (size_t)s * p.num_heads + (size_t)kvh * G;  // first query head row
    if (nblk == 0) {  // unsplit, empty context: zeros
        for (int i = threadIdx.x; i < G * D; i += blockDim.x)
            store_out(p.out, head0 * D + i, 0.f, p.out_dtype);
        return;
    }
    const int first_block = t_begin / BS;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S::kStages; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, 1);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == S::kConsumerWarps) {
        // =========================== producer warp
        const int32_t *row = p.block_tables + (size_t)s * p.max_blocks_per_seq + first_block;
        const size_t block_elems = (size_t)p.num_kv_heads * BS * D;
        const size_t head_off = (size_t)kvh * BS * D;
        const T *kc = static_cast<const T *>(p.k_cache) + head_off;
        const T *vc = static_cast<const T *>(p.v_cache) + head_off;
        const uint64_t pol = l2_evict_first_policy();
        bool ok = true;
        int issued = 0;
        int next = lane < nblk ? __ldg(row + lane) : 0;
        for (int base = 0; base < nblk && ok; base += 32) {
            const int ids = next;
            if (base + 32 + lane < nblk) next = __ldg(row + base + 32 + lane);
            const int n = min(32, nblk - base);
            const bool valid = ids >= 0 && ids < p.num_blocks;
            if (lane < n && !valid) record_error(p.err, PA_DEVERR_BLOCK_ID);
            for (int j = 0; j < n; ++j) {
                const int b = __shfl_sync(0xffffffffu, ids, j);
                const bool v = __shfl_sync(0xffffffffu, valid ? 1 : 0, j) != 0;
#pragma unroll
                for (int h = 0; h < S::kSubs; ++h) {
                    const int k = (base + j) * S::kSubs + h;  // stage
                    if (k >= nstage) break;
                    if (lane == 0) {
                        const int buf = k % S::kStages;
                        if (k >= S::kStages && !mbar_wait(empty + buf, ((k / S::kStages) - 1) & 1)) {
                            ok = false;
                            record_error(p.err, PA_DEVERR_TIMEOUT);
                        } else {
                            if (v) {
                                bad[buf] = 0;
                                unsigned char *dst = ring + (size_t)buf * S::kStageBytes;
                                const size_t src = (size_t)b * block_elems + (size_t)h * S::kTS * D;
                                mbar_arrive_expect_tx(full + buf, S::kStageBytes);
                                bulk_load(dst, kc + src, S::kTileBytes, full + buf, pol);
                                bulk_load(dst + S::kTileBytes, vc + src, S::kTileBytes, full + buf, pol);
                            } else {
                                bad[buf] = 1;
                                mbar_arrive(full + buf);
                            }
                            ++issued;
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                    if (!ok) break;
                }
                if (!ok) break;
            }
        }
        // Before exiting, every copy this CTA started must have landed.
        if (lane == 0) {
            for (int k = max(0, issued - S::kStages); k < issued; ++k)
                if (!mbar_wait(full + (k % S::kStages), (k / S::kStages) & 1))
                    record_error(p.err, PA_DEVERR_TIMEOUT);
        }
        return;
    }

    // =============================== consumer warps
    const int r = lane / S::kLpt;          // row within the warp instruction
    const int c = lane % S::kLpt;          // 16-byte column of the row
    const int rg = warp * S::kRows + r;    // row group
    const int g_lane = c / S::kLanesPerG;  // query head of this lane's kept scores
    const int v0 = (c * S::kNv) / S::kLpt; // index of this lane's first kept score
    const bool counts_l = (c % S::kDup) == 0;

    float q[G][S::kVec];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const uint4 u = *reinterpret_cast<const uint4 *>(static_cast<const T *>(p.query) +
                                                         (head0 + g) * D + c * S::kVec);
        Elt<T>::unpack(u, q[g]);
#pragma unroll
        for (int e = 0; e < S::kVec; ++e) q[g][e] *= p.scale_log2;
    }
    float m_run[G];
    float acc[G][S::kVec];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m_run[g] = -INFINITY;
#pragma unroll
        for (int e = 0; e < S::kVec; ++e) acc[g][e] = 0.f;
    }
    float l_lane = 0.f;

    for (int k = warp; k < nstage; k += S::kConsumerWarps) {
        const int buf = k % S::kStages;
        const bool got = mbar_wait(full + buf, (k / S::kStages) & 1);
        if (!__all_sync(0xffffffffu, got)) {
            if (lane == 0) record_error(p.err, PA_DEVERR_TIMEOUT);
            break;
        }
        if (!bad[buf]) {
            const int nvalid = min(S::kTS, t_end - (t_begin + k * S::kTS));
            const unsigned char *Ks = ring + (size_t)buf * S::kStageBytes;
            const unsigned char *Vs = Ks + S::kTileBytes;
#pragma unroll
            for (int ci = 0; ci < S::kChunks; ++ci) {
                // ---- scores: partial dots over this lane's columns
                float sc[S::kNv];
#pragma unroll
                for (int i = 0; i < S::kTc; ++i) {
                    const int t = (ci * S::kTc + i) * S::kRows + r;
                    const uint4 u = *reinterpret_cast<const uint4 *>(
                        Ks + ((size_t)t * D + c * S::kVec) * S::kElt);
                    float kf[S::kVec];
                    Elt<T>::unpack(u, kf);
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        float d0 = 0.f;
#pragma unroll
                        for (int e = 0; e < S::kVec; ++e) d0 = fmaf(q[g][e], kf[e], d0);
                        sc[g * S::kTc + i] = d0;
                    }
                }
                RowReduce<S::kNv, S::kLpt / 2>::run(sc, lane);
                // ---- mask the tail and take the chunk max per head
                float cmax = -INFINITY;
#pragma unroll
                for (int j = 0; j < S::kNvl; ++j) {
                    const int i = (v0 + j) % S::kTc;
                    const int t = (ci * S::kTc + i) * S::kRows + r;
                    if (t >= nvalid) sc[j] = -INFINITY;
                    cmax = fmaxf(cmax, sc[j]);
                }
#pragma unroll
                for (int mk = 1; mk < S::kLanesPerG; mk <<= 1)
                    cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, mk));
                float my_m = 0.f, my_alpha = 1.f;
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float cm = (G == 1) ? cmax
                                              : __shfl_sync(0xffffffffu, cmax,
                                                            r * S::kLpt + g * S::kLanesPerG);
                    const float mn = fmaxf(m_run[g], cm);
                    const float alpha = (mn == -INFINITY) ? 1.f : fast_exp2(m_run[g] - mn);
                    m_run[g] = mn;
#pragma unroll
                    for (int e = 0; e < S::kVec; ++e) acc[g][e] *= alpha;
                    if (g == g_lane) { my_m = mn; my_alpha = alpha; }
                }
                // ---- probabilities of the kept scores
                float pk[S::kNvl];
                float psum = 0.f;
#pragma unroll
                for (int j = 0; j < S::kNvl; ++j) {
                    pk[j] = (sc[j] == -INFINITY) ? 0.f : fast_exp2(sc[j] - my_m);
                    psum += pk[j];
                }
                l_lane = l_lane * my_alpha + (counts_l ? psum : 0.f);
                // ---- PV: broadcast each token's probability along its row
#pragma unroll
                for (int i = 0; i < S::kTc; ++i) {
                    const int t = (ci * S::kTc + i) * S::kRows + r;
                    const uint4 u = *reinterpret_cast<const uint4 *>(
                        Vs + ((size_t)t * D + c * S::kVec) * S::kElt);
                    float vf[S::kVec];
                    Elt<T>::unpack(u, vf);
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        constexpr int kNvl = S::kNvl;
                        const int v = g * S::kTc + i;
                        const int src_c = (v * S::kLpt) / S::kNv;
                        const float pv = __shfl_sync(0xffffffffu, pk[v % kNvl], r * S::kLpt + src_c);
                        if (t < nvalid) {
#pragma unroll
                            for (int e = 0; e < S::kVec; ++e) acc[g][e] = fmaf(pv, vf[e], acc[g][e]);
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + buf);
    }

    // ---- merge the row groups (log-sum-exp), reusing the ring
#pragma unroll
    for (int mk = 1; mk < S::kLanesPerG; mk <<= 1) l_lane += __shfl_xor_sync(0xffffffffu, l_lane, mk);
    named_bar_sync(1, S::kConsumerWarps * 32);  // every consumer is done with the ring
    float *mg = reinterpret_cast<float *>(ring);    // [row group][G]
    float *lg = mg + S::kRowGroups * G;            // [row group][G]
    float *ag = lg + S::kRowGroups * G;            // [row group][G][D]
    if (c % S::kLanesPerG == 0) {
        float mine = 0.f;
#pragma unroll
        for (int g = 0; g < G; ++g)
            if (g == g_lane) mine = m_run[g];
        mg[rg * G + g_lane] = mine;
        lg[rg * G + g_lane] = l_lane;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float4 *dst = reinterpret_cast<float4 *>(ag + ((size_t)rg * G + g) * D + c * S::kVec);
#pragma unroll
        for (int e = 0; e < S::kVec; e += 4)
            dst[e / 4] = make_float4(acc[g][e], acc[g][e + 1], acc[g][e + 2], acc[g][e + 3]);
    }
    named_bar_sync(1, S::kConsumerWarps * 32);
    for (int idx = threadIdx.x; idx < G * D; idx += S::kConsumerWarps * 32) {
        const int g = idx / D;
        const int d = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int i = 0; i < S::kRowGroups; ++i) M = fmaxf(M, mg[i * G + g]);
        float num = 0.f, den = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int i = 0; i < S::kRowGroups; ++i) {
                const float w = fast_exp2(mg[i * G + g] - M);
                num = fmaf(w, ag[((size_t)i * G + g) * D + d], num);
                den = fmaf(w, lg[i * G + g], den);
            }
        }
        const size_t h = head0 + g;
        if (split) {
            const size_t slot = h * p.max_parts + part;
            p.ws_acc[slot * D + d] = num;
            if (d == 0) {
                p.ws_ml[slot * 2] = M * kLn2;
                p.ws_ml[slot * 2 + 1] = den;
            }
        } else {
            store_out(p.out, h * D + d, den > 0.f ? num / den : 0.f, p.out_dtype);
        }
    }
}

// -------------------------------------------------------------- split reduce

__global__ void __launch_bounds__(128)
    splitk_reduce_kernel(void *out, const float *ws_ml, const float *ws_acc,
                         const int32_t *context_lens, int num_heads, int head_dim,
                         int partition_size, int max_parts, int max_context_len,
                         pa_dtype out_dtype) {
    extern __shared__ float wsm[];  // [max_parts] weights
    __shared__ float red[4];
    __shared__ float bcast;
    const int h = blockIdx.x;
    const int s = blockIdx.y;
    const int tid = threadIdx.x;
    int ctx = context_lens[s];
    ctx = max(0, min(ctx, max_context_len));
    const int n = (ctx + partition_size - 1) / partition_size;
    const size_t row = (size_t)s * num_heads + h;
    if (n == 0) {
        for (int d = tid; d < head_dim; d += blockDim.x) store_out(out, row * head_dim + d, 0.f, out_dtype);
        return;
    }
    const float *ml = ws_ml + row * max_parts * 2;
    const float *acc = ws_acc + row * max_parts * head_dim;
    // M = max_p m_p
    float M = -INFINITY;
    for (int i = tid; i < n; i += blockDim.x) M = fmaxf(M, ml[2 * i]);
    for (int mk = 16; mk >= 1; mk >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, mk));
    if ((tid & 31) == 0) red[tid >> 5] = M;
    __syncthreads();
    if (tid == 0) bcast = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    __syncthreads();
    M = bcast;
    // w_p = e^(m_p - M); den = sum_p w_p l_p
    float den = 0.f;
    for (int i = tid; i < n; i += blockDim.x) {
        const float w = fast_exp2((ml[2 * i] - M) * kLog2e);
        wsm[i] = w;
        den = fmaf(w, ml[2 * i + 1], den);
    }
    for (int mk = 16; mk >= 1; mk >>= 1) den += __shfl_xor_sync(0xffffffffu, den, mk);
    __syncthreads();  // red[] reuse and wsm[] visibility
    if ((tid & 31) == 0) red[tid >> 5] = den;
    __syncthreads();
    den = red[0] + red[1] + red[2] + red[3];
    for (int d = tid; d < head_dim; d += blockDim.x) {
        float num = 0.f;
        for (int i = 0; i < n; ++i) num = fmaf(wsm[i], acc[(size_t)i * head_dim + d], num);
        store_out(out, row * head_dim + d, den > 0.f ? num / den : 0.f, out_dtype);
    }
}

// ------------------------------------------------------------------ launchers

template <typename T, int D, int BS, int G>
static cudaError_t launch_decode_t(const DecodeParams &p, int grid_x, int num_kv_heads, int num_seqs,
                                   cudaStream_t stream) {
    using S = DecodeShape<T, D, BS, G>;
    auto kern = decode_kernel<T, D, BS, G>;
    static unsigned int attr_done = 0;  // one bit per device
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(kern), S::kSmemBytes, &attr_done);
    if (e != cudaSuccess) return e;
    dim3 grid(grid_x, num_kv_heads, num_seqs);
    kern<<<grid, S::kThreads, S::kSmemBytes, stream>>>(p);
    return cudaGetLastError();
}

template <typename T, int D, int BS>
static cudaError_t dispatch_group(const DecodeParams &p, int group, int grid_x, int num_kv_heads,
                                  int num_seqs, cudaStream_t stream) {
    switch (group) {
        case 1: return launch_decode_t<T, D, BS, 1>(p, grid_x, num_kv_heads, num_seqs, stream);
        case 2: return launch_decode_t<T, D, BS, 2>(p, grid_x, num_kv_heads, num_seqs, stream);
        case 4: return launch_decode_t<T, D, BS, 4>(p, grid_x, num_kv_heads, num_seqs, stream);
        case 8: return launch_decode_t<T, D, BS, 8>(p, grid_x, num_kv_heads, num_seqs, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
static cudaError_t dispatch_shape(const DecodeParams &p, int head_dim, int block_size, int group,
                                  int grid_x, int num_kv_heads, int num_seqs, cudaStream_t stream) {
    if (head_dim == 64 && block_size == 16) return dispatch_group<T, 64, 16>(p, group, grid_x, num_kv_heads, num_seqs, stream);
    if (head_dim == 64 && block_size == 32) return dispatch_group<T, 64, 32>(p, group, grid_x, num_kv_heads, num_seqs, stream);
    if (head_dim == 128 && block_size == 16) return dispatch_group<T, 128, 16>(p, group, grid_x, num_kv_heads, num_seqs, stream);
    if (head_dim == 128 && block_size == 32) return dispatch_group<T, 128, 32>(p, group, grid_x, num_kv_heads, num_seqs, stream);
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const DecodeParams &p, pa_dtype kv_dtype, int head_dim, int block_size,
                          int group, int grid_x, int num_kv_heads, int num_seqs,
                          cudaStream_t stream) {
    switch (kv_dtype) {
        case PA_F32: return dispatch_shape<float>(p, head_dim, block_size, group, grid_x, num_kv_heads, num_seqs, stream);
        case PA_F16: return dispatch_shape<__half>(p, head_dim, block_size, group, grid_x, num_kv_heads, num_seqs, stream);
        case PA_BF16: return dispatch_shape<__nv_bfloat16>(p, head_dim, block_size, group, grid_x, num_kv_heads, num_seqs, stream);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_splitk_reduce(void *out, const float *ws_ml, const float *ws_acc,
                                 const int32_t *context_lens, int num_seqs, int num_heads,
                                 int head_dim, int partition_size, int max_parts,
                                 int max_context_len, pa_dtype out_dtype, cudaStream_t stream) {
    const size_t smem = (size_t)max_parts * sizeof(float);
    if (smem > 48 * 1024) {
        static unsigned int attr_done = 0;
        cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(splitk_reduce_kernel),
                                         227 * 1024, &attr_done);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(num_heads, num_seqs);
    splitk_reduce_kernel<<<grid, 128, smem, stream>>>(out, ws_ml, ws_acc, context_lens, num_heads,
                                                      head_dim, partition_size, max_parts,
                                                      max_context_len, out_dtype);
    return cudaGetLastError();
}

}  // namespace pa
