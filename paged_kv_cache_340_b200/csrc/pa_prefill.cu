// Paged prefill (chunked prefill) attention for sm_100a on the 5th-generation
// tensor cores.
//
// What is computed: sequence s has q_len new query tokens (rows q_start[s] ..
// of query), already written into its paged cache; query token i sits at
// position pos = context_len - q_len + i and attends causally to the cache
// tokens 0 .. pos: out = softmax(scale q . K_t) V over t <= pos. Decode is
// q_len = 1. ([P4 "PagedAttention 实现细节", §3.4: the model forward over the
// step's new tokens, each layer's attention over the paged cache]; [P3 "Ascend
// C ... PagedAttention融合算子", §3.1: a num_tokens axis of queries].)
//
// How (B200 design): one CTA per (sequence, kv head, 128-row query tile); the
// rows are (token, query head of the GQA group) pairs, so every K/V tile is
// loaded once for the whole group.
//   * warp 5 loads: the Q tile once and the K/V tiles (64 tokens, gathered
//     block by block through the table, 32 lookups at a time, one per lane)
//     with 2-D/3-D TMA tensor copies in the 128-byte swizzled layout, into
//     two stages each, refilling a stage once the product that read it is done;
//   * warp 4 lane 0 issues S = Q K^T (M 128, N 64, K = head_dim in 8 steps)
//     into one of two S buffers and O += P V (M 128, N = head_dim, K 64 in 4
//     steps) as tcgen05.mma with the fp32 accumulators S and O in tensor
//     memory; tcgen05.commit signals each product's completion on an mbarrier;
//   * warps 0-3 run the softmax: thread r owns row r (tensor-memory lane r),
//     reads its S row with tcgen05.ld, masks positions past its token
//     (causal) and past the context, keeps the running max and sum in fp32
//     (log2 domain), rescales its O row in tensor memory when the max rises
//     by more than 2^8, and writes its probabilities with tcgen05.st as a
//     16-bit row over its own S row, where O += P V reads them (the A operand
//     from tensor memory); the four warps do not wait for each other;
//   * V rows past the context are zeroed in shared memory before P V (they
//     may hold anything, and 0 * NaN is NaN on the tensor cores too).
// Every wait is bounded (PA_DEVERR_TIMEOUT); tensor memory is always freed.
#include <cuda.h>

#include <mutex>
#include <type_traits>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {
namespace prefill {

constexpr int kM = 128;                 // query rows per CTA
constexpr int kN = 64;                  // kv tokens per tile
constexpr int kHalfBytes = 128;         // one swizzled row: 64 16-bit elements
constexpr int kQHalf = kM * kHalfBytes; // 16 KB: rows x d 0-63 (or 64-127)
constexpr int kKVHalf = kN * kHalfBytes;  // 8 KB
constexpr int kSoftmaxWarps = 4;
constexpr int kMmaWarp = kSoftmaxWarps;       // warp 4: issues the tensor-core MMAs
constexpr int kLoadWarp = kSoftmaxWarps + 1;  // warp 5: table lookups and TMA copies
constexpr int kThreads = (kSoftmaxWarps + 2) * 32;
// tensor memory (256 columns x 128 lanes, lane = query row): O and two S
// buffers. The softmax of tile j writes P_j (16-bit pairs; bf16 also its low
// part P - bf16(P)) over its own S_j, and O += P_j V_j reads it from there:
// S_{j+1} is computed while the softmax of tile j runs.
constexpr int kTmemCols = 256;
constexpr int kOCol = 0;      // O: head_dim (64 or 128) fp32 columns
constexpr int kSCol = 128;    // S buffers 0, 1: 64 fp32 columns each
constexpr int kPlOff = 32;    // within an S buffer: P at +0, P's low part at +32

// Shared-memory layout for head_dim D (64 or 128; every operand region
// 1024-byte aligned for the swizzle): Q, and two stages each of K and V, each
// stored as D / 64 swizzled halves of 64 columns.
template <int D>
struct Layout {
    static_assert(D == 64 || D == 128, "head_dim");
    static constexpr int kHalves = D / 64;
    static constexpr int kQBytes = kHalves * kQHalf;
    static constexpr int kKVBytes = kHalves * kKVHalf;  // one K or V tile
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;       // K stages 0, 1
    static constexpr int kOffV = kOffK + 2 * kKVBytes;  // V stages 0, 1
    static constexpr int kOffBar = kOffV + 2 * kKVBytes;
    static constexpr int kSmemBytes = 1024 + kOffBar + 24 * 8;  // ~97 KB at D 128: two CTAs per SM
};
// The running max is raised only when it grows by more than this (log2
// units): probabilities then stay below 2^8 and O is rarely rescaled.
constexpr float kRescaleThreshold = 8.f;

struct Params {
    void *out;
    const int32_t *q_start;
    // rows of a CTA are (token, head slot) pairs: 2^gshift head slots per
    // token (the head group rounded up to a power of two, at most 128); slots
    // past the group are padding, computed but never written. A group above
    // 128 runs as sub_groups CTAs along gridDim.y (kv head = blockIdx.y /
    // sub_groups), each over 128 of its query heads.
    int group;
    int gshift;
    int sub_groups;
    const int32_t *block_tables;
    const int32_t *context_lens;
    int max_blocks_per_seq;
    int num_heads;
    int num_kv_heads;
    int num_blocks;
    int block_size;
    long long kv_rows;  // num_blocks * num_kv_heads * block_size (rows of the 2-D pool view)
    float scale_log2;
    pa_dtype out_dtype;
    unsigned int *err;
    // test hook (pa_prefill_withhold_tile): the CTA of (sequence, kv head,
    // query tile) never issues the copy of its K tile withhold_tile (-1:
    // none), and every wait gives up after wait_limit_ns (0: kWaitLimitNs)
    int withhold_seq = -1, withhold_kvh = -1, withhold_qt = -1, withhold_tile = -1;
    unsigned long long wait_limit_ns = 0;
};

// ---------------------------------------------------------------- helpers

// Shared-memory matrix descriptor, 128-byte swizzle (tcgen05 format: start,
// leading and stride byte offsets in 16-byte units, version 1).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16 with fp32 accumulation.
__host__ __device__ constexpr uint32_t mma_idesc(bool bf16, int M, int N, bool b_mn_major) {
    return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                     uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
                 :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
                 : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int c0, int c1, int c2,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
        "[%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

template <typename T> struct Pack16;
template <> struct Pack16<__nv_bfloat16> {
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&v);
    }
};
template <> struct Pack16<__half> {
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&v);
    }
};

// ----------------------------------------------------------------- kernel

// A operand in tensor memory: O += A B with A read from TMEM columns.
__device__ __forceinline__ void umma_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 consecutive outputs of one row in the output type, as 16-byte stores at
// `dst` (global or shared memory, 16-byte aligned).
__device__ __forceinline__ void store_row32(unsigned char *dst, const float (&v)[32], pa_dtype dt) {
    if (dt == PA_F32) {
        float4 *d = reinterpret_cast<float4 *>(dst);
#pragma unroll
        for (int e = 0; e < 8; ++e) d[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
    } else if (dt == PA_BF16) {
        uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) w[i] = Pack16<__nv_bfloat16>::pack(v[8 * e + 2 * i], v[8 * e + 2 * i + 1]);
            d[e] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    } else {
        uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) w[i] = Pack16<__half>::pack(v[8 * e + 2 * i], v[8 * e + 2 * i + 1]);
            d[e] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

// Barrier over the softmax warps only (named barrier 1): true when `v` holds
// in every one of their threads.
__device__ __forceinline__ bool softmax_sync_and(bool v) {
    uint32_t all;
    asm volatile(
        "{\n\t.reg .pred pv, pa;\n\t"
        "setp.ne.u32 pv, %1, 0;\n\t"
        "barrier.cta.red.and.pred pa, 1, %2, pv;\n\t"
        "selp.u32 %0, 1, 0, pa;\n\t}"
        : "=r"(all)
        : "r"((uint32_t)v), "n"(kSoftmaxWarps * 32)
        : "memory");
    return all != 0;
}

// kGS: log2 of the head slots per token when the head group is exactly 1, 2,
// 4 or 8 (no padding, no sub-groups; compiled for that size), or -1 for any
// other group (slots and sub-groups from Params). Groups of 1-2 stage their
// output rows in shared memory; larger ones store one row per thread.
template <typename T, int kD, int kGS, bool kHook = false>
__global__ void __launch_bounds__(kThreads, 2)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, const Params p) {
    using L = Layout<kD>;
    constexpr int kQBytes = L::kQBytes, kKVBytes = L::kKVBytes, kOffQ = L::kOffQ, kOffK = L::kOffK,
                  kOffV = L::kOffV, kOffBar = L::kOffBar, kHalves = L::kHalves;
    constexpr bool kBf16 = std::is_same_v<T, __nv_bfloat16>;
    constexpr uint32_t kIdescQK = mma_idesc(kBf16, kM, kN, false);
    constexpr uint32_t kIdescPV = mma_idesc(kBf16, kM, kD, true);
    constexpr bool kExact = kGS >= 0;
    constexpr bool kStagedOut = kGS == 0 || kGS == 1;
    const int gshift = kExact ? kGS : p.gshift;
    const int G = 1 << gshift;                         // head slots per token
    const int kTokPerTile = kM >> gshift;

    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *Qs = sm + kOffQ;
    unsigned char *Ks = sm + kOffK;  // stage b at Ks + b * kKVBytes
    unsigned char *Vs = sm + kOffV;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kOffBar);
    uint64_t *q_full = bars + 0;
    uint64_t *k_full = bars + 1;    // [2] stage loaded
    uint64_t *v_full = bars + 3;    // [2]
    uint64_t *k_empty = bars + 5;   // [2] S that read the stage is done
    uint64_t *v_empty = bars + 7;   // [2] PV that read the stage is done
    uint64_t *s_full = bars + 9;    // [2] S buffer computed
    // [2] softmax of tile j done (P_j written), on p_full[j & 1]: the softmax
    // warps do not wait for each other, and one may reach tile j + 1 before
    // another has finished tile j (never tile j + 2, whose S needs P_j V_j),
    // so the arrivals of neighbouring tiles go to different barriers
    uint64_t *p_full = bars + 11;
    uint64_t *o_done = bars + 13;   // PV of the tile done
    uint64_t *mma_idle = bars + 14; // every MMA issued has finished (end of kernel)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 15);
    int *abort_flag = reinterpret_cast<int *>(bars + 16);
    // test hook (kHook instances only): the wait bound and this CTA's
    // withheld K tile, set with the barriers; other instances wait with the
    // library's bound and withhold nothing
    uint64_t *const wl = kHook ? bars + 17 : nullptr;
    int *const withheld = reinterpret_cast<int *>(bars + 18);

    const int qt = gridDim.x - 1 - blockIdx.x;  // longest query tile of each (head, sequence) first
    const int kvh = (!kExact && p.sub_groups > 1) ? (int)blockIdx.y / p.sub_groups : (int)blockIdx.y;
    const int sub = (!kExact && p.sub_groups > 1) ? (int)blockIdx.y % p.sub_groups : 0;
    const int head_base = kExact ? kvh * G : kvh * p.group + sub * G;  // query head of slot 0
    const int g_valid = kExact ? G : min(G, p.group - sub * G);         // slots holding a real query head
    const int s = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const int q0 = p.q_start[s];
    const int q_len = p.q_start[s + 1] - q0;
    const int ctx = p.context_lens[s];
    const int tok0 = qt * kTokPerTile;
    if (tok0 >= q_len) return;
    if (q_len > ctx || ctx > p.max_blocks_per_seq * p.block_size) {
        if (threadIdx.x == 0) record_error(p.err, PA_DEVERR_CONTEXT);
        return;
    }
    const int rows_valid = min(kM, (q_len - tok0) * G);
    const int pos0 = ctx - q_len + tok0;                      // position of the tile's first token
    const int pos_max = pos0 + (rows_valid >> gshift) - 1;
    const int ntiles = pos_max / kN + 1;

    // Pool row of the load warp's 16-token group g0 + lane (16 tokens from
    // (g0 + lane) * 16), past the pool's end when the sequence has no such
    // block (the copy then reads zeros).
    const int32_t *trow = p.block_tables + (size_t)s * p.max_blocks_per_seq;
    const int nblk = (ctx + p.block_size - 1) / p.block_size;
    auto rows_from = [&](int g0) -> int {
        const int g = g0 + lane;
        const int tok = g * 16;
        const int lb = tok / p.block_size;
        long long row = p.kv_rows;
        if (lb < nblk) {
            const int id = __ldg(trow + lb);
            if (id >= 0 && id < p.num_blocks)
                row = ((long long)id * p.num_kv_heads + kvh) * p.block_size + (tok % p.block_size);
            else
                record_error(p.err, PA_DEVERR_BLOCK_ID);
        }
        return (int)row;
    };
    // The load warp starts its first table lookups and the Q copy before the
    // tensor-memory allocation and the CTA barrier, so their latency overlaps
    // the setup.
    int rows = 0, rows_next = 0;  // pool rows of groups g0 .. g0 + 31 and of the next 32
    if (warp == kLoadWarp) {
        rows = rows_from(0);
        rows_next = rows_from(32);
        if (lane == 0) {
            mbar_init(q_full, 1);
            for (int i = 0; i < 2; ++i) {
                mbar_init(k_full + i, 1);
                mbar_init(v_full + i, 1);
                mbar_init(k_empty + i, 1);
                mbar_init(v_empty + i, 1);
                mbar_init(s_full + i, 1);
                mbar_init(p_full + i, kSoftmaxWarps * 32);
            }
            mbar_init(o_done, 1);
            mbar_init(mma_idle, 1);
            *abort_flag = 0;
            if constexpr (kHook) {
                *wl = p.wait_limit_ns ? p.wait_limit_ns : kWaitLimitNs;
                *withheld = (s == p.withhold_seq && kvh == p.withhold_kvh && sub == 0 && qt == p.withhold_qt)
                                ? p.withhold_tile : -1;
            }
            fence_mbar_init();
            fence_proxy_async_smem();  // the initialised barriers, before the copy that signals one
            mbar_arrive_expect_tx(q_full, kQBytes);
#pragma unroll
            for (int h = 0; h < kHalves; ++h) tma_load_3d(Qs + h * kQHalf, &tmap_q, 64 * h, head_base, q0 + tok0, q_full);
        }
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kLoadWarp) {
        // ========================================================= load warp
        // Tile j goes into K/V stage j & 1 (its use j >> 1 of the stage); a
        // stage is refilled once the S (K) or PV (V) product that read it is
        // done. Block ids of 32 16-token groups are looked up at a time, one
        // per lane.
        constexpr int kGroups = kN / 16;  // 16-token groups per tile
        int k_issued = 0, v_issued = 0;
        bool ok = true;
        for (int j = 0; j < ntiles && ok; ++j) {
            const int b = j & 1;
            const int g0 = j * kGroups;
            if (g0 % 32 == 0 && j > 0) {  // the lookups for the next 32 groups start a batch ahead
                rows = rows_next;
                rows_next = rows_from(g0 + 32);
            }
            int r4[kGroups];
#pragma unroll
            for (int g = 0; g < kGroups; ++g) r4[g] = __shfl_sync(0xffffffffu, rows, (g0 + g) % 32);
            for (int kv = 0; kv < 2; ++kv) {
                uint64_t *empty = (kv == 0 ? k_empty : v_empty) + b;
                if (j >= 2) {  // every lane waits; the outcome is made warp-uniform
                    const bool got = mbar_wait(empty, ((j >> 1) - 1) & 1, wl) && !*(volatile int *)abort_flag;
                    if (!__all_sync(0xffffffffu, got)) {
                        ok = false;
                        break;
                    }
                }
                if (lane == 0 && !(kHook && kv == 0 && j == *withheld)) {  // (test hook: never issued)
                    uint64_t *full = (kv == 0 ? k_full : v_full) + b;
                    unsigned char *dst = (kv == 0 ? Ks : Vs) + b * kKVBytes;
                    const CUtensorMap *map = kv == 0 ? &tmap_k : &tmap_v;
                    mbar_arrive_expect_tx(full, kKVBytes);
#pragma unroll
                    for (int g = 0; g < kGroups; ++g)
#pragma unroll
                        for (int h = 0; h < kHalves; ++h)
                            tma_load_2d(dst + h * kKVHalf + g * 16 * kHalfBytes, map, h * 64, r4[g], full);
                }
                if (kv == 0) ++k_issued; else ++v_issued;
            }
        }
        if (!ok) {
            if (lane == 0) {
                record_error(p.err, PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
        }
        // let the copies this warp started land before the CTA leaves
        // (normally the MMA warp has consumed them all: these waits return at once)
        if (lane == 0) {
            mbar_wait(q_full, 0, wl);
            for (int j = max(0, k_issued - 2); j < k_issued; ++j) mbar_wait(k_full + (j & 1), (j >> 1) & 1, wl);
            for (int j = max(0, v_issued - 2); j < v_issued; ++j) mbar_wait(v_full + (j & 1), (j >> 1) & 1, wl);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ========================================================== MMA warp
        // S_0, S_1; then per tile j: (softmax j done) O += P_j V_j; (that
        // product done, so P_j's buffer is free) S_{j+2} into the same buffer.
        if (lane == 0) {
            const uint32_t qa = smem_addr(Qs);
            bool ok = mbar_wait(q_full, 0, wl);
            bool issued = false;
            auto issue_s = [&](int j) -> bool {
                const int b = j & 1;
                if (!mbar_wait(k_full + b, (j >> 1) & 1, wl) || *(volatile int *)abort_flag) return false;
                tc_fence_after();
                const uint32_t ka = smem_addr(Ks + b * kKVBytes);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (kk & 3) * 32;
                    umma(tmem + kSCol + b * kN, sw128_desc(qa + (kk >> 2) * kQHalf + off, 16, 1024),
                         sw128_desc(ka + (kk >> 2) * kKVHalf + off, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
                }
                umma_commit(s_full + b);
                umma_commit(k_empty + b);
                issued = true;
                return true;
            };
            for (int j = 0; ok && j < min(2, ntiles); ++j) ok = issue_s(j);
            for (int j = 0; ok && j < ntiles; ++j) {
                const int b = j & 1;
                if (!mbar_wait(p_full + b, (j >> 1) & 1, wl) || !mbar_wait(v_full + b, (j >> 1) & 1, wl) ||
                    *(volatile int *)abort_flag) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t va = smem_addr(Vs + b * kKVBytes);
                const uint32_t pcol = tmem + kSCol + b * kN;
#pragma unroll
                for (int kk = 0; kk < kN / 16; ++kk) {
                    const uint64_t vdesc = sw128_desc(va + kk * 16 * kHalfBytes, kKVHalf, 1024);
                    umma_ta(tmem + kOCol, pcol + kk * 8, vdesc, kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
                    if constexpr (kBf16) umma_ta(tmem + kOCol, pcol + kPlOff + kk * 8, vdesc, kIdescPV, 1u);
                }
                umma_commit(o_done);
                umma_commit(v_empty + b);
                if (j + 2 < ntiles) {
                    if (!mbar_wait(o_done, j & 1, wl)) { ok = false; break; }
                    ok = issue_s(j + 2);
                }
            }
            if (!ok) {
                record_error(p.err, PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
                mbar_arrive(s_full);      // release the softmax warps from their waits
                mbar_arrive(s_full + 1);
                mbar_arrive(o_done);
            }
            // tensor memory is freed below, and the softmax warps read O: every MMA
            // must have finished (with none issued, release the waiters at once)
            if (issued) {
                umma_commit(mma_idle);
                if (!mbar_wait(mma_idle, 0, wl)) record_error(p.err, PA_DEVERR_TIMEOUT);
            } else {
                mbar_arrive(mma_idle);
            }
        }
        __syncwarp();
    } else {
        // ======================================================= softmax warps
        const int r = threadIdx.x;  // row = tensor-memory lane
        const int tok = r >> gshift;
        const bool valid = r < rows_valid;
        const int pos = valid ? pos0 + tok : -1;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const float sl2 = p.scale_log2;
        float m_run = -INFINITY, l_run = 0.f;
        for (int j = 0; j < ntiles; ++j) {
            const int b = j & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(s_full + b, (j >> 1) & 1, wl) && !*(volatile int *)abort_flag))
                break;
            tc_fence_after();
            const uint32_t sbuf = tmem + lane_base + kSCol + b * kN;
            uint32_t sr[2][32];
            tmem_ld32(sbuf, sr[0]);
            tmem_ld32(sbuf + 32, sr[1]);
            tmem_wait_ld();
            const int kv0 = j * kN;
            float x[kN];
            float mx = -INFINITY;
            const bool full = kv0 + kN - 1 <= pos;  // no position of this tile is masked for this row
            if (full) {
#pragma unroll
                for (int c = 0; c < kN; ++c) {
                    x[c] = __uint_as_float(sr[c >> 5][c & 31]);
                    mx = fmaxf(mx, x[c]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < kN; ++c) {
                    x[c] = (kv0 + c <= pos) ? __uint_as_float(sr[c >> 5][c & 31]) : -INFINITY;
                    mx = fmaxf(mx, x[c]);
                }
            }
            mx *= sl2;  // -inf stays -inf (the scale is positive)
            // raise the running max only when it grows by more than the threshold
            const bool raise = fmaxf(m_run, mx) - m_run > kRescaleThreshold;  // also the first finite max
            const float mn = raise ? fmaxf(m_run, mx) : m_run;
            const float alpha = raise ? fast_exp2(m_run - mn) : 1.f;  // 0 when m_run was -inf
            m_run = mn;
            float psum = 0.f;
            if (full) {
#pragma unroll
                for (int c = 0; c < kN; ++c) {
                    x[c] = fast_exp2(fmaf(x[c], sl2, -mn));
                    psum += x[c];
                }
            } else {
#pragma unroll
                for (int c = 0; c < kN; ++c) {
                    x[c] = (x[c] == -INFINITY) ? 0.f : fast_exp2(fmaf(x[c], sl2, -mn));
                    psum += x[c];
                }
            }
            l_run = l_run * alpha + psum;
            // P as 16-bit pairs (bf16 also its low part P - bf16(P), for ~2^-17
            // relative error through a second P V pass)
            uint32_t ph_[32], pl_[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                ph_[c] = Pack16<T>::pack(x[2 * c], x[2 * c + 1]);
                if constexpr (kBf16) {
                    const float hi0 = __uint_as_float(ph_[c] << 16), hi1 = __uint_as_float(ph_[c] & 0xffff0000u);
                    pl_[c] = Pack16<T>::pack(x[2 * c] - hi0, x[2 * c + 1] - hi1);
                }
            }
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                // O is rescaled: O += P_{j-1} V_{j-1} must be done. (O += P_{j-2} V_{j-2}
                // is: S_j was issued after it, so this parity wait cannot alias.)
                const bool got = mbar_wait(o_done, (j - 1) & 1, wl) && !*(volatile int *)abort_flag;
                if (!__all_sync(0xffffffffu, got)) break;
                tc_fence_after();
#pragma unroll
                for (int ch = 0; ch < kD / 32; ++ch) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_base + kOCol + ch * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(tmem + lane_base + kOCol + ch * 32, o);
                }
            }
            tmem_st32(sbuf, ph_);  // over this row of S_j, already read
            if constexpr (kBf16) tmem_st32(sbuf + kPlOff, pl_);
            tmem_wait_st();
            // V rows past the context: zero (both halves) before P V reads them
            const int zrow = max(0, ctx - kv0);
            if (zrow < kN) {
                // V_j must have landed before its tail rows are overwritten
                if (!__all_sync(0xffffffffu, mbar_wait(v_full + b, (j >> 1) & 1, wl) && !*(volatile int *)abort_flag))
                    break;
                unsigned char *vt = Vs + b * kKVBytes;
                const int nvec = (kN - zrow) * kHalves * (kHalfBytes / 16);
                for (int i = r; i < nvec; i += kSoftmaxWarps * 32) {
                    const int row = zrow + i / (8 * kHalves);
                    const int h = (i / 8) % kHalves;
                    const int c = i & 7;
                    *reinterpret_cast<uint4 *>(vt + h * kKVHalf + row * kHalfBytes + c * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            mbar_arrive(p_full + b);
        }
        // ---- output: O / l for valid rows
        // every product done (the MMA warp's single-use end-of-kernel commit)
        const bool done = __all_sync(0xffffffffu, mbar_wait(mma_idle, 0, wl) && !*(volatile int *)abort_flag);
        tc_fence_after();
        // Each thread holds O of its row in tensor-memory lane r. For G <= 2 it
        // writes O / l in the output type into shared memory (the Q, K and V
        // tiles are dead once every product is done; the row pitch is padded by
        // 16 bytes so the 32 rows of a warp's store fall in different banks),
        // then the four softmax warps copy whole rows out, so consecutive lanes
        // store consecutive 16 bytes of one output row; rows from rows_valid on
        // belong to no query and are not written. For G >= 4 each thread stores
        // its own row directly, which measured faster there (the staged form
        // measured 2 % slower on the 4-head-group chunked-prefill workload and
        // 4 % faster on the MHA prompt workload).
        const int ebytes = p.out_dtype == PA_F32 ? 4 : 2;
        const int row_bytes = kD * ebytes;
        const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
        if constexpr (kStagedOut) {
            if (done) {
                unsigned char *srow = Qs + r * (row_bytes + 16);
#pragma unroll
                for (int ch = 0; ch < kD / 32; ++ch) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_base + kOCol + ch * 32, o);
                    tmem_wait_ld();
                    float v[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(o[e]) * inv;
                    store_row32(srow + ch * 32 * ebytes, v, p.out_dtype);
                }
            }
            // all four softmax warps arrive here whatever their outcome
            if (!softmax_sync_and(done)) {
                if (r == 0) record_error(p.err, PA_DEVERR_TIMEOUT);
            } else {
                // 16-byte pieces per row: 2^cshift (8, 16 or 32)
                const int cshift = (kD == 128 ? 4 : 3) + (ebytes == 4 ? 1 : 0);
                const int cpr = 1 << cshift;
                unsigned char *out = static_cast<unsigned char *>(p.out);
                for (int i = r; i < rows_valid * cpr; i += kSoftmaxWarps * 32) {
                    const int row = i >> cshift, c = i & (cpr - 1);
                    if ((row & (G - 1)) >= g_valid) continue;  // a padding slot
                    const size_t orow =
                        (size_t)(q0 + tok0 + (row >> gshift)) * p.num_heads + (size_t)head_base + (row & (G - 1));
                    *reinterpret_cast<uint4 *>(out + orow * row_bytes + c * 16) =
                        *reinterpret_cast<const uint4 *>(Qs + row * (row_bytes + 16) + c * 16);
                }
            }
        } else {
            if (!done) {
                if (r == 0) record_error(p.err, PA_DEVERR_TIMEOUT);
            } else {
                const size_t orow = (size_t)(q0 + tok0 + tok) * p.num_heads + (size_t)head_base + (r & (G - 1));
                unsigned char *dst = static_cast<unsigned char *>(p.out) + orow * row_bytes;
                const bool write = valid && (r & (G - 1)) < g_valid;
#pragma unroll
                for (int ch = 0; ch < kD / 32; ++ch) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_base + kOCol + ch * 32, o);
                    tmem_wait_ld();
                    if (write) {
                        float v[32];
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(o[e]) * inv;
                        store_row32(dst + ch * 32 * ebytes, v, p.out_dtype);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

}  // namespace prefill
}  // namespace pa

// ------------------------------------------------------------------ host side

namespace pa {
namespace prefill {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// A rank-2 or rank-3 tiled map over 16-bit elements, 128-byte swizzle, zero fill.
static bool make_map(CUtensorMap *map, bool bf16, void *base, int rank, const cuuint64_t *dims,
                     const cuuint64_t *strides_bytes, const cuuint32_t *box) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = f(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, rank, base, dims,
                   strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <typename T, int D, int kGS, bool kHook>
static cudaError_t launch_t(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const Params &p,
                            int q_tiles, int num_kv_heads, int num_seqs, cudaStream_t stream) {
    auto kern = prefill_kernel<T, D, kGS, kHook>;
    static AttrCache attr_done;
    constexpr int kSmem = Layout<D>::kSmemBytes;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(kern), kSmem, &attr_done);
    if (e != cudaSuccess) return e;
    kern<<<dim3(q_tiles, num_kv_heads * p.sub_groups, num_seqs), kThreads, kSmem, stream>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

}  // namespace prefill
}  // namespace pa

namespace {

// pa_prefill, with the test hook's fields of Params (hook.withhold_* -1 and
// hook.wait_limit_ns 0 for a normal call).
int prefill_call(void *out, const void *query, const int32_t *q_start, int num_tokens, int max_q_len,
                 const void *k_cache, const void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                 const int32_t *context_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                 float scale, int block_size, int num_blocks, pa_dtype kv_dtype, pa_dtype out_dtype,
                 const pa::prefill::Params &hook, cudaStream_t stream) {
    using namespace pa::prefill;
    if (num_seqs < 0 || num_tokens < 0 || max_q_len < 0 || num_heads <= 0 || num_kv_heads <= 0 ||
        num_blocks < 0 || max_blocks_per_seq < 0 || num_seqs > 65535 || num_kv_heads > 65535)
        return PA_ERR_SHAPE;
    if (kv_dtype == PA_F32) {  // fp32 caches: exact fp32 arithmetic on the CUDA cores
        if (out_dtype != PA_F32) return PA_ERR_DTYPE;
        return pa::prefill_cuda_cores(out, query, q_start, num_tokens, k_cache, v_cache, block_tables,
                                      max_blocks_per_seq, context_lens, num_seqs, num_heads, num_kv_heads, head_dim,
                                      scale, block_size, num_blocks, stream);
    }
    if (kv_dtype != PA_F16 && kv_dtype != PA_BF16) return PA_ERR_DTYPE;
    if (out_dtype != kv_dtype && out_dtype != PA_F32) return PA_ERR_DTYPE;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_HEAD_DIM;
    if (block_size != 16 && block_size != 32) return PA_ERR_BLOCK_SIZE;
    if (num_heads % num_kv_heads != 0) return PA_ERR_HEADS;
    const int group = num_heads / num_kv_heads;
    int gshift = 0;  // head slots per token: the group rounded up to a power of two, at most 128
    while ((1 << gshift) < group && gshift < 7) ++gshift;
    const int gslots = 1 << gshift;
    const int sub_groups = (group + gslots - 1) / gslots;
    if ((long long)num_kv_heads * sub_groups > 65535) return PA_ERR_SHAPE;
    if (num_seqs == 0 || num_tokens == 0 || max_q_len == 0) return PA_OK;
    if (!out || !query || !q_start || !k_cache || !v_cache || !block_tables || !context_lens) return PA_ERR_NULL;
    auto al = [](const void *ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) == 0; };
    if (!al(out, 16) || !al(query, 16) || !al(k_cache, 16) || !al(v_cache, 16) || !al(q_start, 4) ||
        !al(block_tables, 4) || !al(context_lens, 4))
        return PA_ERR_ALIGN;
    const long long kv_rows = (long long)num_blocks * num_kv_heads * block_size;
    if (kv_rows >= INT32_MAX || (long long)num_tokens * num_heads >= INT32_MAX) return PA_ERR_SHAPE;
    if ((long long)max_q_len * gslots >= INT32_MAX) return PA_ERR_SHAPE;
    const bool bf16 = kv_dtype == PA_BF16;
    CUtensorMap mq, mk, mv;
    {
        const cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_heads, (cuuint64_t)num_tokens};
        const cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, (cuuint64_t)num_heads * head_dim * 2};
        const cuuint32_t box[3] = {64, (cuuint32_t)gslots, (cuuint32_t)(kM / gslots)};
        if (!make_map(&mq, bf16, const_cast<void *>(query), 3, dims, strides, box)) return PA_ERR_CUDA;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)(kv_rows > 0 ? kv_rows : 1)};
        const cuuint64_t strides[1] = {(cuuint64_t)head_dim * 2};
        const cuuint32_t box[2] = {64, 16};
        if (!make_map(&mk, bf16, const_cast<void *>(k_cache), 2, dims, strides, box)) return PA_ERR_CUDA;
        if (!make_map(&mv, bf16, const_cast<void *>(v_cache), 2, dims, strides, box)) return PA_ERR_CUDA;
    }
    unsigned int *err = nullptr;
    if (pa::device_error_word(&err) != cudaSuccess) return PA_ERR_CUDA;
    Params p = hook;
    p.out = out;
    p.q_start = q_start;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.num_blocks = num_blocks;
    p.block_size = block_size;
    p.kv_rows = kv_rows;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.out_dtype = out_dtype;
    p.err = err;
    p.group = group;
    p.gshift = gshift;
    p.sub_groups = sub_groups;
    const int q_tiles = (max_q_len * gslots + kM - 1) / kM;
    cudaError_t e = cudaErrorInvalidValue;
    // the test hook's instances (head_dim 128 only) are separate, so the
    // production instances carry none of it
    const bool with_hook = p.withhold_seq >= 0;
#define PA_PREFILL_GS(T, DD, GS, H) launch_t<T, DD, GS, H>(mq, mk, mv, p, q_tiles, num_kv_heads, num_seqs, stream)
#define PA_PREFILL_CASE(T, DD, H)                                                               \
    e = group == 1 ? PA_PREFILL_GS(T, DD, 0, H) : group == 2 ? PA_PREFILL_GS(T, DD, 1, H)       \
      : group == 4 ? PA_PREFILL_GS(T, DD, 2, H) : group == 8 ? PA_PREFILL_GS(T, DD, 3, H)       \
                   : PA_PREFILL_GS(T, DD, -1, H)
    if (bf16) {
        if (head_dim == 128) {
            if (with_hook) PA_PREFILL_CASE(__nv_bfloat16, 128, true);
            else PA_PREFILL_CASE(__nv_bfloat16, 128, false);
        } else {
            PA_PREFILL_CASE(__nv_bfloat16, 64, false);
        }
    } else {
        if (head_dim == 128) {
            if (with_hook) PA_PREFILL_CASE(__half, 128, true);
            else PA_PREFILL_CASE(__half, 128, false);
        } else {
            PA_PREFILL_CASE(__half, 64, false);
        }
    }
#undef PA_PREFILL_CASE
#undef PA_PREFILL_GS
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace

extern "C" int pa_prefill(void *out, const void *query, const int32_t *q_start, int num_tokens,
                          int max_q_len, const void *k_cache, const void *v_cache,
                          const int32_t *block_tables, int max_blocks_per_seq,
                          const int32_t *context_lens, int num_seqs, int num_heads, int num_kv_heads,
                          int head_dim, float scale, int block_size, int num_blocks, pa_dtype kv_dtype,
                          pa_dtype out_dtype, cudaStream_t stream) {
    const pa::prefill::Params hook{};
    return prefill_call(out, query, q_start, num_tokens, max_q_len, k_cache, v_cache, block_tables,
                        max_blocks_per_seq, context_lens, num_seqs, num_heads, num_kv_heads, head_dim, scale,
                        block_size, num_blocks, kv_dtype, out_dtype, hook, stream);
}

extern "C" int pa_prefill_withhold_tile(void *out, const void *query, const int32_t *q_start, int num_tokens,
                                        int max_q_len, const void *k_cache, const void *v_cache,
                                        const int32_t *block_tables, int max_blocks_per_seq,
                                        const int32_t *context_lens, int num_seqs, int num_heads,
                                        int num_kv_heads, int head_dim, float scale, int block_size,
                                        int num_blocks, pa_dtype kv_dtype, pa_dtype out_dtype, int seq,
                                        int kv_head, int query_tile, int tile, unsigned long long wait_limit_ns,
                                        cudaStream_t stream) {
    if (kv_dtype != PA_F16 && kv_dtype != PA_BF16) return PA_ERR_DTYPE;  // the tensor-core kernel only
    if (head_dim != 128) return PA_ERR_HEAD_DIM;                          // its hook instances
    if (seq < 0 || seq >= num_seqs || kv_head < 0 || kv_head >= num_kv_heads || query_tile < 0 || tile < 0 ||
        wait_limit_ns < 100000ull || wait_limit_ns > 1000000000ull)
        return PA_ERR_SHAPE;
    pa::prefill::Params hook{};
    hook.withhold_seq = seq;
    hook.withhold_kvh = kv_head;
    hook.withhold_qt = query_tile;
    hook.withhold_tile = tile;
    hook.wait_limit_ns = wait_limit_ns;
    return prefill_call(out, query, q_start, num_tokens, max_q_len, k_cache, v_cache, block_tables,
                        max_blocks_per_seq, context_lens, num_seqs, num_heads, num_kv_heads, head_dim, scale,
                        block_size, num_blocks, kv_dtype, out_dtype, hook, stream);
}
