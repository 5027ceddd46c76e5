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
//   * one CTA of four warps per (sequence, kv head[, partition]); all G query
//     heads of the GQA group share every K/V tile, so each tile crosses HBM
//     once;
//   * the token range is cut into 16-token stages; stage k belongs to warp
//     k % 4 and lives in shared-memory buffer k % R, the ring of R = 8
//     buffers (two per warp).
//     The warp loads its own stages: lane 0 streams the stage's K and V tile
//     (16 contiguous token rows of one kv head in this layout) with two
//     one-dimensional bulk copies (cp.async.bulk, TMA engine) completing on
//     the buffer's mbarrier, and right after consuming stage k it reloads the
//     same buffer with stage k + R. No other warp touches the buffer, so
//     there are no empty barriers and a parity wait can never alias. Table
//     entries are read 32 stages ahead, one per lane;
//   * 16-bit GQA groups (G >= 2) compute QK^T and PV with tensor-core MMAs
//     (mma.sync m16n8k16, the group's query heads padded to 16 rows); MHA
//     and fp32 use CUDA cores, where each lane holds one 16-byte column
//     vector of a token row and a transposing butterfly reduces the partial
//     dot products across the row's lanes (each step halves what a lane
//     holds, so a lane ends with whole scores and runs one exp per score);
//   * running max / sum / accumulator in fp32 (log2 domain), per row group;
//     the CTA merges its row groups at the end by the same log-sum-exp rule
//     as the split-K reduce;
//   * every wait is bounded (PA_DEVERR_TIMEOUT), bad table entries skip their
//     stage (PA_DEVERR_BLOCK_ID).
#include <math.h>

#include <type_traits>

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
    // 16-bit GQA groups and every int8 cache run QK^T and PV on the tensor
    // cores; 16-bit MHA and fp32 on the CUDA cores.
    static constexpr bool kInt8 = (kElt == 1);
    static constexpr bool kUseMma = kInt8 || ((kElt == 2) && (G >= 2));
    static constexpr int kWarps = 4;
    static constexpr int kThreads = kWarps * 32;
    static constexpr int kTileBytes = kTS * D * kElt;  // 16 token rows of one kv head, K or V
    static constexpr int kScaleBytes = kInt8 ? kTS * 4 : 0;  // int8: the 16 rows' fp32 scales, K or V
    // The tensor-core consumers (int8 with 128-byte rows, 16-bit head groups
    // of two or more): V tiles come by 2-D TMA in the 128-byte swizzled
    // layout, as kVBoxes boxes of 16 rows x 128 bytes, in their own
    // 1024-byte-aligned region; each stage buffer then holds K (and the
    // scales) only. The V fragment loads read four rows per quarter-warp, a
    // 4-way bank conflict in the plain layout and none in the swizzled one.
    static constexpr bool kVSwizzle = (kInt8 && D == 128) || (kUseMma && kElt == 2);
    static constexpr int kVBoxes = kInt8 ? 1 : D * kElt / 128;
    // 16-bit tensor-core consumer: K comes the same way, into the stage
    // buffer (1024-byte aligned there), and its lanes take the chunks of a
    // row in an order that keeps a quarter-warp's two rows on different banks
    static constexpr bool kKSwizzle = kUseMma && kElt == 2;
    static constexpr int kStageBytes = (kVSwizzle ? 1 : 2) * kTileBytes + 2 * kScaleBytes;
    static constexpr int kScaleOff = (kVSwizzle ? 1 : 2) * kTileBytes;  // scales within a stage buffer
    // Buffers per warp (a ring of kWarps * kBufPerWarp stages). int8 stages
    // are half the bytes; measured, a deeper int8 ring did not help, five
    // CTAs per SM did.
    static constexpr int kBufPerWarp = 2;
    static constexpr int kStages = kWarps * kBufPerWarp;
    static constexpr int kRowGroups = kUseMma ? kWarps : kWarps * kRows;
    static constexpr int kVRegion = kVSwizzle ? kStages * kTileBytes : 0;
    static constexpr int kRingBytes = kVRegion + kStages * kStageBytes;
    static constexpr int kAlign = kVSwizzle ? 1024 : 128;  // ring base alignment
    static constexpr int kAgStride = kUseMma ? D + 1 : D;  // floats per merged accumulator row
    static constexpr int kMergeBytes = kRowGroups * G * (kAgStride + 2) * 4;
    static constexpr int kDataBytes = kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes;
    // int8 groups of more than four heads keep the query's fixed-point MMA
    // fragments (2 D/64 16-byte words per lane) in shared memory and read
    // them once per stage: every O column is live there, and the registers
    // this frees let five CTAs share an SM without spilling.
    static constexpr bool kQShared = kInt8 && G > 4;
    static constexpr int kQBytes = kQShared ? 2 * (D / 64) * 32 * 16 : 0;
    // ring (or merge area), full barriers, per-buffer "skipped" flags, the
    // test hook and head range (32 bytes) and the shared query fragments
    static constexpr int kSmemBytes = kAlign + kDataBytes + kStages * 8 + kStages * 4 + 32 + kQBytes;
    // Resident CTAs per SM the register budget is set for (a sub-partition
    // holds one warp of each CTA, so 3 CTAs leave 170 registers a thread).
    static constexpr int kMinBlocks = kInt8 ? 5 : ((kUseMma || G <= 4) ? 3 : 2);

    static_assert(kStages == kBufPerWarp * kWarps, "stage k: warp k % 4, buffer k % kStages");
    static_assert(BS % kTS == 0, "block size is a multiple of the stage");
    // the CUDA-core consumer's lane layout
    static_assert(kUseMma || (kLpt >= 1 && kLpt <= 32 && (32 % kLpt) == 0), "row width");
    static_assert(kUseMma || (kTS % kRows == 0 && kTpg % kTc == 0), "stage split");
    static_assert(kUseMma || G <= kLpt, "a lane's kept scores must belong to one query head");
    static_assert(kUseMma || kNvl <= kTc, "kept scores within one head");
    static_assert(kDataBytes % 16 == 0, "barriers, flags, hook and query fragments stay 16-byte aligned");
    static_assert(!kKSwizzle || (kVRegion % 1024 == 0 && kStageBytes % 1024 == 0), "swizzled K boxes 1024-byte aligned");
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

// ------------------------------------------------------- CUDA-core consumer

// One warp's share of the CTA on the CUDA cores. Lane = r * kLpt + c: row r of
// a warp instruction (token), 16-byte column c of that row.
template <typename T, int D, int G, typename S>
struct FmaConsumer {
    int r, c, rg, g_lane, v0;
    bool counts_l;
    float q[G][S::kVec];
    float m_run[G];
    float acc[G][S::kVec];
    float l_lane;

    __device__ __forceinline__ void init(const DecodeParams &p, size_t head0, int g_valid, int warp, int lane) {
        r = lane / S::kLpt;
        c = lane % S::kLpt;
        rg = warp * S::kRows + r;
        g_lane = c / S::kLanesPerG;     // query head of this lane's kept scores
        v0 = (c * S::kNv) / S::kLpt;    // index of this lane's first kept score
        counts_l = (c % S::kDup) == 0;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            uint4 u = make_uint4(0u, 0u, 0u, 0u);  // padding heads: zero queries
            if (g < g_valid)
                u = *reinterpret_cast<const uint4 *>(static_cast<const T *>(p.query) + (head0 + g) * D + c * S::kVec);
            Elt<T>::unpack(u, q[g]);
#pragma unroll
            for (int e = 0; e < S::kVec; ++e) q[g][e] *= p.scale_log2;
            m_run[g] = -INFINITY;
#pragma unroll
            for (int e = 0; e < S::kVec; ++e) acc[g][e] = 0.f;
        }
        l_lane = 0.f;
    }

    __device__ __forceinline__ void stage(const unsigned char *Ks, const unsigned char *Vs, int nvalid,
                                          int lane, float) {
#pragma unroll
        for (int ci = 0; ci < S::kChunks; ++ci) {
            // ---- scores: partial dots over this lane's columns
            float sc[S::kNv];
#pragma unroll
            for (int i = 0; i < S::kTc; ++i) {
                const int t = (ci * S::kTc + i) * S::kRows + r;
                const uint4 u = *reinterpret_cast<const uint4 *>(Ks + ((size_t)t * D + c * S::kVec) * S::kElt);
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
                const float cm =
                    (G == 1) ? cmax : __shfl_sync(0xffffffffu, cmax, r * S::kLpt + g * S::kLanesPerG);
                const float mn = fmaxf(m_run[g], cm);
                const float alpha = (mn == -INFINITY) ? 1.f : fast_exp2(m_run[g] - mn);
                m_run[g] = mn;
#pragma unroll
                for (int e = 0; e < S::kVec; ++e) acc[g][e] *= alpha;
                if (g == g_lane) {
                    my_m = mn;
                    my_alpha = alpha;
                }
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
                const uint4 u = *reinterpret_cast<const uint4 *>(Vs + ((size_t)t * D + c * S::kVec) * S::kElt);
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

    // After the ring is drained: this row group's (m, l, acc) to shared memory.
    __device__ __forceinline__ void store(float *mg, float *lg, float *ag, int, int) {
#pragma unroll
        for (int mk = 1; mk < S::kLanesPerG; mk <<= 1) l_lane += __shfl_xor_sync(0xffffffffu, l_lane, mk);
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
            float4 *dst = reinterpret_cast<float4 *>(ag + ((size_t)rg * G + g) * S::kAgStride + c * S::kVec);
#pragma unroll
            for (int e = 0; e < S::kVec; e += 4)
                dst[e / 4] = make_float4(acc[g][e], acc[g][e + 1], acc[g][e + 2], acc[g][e + 3]);
        }
    }
};

// ------------------------------------------------------ tensor-core consumer

// m16n8k16 MMA, fp32 accumulation, for one 16-bit type.
template <typename T> struct Mma;

template <> struct Mma<__nv_bfloat16> {
    // bf16 keeps 8 mantissa bits: a probability rounded once would cost about
    // 1e-3 relative error, so P goes in as hi + lo (two MMAs, ~2^-17).
    static constexpr bool kSplitP = true;
    static __device__ __forceinline__ void mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
            "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&v);
    }
    static __device__ __forceinline__ float2 unpack(uint32_t u) {
        return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
    }
};

template <> struct Mma<__half> {
    // fp16 keeps 11 bits: one rounding of P is ~3e-4 relative, inside the bound.
    static constexpr bool kSplitP = false;
    static __device__ __forceinline__ void mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
            "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&v);
    }
    static __device__ __forceinline__ float2 unpack(uint32_t u) {
        return __half22float2(*reinterpret_cast<__half2 *>(&u));
    }
};

// Transpose of an 8x8 matrix of 16-bit pairs held one row pair per lane
// (lane 4 r + q holds row r, columns 2q, 2q + 1).
__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
    uint32_t y;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
    Mma<__half>::mma(c, a0, a1, a2, a3, b0, b1);
}

// One warp's share on the tensor cores, in transposed form so that the
// 16-row M side of the MMA is filled by tokens and head dims instead of the
// group's 2-8 query heads. Per 16-token stage, with lane = 4 r + q:
//   S^T = K Q^T: M = the stage's 16 tokens, N = 8 query-head columns (the
//     group, zero-padded), K = head_dim. The k -> d map of each k-step is
//     chosen so that one 16-byte shared load of a K row (chunk kchunk(i),
//     d = 8 kchunk(i) .. +8) feeds two k-steps; Q's B fragment, loaded once,
//     uses the same map.
//     Lane holds S^T[t][n] for t in {r, r + 8}, columns n in {2q, 2q + 1};
//     column n is head n, or for groups of at most four heads head n / 2 on
//     even n and padding on odd n (one head per lane, kSpread).
//   O^T += V^T P^T: M = 16 head dims per tile, N = 8 query-head columns,
//     K = 16 tokens. P^T's B fragment is the S^T accumulator, packed to 16
//     bits and transposed in registers (movmatrix). V^T's A fragment is built
//     with byte permutes from 16-byte loads of V rows (no transposing load;
//     the K and V tiles are in the 128-byte swizzled layout, so the rows a
//     quarter-warp reads fall in different banks): tile mt row m holds
//     d = 8 (m % 8) + E % 8 + 64 (E / 8) with E = mt for m < 8 and
//     E = mt + D/16 for m >= 8.
// Running max / sum per (query head, warp); tokens past the context are
// masked to -inf and their V rows zeroed (they may hold NaN).
template <typename T, int D, int G, typename S>
struct MmaConsumer {
    using M = Mma<T>;
    static constexpr int kI = D / 32;    // 16-byte chunks of a K row per lane (2 k-steps each)
    static constexpr int kMT = D / 16;   // PV m-tiles
    static constexpr int kCh = D / 64;   // 16-byte V chunks per token row per lane
    // groups of at most four heads: head g in column 2g, one head per lane
    // (see MmaConsumerQ8)
    static constexpr bool kSpread = G <= 4;
    static constexpr int kH = kSpread ? 1 : 2;  // live columns (heads) per lane
    int q4, r;
    uint32_t qb[kI][4];
    float o[kMT][4];
    float m_run[2], l_lane[2];

    // 16-byte chunk (of a K or Q row) a lane of quarter q takes in QK step i
    __device__ __forceinline__ int kchunk(int i) const { return 2 * q4 + (i & 1) + 8 * (i >> 1); }

    static __device__ __forceinline__ int dim_of(int m, int mt) {  // head dim of m-tile mt, row m
        const int E = m < 8 ? mt : mt + kMT;
        return 8 * (m & 7) + (E & 7) + 64 * (E >> 3);
    }

    __device__ __forceinline__ void init(const DecodeParams &p, size_t head0, int g_valid, int, int lane) {
        q4 = lane & 3;
        r = lane >> 2;
        const int hq = kSpread ? r >> 1 : r;  // the head of this lane's B column r
        const bool live = (!kSpread || (r & 1) == 0) && hq < g_valid;
#pragma unroll
        for (int i = 0; i < kI; ++i) {
            uint4 u = make_uint4(0u, 0u, 0u, 0u);
            if (live)  // the 16-byte chunk K's lanes take in step i (see stage())
                u = *reinterpret_cast<const uint4 *>(static_cast<const T *>(p.query) + (head0 + hq) * D +
                                                     8 * kchunk(i));
            qb[i][0] = u.x;
            qb[i][1] = u.y;
            qb[i][2] = u.z;
            qb[i][3] = u.w;
        }
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
        m_run[0] = m_run[1] = -INFINITY;
        l_lane[0] = l_lane[1] = 0.f;
    }

    __device__ __forceinline__ void stage(const unsigned char *Kb, const unsigned char *Vb, int nvalid, int,
                                          float scale_log2) {
        const T *Vs = reinterpret_cast<const T *>(Vb);
        // ---- S^T = K Q^T. The K tile is in the 128-byte swizzled layout
        // (boxes of 64 dims x 16 rows, chunk c of row t at c ^ t % 8); in step
        // i a lane takes 16-byte chunk kchunk(i) of rows r and r + 8, so the
        // quarter-warp's rows r = 0, 1 read the even and the odd chunks.
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < kI; ++i) {
            const int c = kchunk(i);
            const unsigned char *kbox = Kb + (c >> 3) * 2048;
            const uint4 u0 = *reinterpret_cast<const uint4 *>(kbox + r * 128 + (((c & 7) ^ (r & 7)) << 4));
            const uint4 u1 = *reinterpret_cast<const uint4 *>(kbox + (r + 8) * 128 + (((c & 7) ^ (r & 7)) << 4));
            M::mma(sc, u0.x, u1.x, u0.y, u1.y, qb[i][0], qb[i][1]);
            M::mma(sc, u0.z, u1.z, u0.w, u1.w, qb[i][2], qb[i][3]);
        }
        // ---- online softmax per column n = 2q + h (h = 0, 1) over tokens r, r + 8
        const bool v0 = r < nvalid;
        const bool v1 = r + 8 < nvalid;
        float x[4];
        x[0] = v0 ? sc[0] * scale_log2 : -INFINITY;  // t = r,     n = 2q
        x[1] = (v0 && !kSpread) ? sc[1] * scale_log2 : -INFINITY;  // t = r,     n = 2q + 1
        x[2] = v1 ? sc[2] * scale_log2 : -INFINITY;  // t = r + 8, n = 2q
        x[3] = (v1 && !kSpread) ? sc[3] * scale_log2 : -INFINITY;  // t = r + 8, n = 2q + 1
        float mx0 = fmaxf(x[0], x[2]);
#pragma unroll
        for (int mk = 4; mk < 32; mk <<= 1) mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, mk));
        const float mn0 = fmaxf(m_run[0], mx0);
        const float al0 = (mn0 == -INFINITY) ? 1.f : fast_exp2(m_run[0] - mn0);
        m_run[0] = mn0;
        float pr[4];
        pr[0] = (x[0] == -INFINITY) ? 0.f : fast_exp2(x[0] - mn0);
        pr[2] = (x[2] == -INFINITY) ? 0.f : fast_exp2(x[2] - mn0);
        l_lane[0] = l_lane[0] * al0 + pr[0] + pr[2];
        pr[1] = pr[3] = 0.f;
        float al1 = 1.f;
        if constexpr (!kSpread) {
            float mx1 = fmaxf(x[1], x[3]);
#pragma unroll
            for (int mk = 4; mk < 32; mk <<= 1) mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, mk));
            const float mn1 = fmaxf(m_run[1], mx1);
            al1 = (mn1 == -INFINITY) ? 1.f : fast_exp2(m_run[1] - mn1);
            m_run[1] = mn1;
            pr[1] = (x[1] == -INFINITY) ? 0.f : fast_exp2(x[1] - mn1);
            pr[3] = (x[3] == -INFINITY) ? 0.f : fast_exp2(x[3] - mn1);
            l_lane[1] = l_lane[1] * al1 + pr[1] + pr[3];
        }
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt) {
            o[mt][0] *= al0;
            o[mt][2] *= al0;
            if constexpr (!kSpread) {  // else the odd (padding) columns stay 0 and are never stored
                o[mt][1] *= al1;
                o[mt][3] *= al1;
            }
        }
        // ---- P^T fragments -> PV's B fragments (tokens 0-7 and 8-15)
        const uint32_t h01 = M::pack(pr[0], pr[1]);
        const uint32_t h23 = M::pack(pr[2], pr[3]);
        const uint32_t bh0 = transpose8x8(h01);
        const uint32_t bh1 = transpose8x8(h23);
        uint32_t bl0 = 0u, bl1 = 0u;
        if constexpr (M::kSplitP) {
            const float2 f01 = M::unpack(h01);
            const float2 f23 = M::unpack(h23);
            bl0 = transpose8x8(M::pack(pr[0] - f01.x, pr[1] - f01.y));
            bl1 = transpose8x8(M::pack(pr[2] - f23.x, pr[3] - f23.y));
        }
        // ---- O^T += V^T P^T
        uint32_t a_lo[kMT][4];  // V^T A fragments of this stage
#pragma unroll
        for (int ch = 0; ch < kCh; ++ch) {
            uint4 va, vb, vc, vd;
            if constexpr (S::kVSwizzle) {
                // box ch (dims 64 ch ..): row t at 128 t, its 16-byte chunk c at (c ^ t % 8) * 16
                const unsigned char *vbox = Vb + ch * 2048;
                auto row = [&](int t) {
                    return *reinterpret_cast<const uint4 *>(vbox + t * 128 + ((r ^ (t & 7)) << 4));
                };
                va = row(2 * q4);
                vb = row(2 * q4 + 1);
                vc = row(2 * q4 + 8);
                vd = row(2 * q4 + 9);
            } else {
                const T *vcol = Vs + 64 * ch + 8 * r;
                va = *reinterpret_cast<const uint4 *>(vcol + (2 * q4) * D);
                vb = *reinterpret_cast<const uint4 *>(vcol + (2 * q4 + 1) * D);
                vc = *reinterpret_cast<const uint4 *>(vcol + (2 * q4 + 8) * D);
                vd = *reinterpret_cast<const uint4 *>(vcol + (2 * q4 + 9) * D);
            }
            if (nvalid < S::kTS) {  // rows past the context may hold anything
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                if (2 * q4 >= nvalid) va = z;
                if (2 * q4 + 1 >= nvalid) vb = z;
                if (2 * q4 + 8 >= nvalid) vc = z;
                if (2 * q4 + 9 >= nvalid) vd = z;
            }
            // element e of chunk ch is E = 8 ch + e: tile E (rows < 8) or tile E - kMT (rows >= 8)
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int E = 8 * ch + e;
                const unsigned sel = (e & 1) ? 0x7632u : 0x5410u;
                const uint32_t lo_t = __byte_perm(word_of(va, e >> 1), word_of(vb, e >> 1), sel);  // t = 2q, 2q+1
                const uint32_t hi_t = __byte_perm(word_of(vc, e >> 1), word_of(vd, e >> 1), sel);  // t = 2q+8, 2q+9
                if (E < kMT) {
                    a_lo[E][0] = lo_t;
                    a_lo[E][2] = hi_t;
                } else {
                    a_lo[E - kMT][1] = lo_t;
                    a_lo[E - kMT][3] = hi_t;
                }
            }
        }
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt) {
            M::mma(o[mt], a_lo[mt][0], a_lo[mt][1], a_lo[mt][2], a_lo[mt][3], bh0, bh1);
            if constexpr (M::kSplitP) M::mma(o[mt], a_lo[mt][0], a_lo[mt][1], a_lo[mt][2], a_lo[mt][3], bl0, bl1);
        }
    }
    // After the ring is drained: this warp's (m, l, O) to shared memory.
    // Row stride D + 1 keeps the scattered stores off a single bank.
    __device__ __forceinline__ void store(float *mg, float *lg, float *ag, int warp, int) {
#pragma unroll
        for (int h = 0; h < kH; ++h) {
#pragma unroll
            for (int mk = 4; mk < 32; mk <<= 1) l_lane[h] += __shfl_xor_sync(0xffffffffu, l_lane[h], mk);
        }
#pragma unroll
        for (int h = 0; h < kH; ++h) {
            const int g = kSpread ? q4 : 2 * q4 + h;  // the head of column 2 q4 + h
            if (g < G) {
                if (r == 0) {
                    mg[warp * G + g] = m_run[h];
                    lg[warp * G + g] = l_lane[h];
                }
                float *row = ag + ((size_t)warp * G + g) * S::kAgStride;
#pragma unroll
                for (int mt = 0; mt < kMT; ++mt) {
                    row[dim_of(r, mt)] = o[mt][h];
                    row[dim_of(r + 8, mt)] = o[mt][2 + h];
                }
            }
        }
    }
};

// ------------------------------------------------- int8 tensor-core consumer

// int8 codes -> exact fp16: x + 128 as an unsigned byte becomes the mantissa
// of 1024 + (x + 128) (fp16 0x64xx), then 1152 is subtracted (0x6480).
__device__ __forceinline__ uint32_t i8pair_to_h2(uint32_t biased, unsigned sel) {
    const uint32_t m = __byte_perm(biased, 0x64646464u, sel);
    __half2 h = *reinterpret_cast<const __half2 *>(&m);
    const uint32_t k1152 = 0x64806480u;
    h = __hsub2(h, *reinterpret_cast<const __half2 *>(&k1152));
    return *reinterpret_cast<uint32_t *>(&h);
}

// As MmaConsumer, for int8 caches with per-row scales. Per 16-token stage,
// lane = 4 r + q:
//   S^T = Kq Q^T on the int8 tensor cores (mma.sync m16n8k32, int32
//     accumulation): the query of each head is held as 16-bit fixed point
//     (step = its largest |q_d| / 32767, split into a signed high byte and an
//     unsigned low byte: two exact integer products); lane loads 16-byte
//     chunks q + 4 j of token rows r and r + 8 and feeds their words to the
//     MMAs' A fragments directly (no conversion). The score of token t is the
//     integer product times the step and its K row scale.
//   O^T += Vq^T P'^T with P'_t = p_t * sv_t / svmax (sv_t the V row scale,
//     svmax the stage's largest), so P' is in [0, 1] in fp16; the stage's
//     product is added to O times svmax (fp32). Lane loads W = D/8 dims
//     (W r .. W r + W - 1) of token rows 2q, 2q+1, 2q+8, 2q+9; byte permutes
//     pair two tokens' codes of one dim before the fp16 conversion. m-tile
//     mt row m holds dim W (m % 8) + mt + (m >= 8 ? W/2 : 0).
// Tokens past the context have p = 0 and P' = 0 (their scales may hold
// anything; int8 codes are always finite).
// Groups of at most four heads put head g in column 2g (kSpread): every
// lane's even column is a head (lane q: head q) and its odd column padding,
// so a lane runs the softmax, the rescale and the O update of one head
// instead of two, for four heads as for one.
template <typename TQ, int D, int G, typename S>
struct MmaConsumerQ8 {
    static constexpr int kJ = D / 64;    // 16-byte K chunks per lane per row
    static constexpr int kMT = D / 16;   // PV m-tiles
    static constexpr int kW = D / 8;     // V dims per lane
    static constexpr bool kQShared = S::kQShared;
    static constexpr bool kSpread = G <= 4;
    static constexpr int kH = kSpread ? 1 : 2;  // live columns (heads) per lane
    int q4, r;
    // query as 16-bit fixed point: signed high bytes, unsigned low bytes; in
    // registers (kQShared false) or as words [2 j + 0/1][lane] of qsm
    uint32_t qhi[kQShared ? 1 : kJ][4], qlo[kQShared ? 1 : kJ][4];
    const uint4 *qsm;                    // this lane's word 0 of the shared fragments
    float qs[2];                         // fixed-point step of columns 2q, 2q + 1
    float o[kMT][4];
    float m_run[2], l_lane[2];

    static __device__ __forceinline__ int dim_of(int m, int mt) {
        return kW * (m & 7) + mt + (m >= 8 ? kW / 2 : 0);
    }

    // mma.sync m16n8k32, int8 x int8 -> int32 (B signed or unsigned)
    static __device__ __forceinline__ void mma_s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                  uint32_t b0, uint32_t b1) {
        asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
    static __device__ __forceinline__ void mma_u8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                  uint32_t b0, uint32_t b1) {
        asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }

    // The query of head r (this lane's B column) as Q = rint(q / step) with
    // step = max_d |q_d| / 32767 (|Q| <= 32767), split Q = 256 hi + lo (hi
    // signed, lo in [0, 255]): q . k = step (256 hi.k + lo.k), both products
    // exact in int32 on the int8 tensor cores. |q - step Q| <= step / 2, i.e.
    // 2^-16 of the head's largest component.
    // qarea: the CTA's shared query fragments (kQShared), written by warp 0;
    // every thread of the CTA calls init.
    __device__ __forceinline__ void init(const DecodeParams &p, size_t head0, int g_valid, int warp, int lane,
                                         uint4 *qarea) {
        q4 = lane & 3;
        r = lane >> 2;
        float f[kJ][16];
        float amax = 0.f;
        // this lane's B column r holds head hq (kSpread: even columns only)
        const int hq = kSpread ? r >> 1 : r;
        const bool live = (!kSpread || (r & 1) == 0) && hq < g_valid;
#pragma unroll
        for (int j = 0; j < kJ; ++j) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint4 u = make_uint4(0u, 0u, 0u, 0u);
                if (live)
                    u = *reinterpret_cast<const uint4 *>(static_cast<const TQ *>(p.query) + (head0 + hq) * D +
                                                         16 * (q4 + 4 * j) + 8 * h);
                Elt<TQ>::unpack(u, f[j] + 8 * h);
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(f[j][e]));
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const float inv = amax > 0.f ? __fdiv_rn(32767.f, amax) : 0.f;
        const float step = amax > 0.f ? __fdiv_rn(amax, 32767.f) : 0.f;
#pragma unroll
        for (int j = 0; j < kJ; ++j) {
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) {  // word w: dims 4w .. 4w + 3 of the chunk
                uint32_t hi = 0, lo = 0;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int Q = max(-32767, min(32767, __float2int_rn(f[j][4 * w + e] * inv)));
                    hi |= (uint32_t)((Q >> 8) & 0xff) << (8 * e);
                    lo |= (uint32_t)(Q & 0xff) << (8 * e);
                }
                hw[w] = hi;
                lw[w] = lo;
            }
            if constexpr (kQShared) {
                if (warp == 0) {
                    qarea[(2 * j) * 32 + lane] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    qarea[(2 * j + 1) * 32 + lane] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                }
            } else {
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    qhi[j][w] = hw[w];
                    qlo[j][w] = lw[w];
                }
            }
        }
        qsm = qarea + lane;
        if constexpr (kQShared) __syncthreads();
        qs[0] = __shfl_sync(0xffffffffu, step, (2 * q4) * 4);
        qs[1] = __shfl_sync(0xffffffffu, step, (2 * q4 + 1) * 4);
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
        m_run[0] = m_run[1] = -INFINITY;
        l_lane[0] = l_lane[1] = 0.f;
    }

    __device__ __forceinline__ void stage(const unsigned char *Kb, const unsigned char *Vb, int nvalid, int,
                                          float scale_log2) {
        const float *ksc = reinterpret_cast<const float *>(Kb + S::kScaleOff);
        const float *vsc = ksc + S::kTS;
        // ---- S^T = Kq Q^T on the int8 tensor cores: MMA (j, m) takes dims
        // 16 (q + 4 j) + 8 m + 0..3 as k columns 4q..4q+3 and + 4..7 as 16 + 4q..
        int chi[4] = {0, 0, 0, 0}, clo[4] = {0, 0, 0, 0};
#pragma unroll
        for (int j = 0; j < kJ; ++j) {
            const uint4 u0 = *reinterpret_cast<const uint4 *>(Kb + r * D + 16 * (q4 + 4 * j));
            const uint4 u1 = *reinterpret_cast<const uint4 *>(Kb + (r + 8) * D + 16 * (q4 + 4 * j));
            uint32_t bh[4], bl[4];
            if constexpr (kQShared) {
                const uint4 h = qsm[(2 * j) * 32], l = qsm[(2 * j + 1) * 32];
                bh[0] = h.x; bh[1] = h.y; bh[2] = h.z; bh[3] = h.w;
                bl[0] = l.x; bl[1] = l.y; bl[2] = l.z; bl[3] = l.w;
            } else {
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    bh[w] = qhi[j][w];
                    bl[w] = qlo[j][w];
                }
            }
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const uint32_t a0 = word_of(u0, 2 * m), a2 = word_of(u0, 2 * m + 1);
                const uint32_t a1 = word_of(u1, 2 * m), a3 = word_of(u1, 2 * m + 1);
                mma_s8(chi, a0, a1, a2, a3, bh[2 * m], bh[2 * m + 1]);
                mma_u8(clo, a0, a1, a2, a3, bl[2 * m], bl[2 * m + 1]);
            }
        }
        float sc[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) sc[i] = (float)((chi[i] << 8) + clo[i]) * qs[i & 1];
        // ---- online softmax per column n = 2q + h over tokens r, r + 8
        const bool v0 = r < nvalid;
        const bool v1 = r + 8 < nvalid;
        const float s0 = v0 ? ksc[r] * scale_log2 : 0.f;
        const float s1 = v1 ? ksc[r + 8] * scale_log2 : 0.f;
        float x[4];
        x[0] = v0 ? sc[0] * s0 : -INFINITY;
        x[1] = (v0 && !kSpread) ? sc[1] * s0 : -INFINITY;
        x[2] = v1 ? sc[2] * s1 : -INFINITY;
        x[3] = (v1 && !kSpread) ? sc[3] * s1 : -INFINITY;
        float mx0 = fmaxf(x[0], x[2]);
#pragma unroll
        for (int mk = 4; mk < 32; mk <<= 1) mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, mk));
        const float mn0 = fmaxf(m_run[0], mx0);
        const float al0 = (mn0 == -INFINITY) ? 1.f : fast_exp2(m_run[0] - mn0);
        m_run[0] = mn0;
        float pr[4];
        pr[0] = (x[0] == -INFINITY) ? 0.f : fast_exp2(x[0] - mn0);
        pr[2] = (x[2] == -INFINITY) ? 0.f : fast_exp2(x[2] - mn0);
        l_lane[0] = l_lane[0] * al0 + pr[0] + pr[2];
        float al1 = 1.f;
        pr[1] = pr[3] = 0.f;
        if constexpr (!kSpread) {
            float mx1 = fmaxf(x[1], x[3]);
#pragma unroll
            for (int mk = 4; mk < 32; mk <<= 1) mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, mk));
            const float mn1 = fmaxf(m_run[1], mx1);
            al1 = (mn1 == -INFINITY) ? 1.f : fast_exp2(m_run[1] - mn1);
            m_run[1] = mn1;
            pr[1] = (x[1] == -INFINITY) ? 0.f : fast_exp2(x[1] - mn1);
            pr[3] = (x[3] == -INFINITY) ? 0.f : fast_exp2(x[3] - mn1);
            l_lane[1] = l_lane[1] * al1 + pr[1] + pr[3];
        }
        // ---- V scales: P' = p * sv / svmax
        const float sv0 = v0 ? vsc[r] : 0.f;
        const float sv1 = v1 ? vsc[r + 8] : 0.f;
        float svmax = fmaxf(sv0, sv1);
#pragma unroll
        for (int mk = 4; mk < 32; mk <<= 1) svmax = fmaxf(svmax, __shfl_xor_sync(0xffffffffu, svmax, mk));
        const float inv = svmax > 0.f ? 1.f / svmax : 0.f;
        const float w0 = sv0 * inv, w1 = sv1 * inv;
        const uint32_t bh0 = transpose8x8(Mma<__half>::pack(pr[0] * w0, pr[1] * w0));
        const uint32_t bh1 = transpose8x8(Mma<__half>::pack(pr[2] * w1, pr[3] * w1));
        // ---- O^T = O^T alpha + svmax (Vq^T P'^T)
        uint32_t wa[kW / 4], wb[kW / 4], wc[kW / 4], wd[kW / 4];  // token rows 2q, 2q+1, 2q+8, 2q+9
        const unsigned char *vcol = Vb + kW * r;
        if constexpr (S::kVSwizzle) {
            // swizzled tile: 16-byte chunk c of row t sits at chunk c ^ (t % 8), so the
            // four lanes reading dims W r .. of rows 2q, .. hit four different chunks
            const int c0 = r ^ (2 * q4), c1 = r ^ (2 * q4 + 1);
            const uint4 a = *reinterpret_cast<const uint4 *>(Vb + (2 * q4) * D + 16 * c0);
            const uint4 b = *reinterpret_cast<const uint4 *>(Vb + (2 * q4 + 1) * D + 16 * c1);
            const uint4 c = *reinterpret_cast<const uint4 *>(Vb + (2 * q4 + 8) * D + 16 * c0);
            const uint4 d = *reinterpret_cast<const uint4 *>(Vb + (2 * q4 + 9) * D + 16 * c1);
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                wa[w] = word_of(a, w);
                wb[w] = word_of(b, w);
                wc[w] = word_of(c, w);
                wd[w] = word_of(d, w);
            }
        } else if constexpr (kW == 16) {
            const uint4 a = *reinterpret_cast<const uint4 *>(vcol + (2 * q4) * D);
            const uint4 b = *reinterpret_cast<const uint4 *>(vcol + (2 * q4 + 1) * D);
            const uint4 c = *reinterpret_cast<const uint4 *>(vcol + (2 * q4 + 8) * D);
            const uint4 d = *reinterpret_cast<const uint4 *>(vcol + (2 * q4 + 9) * D);
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                wa[w] = word_of(a, w);
                wb[w] = word_of(b, w);
                wc[w] = word_of(c, w);
                wd[w] = word_of(d, w);
            }
        } else {
            const uint2 a = *reinterpret_cast<const uint2 *>(vcol + (2 * q4) * D);
            const uint2 b = *reinterpret_cast<const uint2 *>(vcol + (2 * q4 + 1) * D);
            const uint2 c = *reinterpret_cast<const uint2 *>(vcol + (2 * q4 + 8) * D);
            const uint2 d = *reinterpret_cast<const uint2 *>(vcol + (2 * q4 + 9) * D);
            wa[0] = a.x; wa[1] = a.y;
            wb[0] = b.x; wb[1] = b.y;
            wc[0] = c.x; wc[1] = c.y;
            wd[0] = d.x; wd[1] = d.y;
        }
        // pairs (token lo, token hi) of one dim e: lo tokens (2q, 2q+1) -> cols 2q, 2q+1; hi -> 2q+8, 2q+9
        uint32_t plo[kW], phi[kW];
#pragma unroll
        for (int w = 0; w < kW / 4; ++w) {
            const uint32_t l01 = __byte_perm(wa[w], wb[w], 0x5140u) ^ 0x80808080u;  // dims 4w, 4w+1
            const uint32_t l23 = __byte_perm(wa[w], wb[w], 0x7362u) ^ 0x80808080u;  // dims 4w+2, 4w+3
            const uint32_t h01 = __byte_perm(wc[w], wd[w], 0x5140u) ^ 0x80808080u;
            const uint32_t h23 = __byte_perm(wc[w], wd[w], 0x7362u) ^ 0x80808080u;
            plo[4 * w + 0] = i8pair_to_h2(l01, 0x4140u);
            plo[4 * w + 1] = i8pair_to_h2(l01, 0x4342u);
            plo[4 * w + 2] = i8pair_to_h2(l23, 0x4140u);
            plo[4 * w + 3] = i8pair_to_h2(l23, 0x4342u);
            phi[4 * w + 0] = i8pair_to_h2(h01, 0x4140u);
            phi[4 * w + 1] = i8pair_to_h2(h01, 0x4342u);
            phi[4 * w + 2] = i8pair_to_h2(h23, 0x4140u);
            phi[4 * w + 3] = i8pair_to_h2(h23, 0x4342u);
        }
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt) {
            float t[4] = {0.f, 0.f, 0.f, 0.f};
            // row r: dim mt; row r + 8: dim kW/2 + mt (of this lane's W dims)
            mma_f16(t, plo[mt], plo[kW / 2 + mt], phi[mt], phi[kW / 2 + mt], bh0, bh1);
            o[mt][0] = fmaf(svmax, t[0], o[mt][0] * al0);
            o[mt][2] = fmaf(svmax, t[2], o[mt][2] * al0);
            if constexpr (!kSpread) {  // else the odd (padding) columns are never stored
                o[mt][1] = fmaf(svmax, t[1], o[mt][1] * al1);
                o[mt][3] = fmaf(svmax, t[3], o[mt][3] * al1);
            }
        }
    }

    __device__ __forceinline__ void store(float *mg, float *lg, float *ag, int warp, int) {
#pragma unroll
        for (int h = 0; h < kH; ++h) {
#pragma unroll
            for (int mk = 4; mk < 32; mk <<= 1) l_lane[h] += __shfl_xor_sync(0xffffffffu, l_lane[h], mk);
        }
#pragma unroll
        for (int h = 0; h < kH; ++h) {
            const int g = kSpread ? q4 : 2 * q4 + h;  // the head of column 2 q4 + h
            if (g < G) {
                if (r == 0) {
                    mg[warp * G + g] = m_run[h];
                    lg[warp * G + g] = l_lane[h];
                }
                float *row = ag + ((size_t)warp * G + g) * S::kAgStride;
#pragma unroll
                for (int mt = 0; mt < kMT; ++mt) {
                    row[dim_of(r, mt)] = o[mt][h];
                    row[dim_of(r + 8, mt)] = o[mt][2 + h];
                }
            }
        }
    }
};

// -------------------------------------------------------------------- kernel

// T: the cache's element type (int8_t: codes with per-row scales); TQ: the
// query's type (T for 16- and 32-bit caches); kAppend: each sequence's newest
// token comes from p.new_key / p.new_value (pa_decode_append; 16- and 32-bit
// caches).
template <typename T, int D, int BS, int G, typename TQ = T, bool kAppend = false>
__global__ void __launch_bounds__(DecodeShape<T, D, BS, G>::kThreads, DecodeShape<T, D, BS, G>::kMinBlocks)
    decode_kernel(const __grid_constant__ DecodeParams p) {
    using S = DecodeShape<T, D, BS, G>;
    using Consumer = std::conditional_t<
        S::kInt8, MmaConsumerQ8<TQ, D, G, S>,
        std::conditional_t<S::kUseMma, MmaConsumer<T, D, G, S>, FmaConsumer<T, D, G, S>>>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *ring = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + S::kAlign - 1) & ~uintptr_t(S::kAlign - 1));
    uint64_t *full = reinterpret_cast<uint64_t *>(ring + S::kDataBytes);
    int *bad = reinterpret_cast<int *>(full + S::kStages);
    // test hook, staged by thread 0 and read only where used: [0] this CTA's
    // withheld stage (-1: none); [2..3] the wait bound in ns. [4..5] the
    // CTA's first query head and [6] its head count, kept here across the
    // stage loop instead of in registers.
    int *hook = bad + S::kStages;
    const uint64_t *wait_limit = reinterpret_cast<const uint64_t *>(hook + 2);

    // prefill through this kernel is for fp32 caches only (the other types
    // prefill on the tensor cores); one CTA column per query token
    constexpr bool kPrefillMode = std::is_same_v<T, float>;
    const bool prefill = kPrefillMode && p.q_start != nullptr;
    const int part = prefill ? 0 : (int)blockIdx.x;
    // groups of 1 and 2 run unpadded; only the compiled size 8 has sub-groups
    const int kvh = (G == 8 && p.sub_groups > 1) ? (int)blockIdx.y / p.sub_groups : (int)blockIdx.y;
    const int sub = (G == 8 && p.sub_groups > 1) ? (int)blockIdx.y % p.sub_groups : 0;
    const int g_valid = G <= 2 ? G : min(G, p.group - sub * G);  // real query heads of this CTA
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const bool split = p.partition_size > 0;
    int s, qrow;  // sequence (table row, context) and query / output row
    int ctx;
    bool ctx_bad = false;
    if (kPrefillMode && prefill) {
        qrow = blockIdx.x;
        if (qrow < p.q_start[0] || qrow >= p.q_start[p.num_seqs]) return;  // a token of no sequence
        int lo = 0, hi = p.num_seqs;  // q_start[lo] <= qrow < q_start[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (p.q_start[mid] <= qrow) lo = mid; else hi = mid;
        }
        s = lo;
        const int q_len = p.q_start[s + 1] - p.q_start[s];
        const int ctx_s = p.context_lens[s];
        if (q_len > ctx_s) {  // more new tokens than cached ones: the sequence is skipped
            if (threadIdx.x == 0 && kvh == 0) record_error(p.err, PA_DEVERR_CONTEXT);
            return;
        }
        ctx = ctx_s - q_len + (qrow - p.q_start[s]) + 1;  // causal: up to this token's own position
    } else {
        s = p.seq_order ? p.seq_order[blockIdx.z] : (int)blockIdx.z;
        if (s < 0 || s >= (int)gridDim.z) {  // a bad schedule entry: nothing to do for it
            if (threadIdx.x == 0 && part == 0 && kvh == 0) record_error(p.err, PA_DEVERR_CONTEXT);
            return;
        }
        qrow = s;
        ctx = p.context_lens[s];
    }

    // ---- token range of this CTA
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
    const int nstage = (t_end - t_begin + S::kTS - 1) / S::kTS;  // 16-token stages

    const size_t head0 = (size_t)qrow * p.num_heads + (size_t)kvh * (G <= 2 ? G : p.group) + (size_t)sub * G;
    if (nstage == 0) {  // unsplit, empty context: zeros
        for (int i = threadIdx.x; i < g_valid * D; i += blockDim.x) store_out(p.out, head0 * D + i, 0.f, p.out_dtype);
        return;
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < S::kStages; ++i) mbar_init(full + i, 1);
        fence_mbar_init();
        hook[0] = (s == p.withhold_seq && kvh == p.withhold_kvh && part == 0) ? p.withhold_stage : -1;
        *reinterpret_cast<uint64_t *>(hook + 2) = p.wait_limit_ns ? p.wait_limit_ns : kWaitLimitNs;
        *reinterpret_cast<uint64_t *>(hook + 4) = head0;
        hook[6] = g_valid;
    }
    __syncthreads();

    // ---- this warp's stages k = warp + 4 m, m < nmine
    const int nmine = nstage > warp ? (nstage - warp + S::kWarps - 1) / S::kWarps : 0;
    const int32_t *row = p.block_tables + (size_t)s * p.max_blocks_per_seq + t_begin / BS;
    const size_t block_elems = (size_t)p.num_kv_heads * BS * D;
    const T *kc = static_cast<const T *>(p.k_cache) + (size_t)kvh * BS * D;
    const T *vc = static_cast<const T *>(p.v_cache) + (size_t)kvh * BS * D;
    const float *ksc = S::kInt8 ? p.k_scale + (size_t)kvh * BS : nullptr;
    const float *vsc = S::kInt8 ? p.v_scale + (size_t)kvh * BS : nullptr;
    const uint64_t pol = l2_evict_first_policy();

    // Block id of local stage m0 + lane (-1: none, or a bad entry).
    auto load_ids = [&](int m0) -> int {
        const int m = m0 + lane;
        int id = -1;
        if (m < nmine) {
            id = __ldg(row + ((warp + S::kWarps * m) * S::kTS) / BS);
            if (id < 0 || id >= p.num_blocks) {
                record_error(p.err, PA_DEVERR_BLOCK_ID);
                id = -1;
            }
        }
        return id;
    };
    int m0 = 0;
    int ids_cur = load_ids(0);
    int ids_next = load_ids(32);
    auto id_of = [&](int m) -> int {  // whole warp; m0 <= m < m0 + 64
        const int a = __shfl_sync(0xffffffffu, ids_cur, (m - m0) & 31);
        const int b = __shfl_sync(0xffffffffu, ids_next, (m - m0) & 31);
        return (m - m0 < 32) ? a : b;
    };
    auto issue = [&](int m, int id) {  // lane 0
        const int k = warp + S::kWarps * m;
        const int buf = k % S::kStages;
        if (k == hook[0]) {
            // test hook: no copy and no arrival, so this stage's wait runs out
            bad[buf] = 1;
        } else if (id >= 0) {
            bad[buf] = 0;
            const size_t src = (size_t)id * block_elems + (size_t)(k % S::kSubs) * S::kTS * D;
            unsigned char *dst = ring + S::kVRegion + (size_t)buf * S::kStageBytes;
            mbar_arrive_expect_tx(full + buf, 2 * S::kTileBytes + 2 * S::kScaleBytes);
            if constexpr (S::kKSwizzle) {  // K: the same pool rows as V, boxes of 128 bytes
                const int krow = (int)(((long long)id * p.num_kv_heads + kvh) * BS + (k % S::kSubs) * S::kTS);
#pragma unroll
                for (int h = 0; h < S::kVBoxes; ++h)
                    tma_load_2d(dst + h * 2048, &p.k_map, h * (128 / S::kElt), krow, full + buf);
            } else {
                bulk_load(dst, kc + src, S::kTileBytes, full + buf, pol);
            }
            if constexpr (S::kVSwizzle) {  // V: pool rows (block, kv head, token) as 2-D boxes of 128 bytes
                const int vrow = (int)(((long long)id * p.num_kv_heads + kvh) * BS + (k % S::kSubs) * S::kTS);
#pragma unroll
                for (int h = 0; h < S::kVBoxes; ++h)
                    tma_load_2d(ring + (size_t)buf * S::kTileBytes + h * 2048, &p.v_map, h * (128 / S::kElt), vrow,
                                full + buf);
            } else {
                bulk_load(dst + S::kTileBytes, vc + src, S::kTileBytes, full + buf, pol);
            }
            if constexpr (S::kInt8) {  // the 16 rows' scales: 64 contiguous bytes each
                const size_t ssrc = (size_t)id * p.num_kv_heads * BS + (size_t)(k % S::kSubs) * S::kTS;
                bulk_load(dst + S::kScaleOff, ksc + ssrc, S::kScaleBytes, full + buf, pol);
                bulk_load(dst + S::kScaleOff + S::kScaleBytes, vsc + ssrc, S::kScaleBytes, full + buf, pol);
            }
        } else {
            bad[buf] = 1;
            mbar_arrive(full + buf);
        }
    };
#pragma unroll
    for (int m = 0; m < S::kBufPerWarp; ++m) {
        const int id = id_of(m);
        if (lane == 0 && m < nmine) issue(m, id);
    }

    // pa_decode_append: the sequence's newest token (position ctx - 1) comes
    // from new_key / new_value. The warp whose stage k_new holds it loads the
    // two rows now; once that stage has landed it puts them over the tile
    // rows (the pool's copy may be stale) and writes them into the pool.
    static_assert(!(kAppend && S::kInt8), "the append form is for 16- and 32-bit caches");
    constexpr int kRowChunks = D * S::kElt / 16;  // 16-byte pieces of one K or V row
    constexpr int kNewPerLane = kAppend ? (2 * kRowChunks + 31) / 32 : 1;
    int k_new = -1;
    uint4 nrow[kNewPerLane];
    if constexpr (kAppend) {
        if (ctx > 0 && ctx - 1 >= t_begin && ctx - 1 < t_end)
            k_new = (ctx - 1 - t_begin) / S::kTS;
        if (k_new >= 0 && k_new % S::kWarps == warp) {
            const size_t row0 = ((size_t)s * p.num_kv_heads + kvh) * D * S::kElt;  // bytes
#pragma unroll
            for (int i = 0; i < kNewPerLane; ++i) {
                const int c = lane + 32 * i;
                nrow[i] = make_uint4(0u, 0u, 0u, 0u);
                if (c < 2 * kRowChunks) {
                    const unsigned char *src = static_cast<const unsigned char *>(c < kRowChunks ? p.new_key : p.new_value);
                    nrow[i] = __ldg(reinterpret_cast<const uint4 *>(src + row0) + (c % kRowChunks));
                }
            }
        }
    }

    Consumer cons;
    if constexpr (S::kInt8) {
        cons.init(p, head0, g_valid, warp, lane, reinterpret_cast<uint4 *>(hook + 8));
    } else {
        cons.init(p, head0, g_valid, warp, lane);
    }
    int waited = 0;
    bool ok = true;
    for (int m = 0; m < nmine; ++m) {
        if (m - m0 == 32) {
            m0 = m;
            ids_cur = ids_next;
            ids_next = load_ids(m0 + 32);
        }
        const int k = warp + S::kWarps * m;
        const int buf = k % S::kStages;
        // Lane 0 polls the barrier (32 lanes polling would serialise on it);
        // __syncwarp then orders the other lanes' reads after its acquire.
        const bool got = mbar_wait(full + buf, (k / S::kStages) & 1, wait_limit);
        if (!__all_sync(0xffffffffu, got)) {
            if (lane == 0) record_error(p.err, PA_DEVERR_TIMEOUT);
            ok = false;
            break;
        }
        waited = m + 1;
        if constexpr (kAppend) {
            if (k == k_new) {
                const int id = id_of(m);  // the stage's block (whole warp)
                if (!bad[buf]) {
                    const int r = (ctx - 1 - t_begin) % S::kTS;  // row in the stage
                    unsigned char *Kw = ring + S::kVRegion + (size_t)buf * S::kStageBytes;
                    const size_t prow = ((size_t)id * block_elems + (size_t)((ctx - 1) % BS) * D) * S::kElt;
#pragma unroll
                    for (int i = 0; i < kNewPerLane; ++i) {
                        const int c = lane + 32 * i;
                        if (c < 2 * kRowChunks) {
                            const bool isv = c >= kRowChunks;
                            const int cc = c % kRowChunks;
                            if (S::kVSwizzle && isv) {  // the swizzled V box of chunk cc (128 bytes a box)
                                unsigned char *vbox = ring + (size_t)buf * S::kTileBytes + (cc >> 3) * 2048;
                                *reinterpret_cast<uint4 *>(vbox + r * 128 + (((cc & 7) ^ (r & 7)) << 4)) = nrow[i];
                            } else if (S::kKSwizzle && !isv) {  // the swizzled K box
                                *reinterpret_cast<uint4 *>(Kw + (cc >> 3) * 2048 + r * 128 + (((cc & 7) ^ (r & 7)) << 4)) =
                                    nrow[i];
                            } else {
                                reinterpret_cast<uint4 *>(Kw + (isv ? S::kTileBytes : 0) + (size_t)r * D * S::kElt)[cc] =
                                    nrow[i];
                            }
                            if (sub == 0) {  // one CTA of the kv head writes the pool
                                const unsigned char *pool = reinterpret_cast<const unsigned char *>(isv ? vc : kc);
                                reinterpret_cast<uint4 *>(const_cast<unsigned char *>(pool) + prow)[cc] = nrow[i];
                            }
                        }
                    }
                }
                __syncwarp();
            }
        }
        if (!bad[buf]) {
            const int nvalid = min(S::kTS, t_end - (t_begin + k * S::kTS));
            const unsigned char *Kb = ring + S::kVRegion + (size_t)buf * S::kStageBytes;
            const unsigned char *Vb = S::kVSwizzle ? ring + (size_t)buf * S::kTileBytes : Kb + S::kTileBytes;
            cons.stage(Kb, Vb, nvalid, lane, p.scale_log2);
        }
        // Reload this buffer with this warp's stage m + kBufPerWarp.
        const int idn = id_of(m + S::kBufPerWarp);
        __syncwarp();
        if (lane == 0 && m + S::kBufPerWarp < nmine) {
            fence_proxy_async_smem();
            issue(m + S::kBufPerWarp, idn);
        }
    }
    if (!ok && lane == 0) {  // after a timeout: let every copy this warp started land
        for (int m = waited; m < min(nmine, waited + S::kBufPerWarp); ++m) {
            const int k = warp + S::kWarps * m;
            if (!mbar_wait(full + (k % S::kStages), (k / S::kStages) & 1, wait_limit))
                record_error(p.err, PA_DEVERR_TIMEOUT);
        }
    }

    // ---- merge the row groups (log-sum-exp), reusing the drained ring
    float *mg = reinterpret_cast<float *>(ring);  // [row group][G]
    float *lg = mg + S::kRowGroups * G;          // [row group][G]
    float *ag = lg + S::kRowGroups * G;          // [row group][G][D]
    __syncthreads();
    cons.store(mg, lg, ag, warp, lane);
    __syncthreads();
    // the head range, read back from shared memory (nothing keeps it live
    // through the loop)
    const size_t head_first = *reinterpret_cast<volatile uint64_t *>(hook + 4);
    const int heads = *reinterpret_cast<volatile int *>(hook + 6);
    for (int idx = threadIdx.x; idx < heads * D; idx += S::kThreads) {
        const int g = idx / D;
        const int d = idx % D;
        float Mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < S::kRowGroups; ++i) Mx = fmaxf(Mx, mg[i * G + g]);
        float num = 0.f, den = 0.f;
        if (Mx != -INFINITY) {
#pragma unroll
            for (int i = 0; i < S::kRowGroups; ++i) {
                const float w = fast_exp2(mg[i * G + g] - Mx);
                num = fmaf(w, ag[((size_t)i * G + g) * S::kAgStride + d], num);
                den = fmaf(w, lg[i * G + g], den);
            }
        }
        const size_t h = head_first + g;
        if (split) {
            const size_t slot = h * p.max_parts + part;
            p.ws_acc[slot * D + d] = num;
            if (d == 0) {
                p.ws_ml[slot * 2] = Mx * kLn2;
                p.ws_ml[slot * 2 + 1] = den;
            }
        } else {
            store_out(p.out, h * D + d, den > 0.f ? num / den : 0.f, p.out_dtype);
        }
    }
}

// -------------------------------------------------------------- split reduce

// One CTA of 8 warps per (sequence, query head): warp w folds partitions
// w, w + 8, ... (each lane holding 4 consecutive head dims as one float4, so
// a partition row is one coalesced 512-byte read), then the warps combine
// through shared memory.
constexpr int kReduceWarps = 8;

__global__ void __launch_bounds__(kReduceWarps * 32)
    splitk_reduce_kernel(void *out, const float *ws_ml, const float *ws_acc,
                         const int32_t *context_lens, int num_heads, int head_dim,
                         int partition_size, int max_parts, int max_context_len,
                         pa_dtype out_dtype) {
    __shared__ float red_m[kReduceWarps], red_l[kReduceWarps];
    __shared__ float4 red_acc[kReduceWarps][32];
    const int h = blockIdx.x;
    const int s = blockIdx.y;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    int ctx = context_lens[s];
    ctx = max(0, min(ctx, max_context_len));
    const int n = (ctx + partition_size - 1) / partition_size;
    const size_t row = (size_t)s * num_heads + h;
    const int vec = head_dim / 4;  // float4 per partition row (16 or 32)
    if (n == 0) {
        for (int d = threadIdx.x; d < head_dim; d += blockDim.x) store_out(out, row * head_dim + d, 0.f, out_dtype);
        return;
    }
    const float *ml = ws_ml + row * max_parts * 2;
    const float4 *acc = reinterpret_cast<const float4 *>(ws_acc + row * max_parts * head_dim);
    // One pass: warp w takes partitions w, w + 8, ... in batches of kU whose
    // loads are all issued before any is used (one L2 round trip per batch),
    // keeping its own running max m_w: sum of e^(m_p - m_w) l_p and of
    // e^(m_p - m_w) acc_p, rescaled when m_w grows. The warps then merge with
    // weights e^(m_w - M), M the largest m_w.
    constexpr int kU = 8;
    float m_w = -INFINITY, den = 0.f;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = warp; i < n; i += kReduceWarps * kU) {
        float m[kU], l[kU];
        float4 a[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int iu = i + u * kReduceWarps;
            const bool ok = iu < n;
            m[u] = ok ? ml[2 * iu] : -INFINITY;
            l[u] = ok ? ml[2 * iu + 1] : 0.f;
            a[u] = (ok && lane < vec) ? acc[(size_t)iu * vec + lane] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float mb = m_w;
#pragma unroll
        for (int u = 0; u < kU; ++u) mb = fmaxf(mb, m[u]);
        if (mb == -INFINITY) continue;  // nothing finite yet
        const float r = fast_exp2((m_w - mb) * kLog2e);  // 0 while m_w is -inf
        den *= r;
        num.x *= r;
        num.y *= r;
        num.z *= r;
        num.w *= r;
        m_w = mb;
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            if (i + u * kReduceWarps >= n) break;
            const float w = fast_exp2((m[u] - m_w) * kLog2e);
            den = fmaf(w, l[u], den);
            num.x = fmaf(w, a[u].x, num.x);
            num.y = fmaf(w, a[u].y, num.y);
            num.z = fmaf(w, a[u].z, num.z);
            num.w = fmaf(w, a[u].w, num.w);
        }
    }
    if (lane == 0) {
        red_m[warp] = m_w;
        red_l[warp] = den;
    }
    red_acc[warp][lane] = num;
    __syncthreads();
    if (warp == 0) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kReduceWarps; ++w) M = fmaxf(M, red_m[w]);
        float dsum = 0.f;
        float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kReduceWarps; ++w) {
            const float mw = red_m[w];
            const float f = (mw == -INFINITY) ? 0.f : fast_exp2((mw - M) * kLog2e);
            dsum = fmaf(f, red_l[w], dsum);
            const float4 a = red_acc[w][lane];
            t.x = fmaf(f, a.x, t.x);
            t.y = fmaf(f, a.y, t.y);
            t.z = fmaf(f, a.z, t.z);
            t.w = fmaf(f, a.w, t.w);
        }
        if (lane < vec) {
            const float inv = dsum > 0.f ? 1.f / dsum : 0.f;
            const size_t o = row * head_dim + 4 * lane;
            store_out(out, o + 0, t.x * inv, out_dtype);
            store_out(out, o + 1, t.y * inv, out_dtype);
            store_out(out, o + 2, t.z * inv, out_dtype);
            store_out(out, o + 3, t.w * inv, out_dtype);
        }
    }
}

// ------------------------------------------------------------------ launchers

template <typename T, int D, int BS, int G, typename TQ = T, bool kAppend = false>
static cudaError_t launch_decode_t(const DecodeParams &p, int grid_x, int num_kv_heads, int num_seqs,
                                   cudaStream_t stream) {
    using S = DecodeShape<T, D, BS, G>;
    auto kern = decode_kernel<T, D, BS, G, TQ, kAppend>;
    static AttrCache attr_done;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(kern), S::kSmemBytes, &attr_done);
    if (e != cudaSuccess) return e;
    dim3 grid(grid_x, num_kv_heads * p.sub_groups, num_seqs);
    kern<<<grid, S::kThreads, S::kSmemBytes, stream>>>(p);
    return cudaGetLastError();
}

// The compiled group size serving a head group of `group` query heads: the
// next power of two up to 8 (larger groups run as sub-groups of 8).
static int padded_group(int group) { return group <= 1 ? 1 : group <= 2 ? 2 : group <= 4 ? 4 : 8; }

template <typename T, int D, int BS, typename TQ = T, bool kAppend = false>
static cudaError_t dispatch_group(const DecodeParams &p0, int group, int grid_x, int num_kv_heads,
                                  int num_seqs, cudaStream_t stream) {
    if (group < 1) return cudaErrorInvalidValue;
    DecodeParams p = p0;
    const int gt = padded_group(group);
    p.group = group;
    p.sub_groups = (group + gt - 1) / gt;
    switch (gt) {
        case 1: return launch_decode_t<T, D, BS, 1, TQ, kAppend>(p, grid_x, num_kv_heads, num_seqs, stream);
        case 2: return launch_decode_t<T, D, BS, 2, TQ, kAppend>(p, grid_x, num_kv_heads, num_seqs, stream);
        case 4: return launch_decode_t<T, D, BS, 4, TQ, kAppend>(p, grid_x, num_kv_heads, num_seqs, stream);
        default: return launch_decode_t<T, D, BS, 8, TQ, kAppend>(p, grid_x, num_kv_heads, num_seqs, stream);
    }
}

template <typename T, typename TQ = T, bool kAppend = false>
static cudaError_t dispatch_shape(const DecodeParams &p, int head_dim, int block_size, int group,
                                  int grid_x, int num_kv_heads, int num_seqs, cudaStream_t stream) {
    if (head_dim == 64 && block_size == 16) return dispatch_group<T, 64, 16, TQ, kAppend>(p, group, grid_x, num_kv_heads, num_seqs, stream);
    if (head_dim == 64 && block_size == 32) return dispatch_group<T, 64, 32, TQ, kAppend>(p, group, grid_x, num_kv_heads, num_seqs, stream);
    if (head_dim == 128 && block_size == 16) return dispatch_group<T, 128, 16, TQ, kAppend>(p, group, grid_x, num_kv_heads, num_seqs, stream);
    if (head_dim == 128 && block_size == 32) return dispatch_group<T, 128, 32, TQ, kAppend>(p, group, grid_x, num_kv_heads, num_seqs, stream);
    return cudaErrorInvalidValue;
}

template <typename T>
static cudaError_t dispatch_append(const DecodeParams &p, int head_dim, int block_size, int group, int grid_x,
                                   int num_kv_heads, int num_seqs, cudaStream_t stream) {
    return p.new_key ? dispatch_shape<T, T, true>(p, head_dim, block_size, group, grid_x, num_kv_heads, num_seqs, stream)
                     : dispatch_shape<T, T, false>(p, head_dim, block_size, group, grid_x, num_kv_heads, num_seqs, stream);
}

cudaError_t launch_decode(const DecodeParams &p0, pa_dtype kv_dtype, int head_dim, int block_size,
                          int group, int grid_x, int num_kv_heads, int num_seqs,
                          cudaStream_t stream) {
    DecodeParams p = p0;
    if ((kv_dtype == PA_F16 || kv_dtype == PA_BF16) && padded_group(group) >= 2) {
        // the tensor-core consumer's V tiles: the V pool as rows of head_dim
        // 16-bit elements, boxes of 64 elements x 16 rows, 128-byte swizzle
        const long long rows = (long long)p.num_blocks * num_kv_heads * block_size;
        if (rows >= INT_MAX) return cudaErrorInvalidValue;  // TMA row coordinates are 32-bit
        const CUtensorMapDataType dt =
            kv_dtype == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
        if (rows > 0 &&
            (!encode_rows_2d(&p.v_map, dt, p.v_cache, (unsigned long long)head_dim, (unsigned long long)rows,
                             (unsigned long long)head_dim * 2, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B) ||
             !encode_rows_2d(&p.k_map, dt, p.k_cache, (unsigned long long)head_dim, (unsigned long long)rows,
                             (unsigned long long)head_dim * 2, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B)))
            return cudaErrorInvalidValue;
    }
    switch (kv_dtype) {
        case PA_F32: return dispatch_append<float>(p, head_dim, block_size, group, grid_x, num_kv_heads, num_seqs, stream);
        case PA_F16: return dispatch_append<__half>(p, head_dim, block_size, group, grid_x, num_kv_heads, num_seqs, stream);
        case PA_BF16: return dispatch_append<__nv_bfloat16>(p, head_dim, block_size, group, grid_x, num_kv_heads, num_seqs, stream);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode_q8(const DecodeParams &p, pa_dtype q_dtype, int head_dim, int block_size, int group,
                             int grid_x, int num_kv_heads, int num_seqs, cudaStream_t stream) {
    switch (q_dtype) {
        case PA_F16: return dispatch_shape<int8_t, __half>(p, head_dim, block_size, group, grid_x, num_kv_heads, num_seqs, stream);
        case PA_BF16: return dispatch_shape<int8_t, __nv_bfloat16>(p, head_dim, block_size, group, grid_x, num_kv_heads, num_seqs, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_splitk_reduce(void *out, const float *ws_ml, const float *ws_acc,
                                 const int32_t *context_lens, int num_seqs, int num_heads,
                                 int head_dim, int partition_size, int max_parts,
                                 int max_context_len, pa_dtype out_dtype, cudaStream_t stream) {
    dim3 grid(num_heads, num_seqs);
    splitk_reduce_kernel<<<grid, kReduceWarps * 32, 0, stream>>>(out, ws_ml, ws_acc, context_lens,
                                                                 num_heads, head_dim, partition_size,
                                                                 max_parts, max_context_len, out_dtype);
    return cudaGetLastError();
}

}  // namespace pa
