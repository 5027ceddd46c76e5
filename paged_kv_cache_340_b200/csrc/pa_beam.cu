// Device block pool and the beam-search step on the GPU.
//
// The host pool's state (reference counts and the free list) lives in one
// device buffer, so a decoding loop whose beam choices are made on the GPU
// (a device top-k) can fork, release and copy-on-write without a host round
// trip, and the whole step can be captured in a CUDA graph.
//
// One beam step ([P2 "PagedAttention原理与KV Cache显存优化", §3.4: beam search
// shares blocks between beams and copies a shared block before a beam
// writes into it]; [P4 "PagedAttention 实现细节", §3.3: the copy-on-write
// rule]): new beam i continues old beam parents[i] and writes one token.
// The result is exactly that of running, one after another,
//   1. every new beam forks its parent (each block's count goes up),
//   2. every old beam is released in beam order, each table in order (a
//      block reaching count 0 goes to the back of the free list),
//   3. every new beam writes its token in beam order: at a block boundary it
//      takes a free block; otherwise, if its block's count is above 1, it
//      takes a free block, records (old, new) for the copy and drops the old
//      block's count; else it writes in place.
// The kernel reaches that sequential result in parallel with one CTA:
//   * counts: net change per block accumulated with atomics in a scratch
//     array, applied once;
//   * free-list order: a block is freed at its last decrement, the largest
//     flattened (beam, table position) index holding it; a block-wide scan
//     over those indices gives each freed block its place;
//   * copy-on-write: writer i into block b finds count > 1 unless it is the
//     last writer into b (largest i) and no other new beam holds b, so
//     copies = (not last writer) or (other holders > 0);
//   * takes: a block-wide scan of "needs a block" in beam order gives each
//     writer its position in the free list (front for FIFO, back for LIFO).
// Everything is checked before anything changes: on an error the state is
// unchanged, every slot is -1 and the copy count is 0.
#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {
namespace beam {

constexpr int kThreads = 1024;
constexpr int kItems = 16;         // table entries per thread per pass
constexpr int kScanItems = 8;      // the same in the scanned pass (four values per entry)
// per-beam values staged in shared memory: 3 words per old beam, 1 per new beam
constexpr int kMaxStageBytes = PA_BEAM_MAX_STAGED * 4;
// per-beam values plus the old tables, when they fit in this much
constexpr int kMaxDynBytes = 200 * 1024;
constexpr int32_t kMagic = 0x50414250;

struct Pool {
    int32_t *hdr, *ref, *ring, *delta, *last_old, *writers, *last_writer;
};

__device__ __forceinline__ Pool views(int32_t *state, int nb) {
    Pool p;
    p.hdr = state;
    p.ref = state + PA_DPOOL_HEADER_WORDS;
    p.ring = p.ref + nb;
    p.delta = p.ring + nb;
    p.last_old = p.delta + nb;
    p.writers = p.last_old + nb;
    p.last_writer = p.writers + nb;
    return p;
}

// Exclusive scan of v over the CTA (all kThreads threads call it); *total
// receives the sum. Ends with a barrier, so warp_sums can be reused.
__device__ __forceinline__ int cta_exclusive_scan(int v, int *warp_sums, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, d);
        if (lane >= d) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = warp_sums[lane];
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, d);
            if (lane >= d) w += y;
        }
        warp_sums[lane] = w;
    }
    __syncthreads();
    const int excl = x - v + (warp ? warp_sums[warp - 1] : 0);
    *total = warp_sums[31];
    __syncthreads();
    return excl;
}

__global__ void __launch_bounds__(256) dpool_fill_kernel(int32_t *state, int nb, const int32_t *free_order) {
    const Pool p = views(state, nb);
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nb; i += gridDim.x * blockDim.x) {
        p.ref[i] = 0;
        p.ring[i] = free_order ? free_order[i] : i;
        p.delta[i] = 0;
        p.last_old[i] = -1;
        p.writers[i] = 0;
        p.last_writer[i] = -1;
    }
}

// Checks that the free list is a permutation (using delta as a counter and
// leaving it at zero), then writes the header.
__global__ void __launch_bounds__(kThreads, 1)
    dpool_seal_kernel(int32_t *state, int nb, int bs, int policy, int check, unsigned int *err) {
    __shared__ int s_bad;
    const Pool p = views(state, nb);
    if (threadIdx.x == 0) s_bad = 0;
    __syncthreads();
    if (check) {
        for (int i = threadIdx.x; i < nb; i += kThreads) {
            const int b = p.ring[i];
            if (b < 0 || b >= nb)
                s_bad = 1;
            else
                atomicAdd(&p.delta[b], 1);
        }
        __syncthreads();
        for (int i = threadIdx.x; i < nb; i += kThreads) {
            if (p.delta[i] != 1) s_bad = 1;
            p.delta[i] = 0;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        p.hdr[0] = nb;
        p.hdr[1] = bs;
        p.hdr[2] = policy;
        p.hdr[3] = 0;   // head
        p.hdr[4] = nb;  // count
        p.hdr[5] = s_bad ? 0 : kMagic;
        p.hdr[6] = 0;
        p.hdr[7] = 0;
        if (s_bad) record_error(err, PA_DEVERR_POOL);
    }
}

// Loads counts and a free list, then checks them: free-list ids in range,
// distinct and of count 0; counts not negative; as many blocks of count 0 as
// free-list entries.
__global__ void __launch_bounds__(kThreads, 1)
    dpool_load_kernel(int32_t *state, int nb, int bs, int policy, const int32_t *ref_counts,
                      const int32_t *free_list, int num_free, unsigned int *err) {
    __shared__ int s_bad, s_zero;
    const Pool p = views(state, nb);
    if (threadIdx.x == 0) {
        s_bad = 0;
        s_zero = 0;
    }
    for (int i = threadIdx.x; i < nb; i += kThreads) {
        const int r = ref_counts[i];
        p.ref[i] = r;
        p.ring[i] = i < num_free ? free_list[i] : -1;
        p.delta[i] = 0;
        p.last_old[i] = -1;
        p.writers[i] = 0;
        p.last_writer[i] = -1;
    }
    __syncthreads();
    int zeros = 0;
    for (int i = threadIdx.x; i < nb; i += kThreads) {
        if (p.ref[i] < 0) s_bad = 1;
        zeros += p.ref[i] == 0;
        if (i < num_free) {
            const int b = p.ring[i];
            if (b < 0 || b >= nb || p.ref[b] != 0)
                s_bad = 1;
            else
                atomicAdd(&p.delta[b], 1);
        }
    }
    atomicAdd(&s_zero, zeros);
    __syncthreads();
    for (int i = threadIdx.x; i < nb; i += kThreads) {
        if (p.delta[i] > 1) s_bad = 1;
        p.delta[i] = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (s_zero != num_free) s_bad = 1;
        p.hdr[0] = nb;
        p.hdr[1] = bs;
        p.hdr[2] = policy;
        p.hdr[3] = 0;
        p.hdr[4] = num_free;
        p.hdr[5] = s_bad ? 0 : kMagic;
        p.hdr[6] = 0;
        p.hdr[7] = 0;
        if (s_bad) record_error(err, PA_DEVERR_POOL);
    }
}

struct StepParams {
    int32_t *state;
    const int32_t *old_tables;
    const int32_t *old_ctx;
    const int32_t *parents;
    int32_t *new_tables;
    int32_t *new_ctx;
    int32_t *slots;
    int64_t *cow_pairs;
    int32_t *num_cow;
    int num_old;
    int num_new;
    int max_blocks;
    int num_blocks;
    int block_size;
    unsigned int *err;
};

__device__ __forceinline__ int nblk(int ctx, int bs) { return (ctx + bs - 1) / bs; }

// Beam j and table position pos of the flattened entries e0, e0 + stride, ...
// of [beams][mb] tables: one division, then per step one add and at most one
// carry (the step's remainder is below mb). The passes below visit 16 entries
// per thread; a division per entry cost more than the memory traffic.
struct EntryWalk {
    int j, pos;
    __device__ __forceinline__ EntryWalk(int e0, int mb) : j(e0 / mb), pos(e0 % mb) {}
    __device__ __forceinline__ void step(int dj, int dpos, int mb) {
        j += dj;
        pos += dpos;
        if (pos >= mb) {
            pos -= mb;
            ++j;
        }
    }
};

// The kernel is latency-bound (one CTA, dependent loads), so every pass over
// table entries first loads kItems entries per thread into registers, then
// acts on them: one or two memory round trips per pass instead of one per
// entry. Table, context and parent arrays are read-only here (__ldg).
// kStaged: the old tables are first copied to shared memory (when they fit),
// so the passes below read them there instead of from L2.
template <bool kStaged>
__global__ void __launch_bounds__(kThreads, 1) beam_step_kernel(const StepParams q) {
    extern __shared__ int dyn[];
    __shared__ int warp_sums[32];
    __shared__ int s_bad;
    const int tid = threadIdx.x;
    const int nb = q.num_blocks, bs = q.block_size, MB = q.max_blocks;
    const Pool p = views(q.state, nb);
    const int n_old = q.num_old, n_new = q.num_new;
    const int old_entries = n_old * MB;  // < 2^31 (host check)
    const int new_entries = n_new * MB;
    const int sdj = kThreads / MB, sdp = kThreads % MB;  // a step of kThreads entries
    int *s_ctx = dyn;                    // [n_old] context length of old beam j
    int *s_nb = dyn + n_old;             // [n_old] its block count
    int *s_nch = dyn + 2 * n_old;        // [n_old] its number of children
    int *s_par = dyn + 3 * n_old;        // [n_new] parent of new beam i
    int *s_tab = dyn + 3 * n_old + n_new;  // kStaged: [n_old * MB] the old tables
    const int32_t *__restrict__ otab = q.old_tables;
    auto tab = [&](int e) -> int {
        if constexpr (kStaged)
            return s_tab[e];
        else
            return __ldg(otab + e);
    };

    if (tid == 0) s_bad = 0;
    __syncthreads();
    const int policy = p.hdr[2], head = p.hdr[3], count = p.hdr[4];
    if (tid == 0 && (p.hdr[5] != kMagic || p.hdr[0] != nb || p.hdr[1] != bs || count < 0 || count > nb ||
                     head < 0 || head >= nb))
        atomicOr(&s_bad, PA_DEVERR_POOL);
    // ---- phase 0: stage and check the inputs (nothing is changed yet)
    for (int j = tid; j < n_old; j += kThreads) {
        const int c = __ldg(q.old_ctx + j);
        s_ctx[j] = c;
        s_nb[j] = c < 0 ? 0 : nblk(c, bs);
        s_nch[j] = 0;
        if (c < 0 || nblk(c, bs) > MB) atomicOr(&s_bad, PA_DEVERR_CONTEXT);
    }
    if constexpr (kStaged) {
        for (int base = 0; base < old_entries; base += kThreads * kItems) {
            int v[kItems];
#pragma unroll
            for (int k = 0; k < kItems; ++k) {
                const int e = base + k * kThreads + tid;
                v[k] = e < old_entries ? __ldg(otab + e) : 0;
            }
#pragma unroll
            for (int k = 0; k < kItems; ++k) {
                const int e = base + k * kThreads + tid;
                if (e < old_entries) s_tab[e] = v[k];
            }
        }
    }
    __syncthreads();
    for (int i = tid; i < n_new; i += kThreads) {
        const int par = __ldg(q.parents + i);
        s_par[i] = par;
        if (par < 0 || par >= n_old)
            atomicOr(&s_bad, PA_DEVERR_CONTEXT);
        else
            atomicAdd(&s_nch[par], 1);
    }
    __syncthreads();
    if (!s_bad) {
        for (int base = 0; base < old_entries; base += kThreads * kItems) {
            int blk[kItems], in_use = 0;
            EntryWalk w(base + tid, MB);
#pragma unroll
            for (int k = 0; k < kItems; ++k) {
                const int e = base + k * kThreads + tid;
                blk[k] = 0;
                if (e < old_entries && w.pos < s_nb[w.j]) {
                    blk[k] = tab(e);
                    in_use |= 1 << k;
                }
                w.step(sdj, sdp, MB);
            }
#pragma unroll
            for (int k = 0; k < kItems; ++k) {
                const int b = blk[k];
                if ((in_use >> k & 1) && (b < 0 || b >= nb || p.ref[b] <= 0)) atomicOr(&s_bad, PA_DEVERR_BLOCK_ID);
            }
        }
        for (int i = tid; i < n_new; i += kThreads)
            if (s_ctx[s_par[i]] / bs >= MB) atomicOr(&s_bad, PA_DEVERR_POOL);  // no room for the token
    }
    __syncthreads();
    if (s_bad) {
        for (int i = tid; i < n_new; i += kThreads) q.slots[i] = -1;
        if (tid == 0) {
            *q.num_cow = 0;
            record_error(q.err, (unsigned)s_bad);
        }
        return;
    }

    // ---- phase 1: net count change. A child's table is its parent's, so a
    // block of old beam j gains (children of j) - 1 references: only beams
    // with other than one child touch the counts. Then the writers.
    for (int base = 0; base < old_entries; base += kThreads * kItems) {
        int blk[kItems];
        EntryWalk w(base + tid, MB);
#pragma unroll
        for (int k = 0; k < kItems; ++k) {
            const int e = base + k * kThreads + tid;
            blk[k] = -1;
            if (e < old_entries && w.pos < s_nb[w.j] && s_nch[w.j] != 1) blk[k] = tab(e);
            w.step(sdj, sdp, MB);
        }
        EntryWalk w2(base + tid, MB);
#pragma unroll
        for (int k = 0; k < kItems; ++k) {
            if (blk[k] >= 0) atomicAdd(&p.delta[blk[k]], s_nch[w2.j] - 1);
            w2.step(sdj, sdp, MB);
        }
    }
    for (int i = tid; i < n_new; i += kThreads) {
        const int par = s_par[i];
        const int t = s_ctx[par];
        if (t % bs) {
            const int o = tab(par * MB + t / bs);
            atomicAdd(&p.writers[o], 1);
            atomicMax(&p.last_writer[o], i);
        }
    }
    __syncthreads();
    // a block is freed only if every old beam holding it has no child; mark
    // the last such entry (in release order) of each block reaching zero
    for (int base = 0; base < old_entries; base += kThreads * kItems) {
        int blk[kItems], r0[kItems];
        EntryWalk w(base + tid, MB);
#pragma unroll
        for (int k = 0; k < kItems; ++k) {
            const int e = base + k * kThreads + tid;
            blk[k] = -1;
            if (e < old_entries && w.pos < s_nb[w.j] && s_nch[w.j] == 0) blk[k] = tab(e);
            w.step(sdj, sdp, MB);
        }
#pragma unroll
        for (int k = 0; k < kItems; ++k)
            if (blk[k] >= 0) r0[k] = p.ref[blk[k]] + p.delta[blk[k]];
#pragma unroll
        for (int k = 0; k < kItems; ++k) {
            if (blk[k] >= 0) {
                if (r0[k] < 0) atomicOr(&s_bad, PA_DEVERR_POOL);  // a table holds a block more often than counted
                if (r0[k] == 0) atomicMax(&p.last_old[blk[k]], base + k * kThreads + tid);
            }
        }
    }
    __syncthreads();

    // ---- phase 2: freed blocks, pushed to the back of the free list in
    // order of their last release (written past the list's end: harmless
    // until the count is updated). Items are contiguous per thread so the
    // scan runs in entry order.
    int freed = 0;
    for (int base = 0; base < old_entries; base += kThreads * kScanItems) {
        int blk[kScanItems], r0[kScanItems], d0[kScanItems], l0[kScanItems];
        EntryWalk w(base + tid * kScanItems, MB);
#pragma unroll
        for (int k = 0; k < kScanItems; ++k) {
            const int e = base + tid * kScanItems + k;
            blk[k] = -1;
            if (e < old_entries && w.pos < s_nb[w.j] && s_nch[w.j] == 0) blk[k] = tab(e);
            w.step(MB == 1 ? 1 : 0, MB == 1 ? 0 : 1, MB);
        }
#pragma unroll
        for (int k = 0; k < kScanItems; ++k) {
            if (blk[k] >= 0) {
                r0[k] = p.ref[blk[k]];
                d0[k] = p.delta[blk[k]];
                l0[k] = p.last_old[blk[k]];
            }
        }
        int flag = 0, mine = 0;
#pragma unroll
        for (int k = 0; k < kScanItems; ++k) {
            if (blk[k] >= 0) {
                const int r = r0[k] + d0[k];
                if (r == 0 && l0[k] == base + tid * kScanItems + k) {
                    flag |= 1 << k;
                    ++mine;
                }
            }
        }
        int tot;
        int r = cta_exclusive_scan(mine, warp_sums, &tot);
#pragma unroll
        for (int k = 0; k < kScanItems; ++k)
            if (flag >> k & 1) p.ring[(head + count + freed + r++) % nb] = blk[k];
        freed += tot;
    }

    // ---- phase 3: blocks the new tokens take, and the copies
    int takes = 0, copies = 0;
    for (int base = 0; base < n_new; base += kThreads) {
        const int i = base + tid;
        int need = 0, copy = 0;
        if (i < n_new) {
            const int par = s_par[i];
            const int t = s_ctx[par];
            if (t % bs == 0) {
                need = 1;
            } else {
                const int o = tab(par * MB + t / bs);
                const int others = p.ref[o] + p.delta[o] - p.writers[o];
                copy = (others > 0 || p.last_writer[o] != i);
                need = copy;
            }
        }
        int tt, tc;
        cta_exclusive_scan(need, warp_sums, &tt);
        cta_exclusive_scan(copy, warp_sums, &tc);
        takes += tt;
        copies += tc;
    }
    __syncthreads();
    const bool ok = !s_bad && takes <= count + freed;

    // ---- phase 4: apply the net counts (each block once: whoever swaps its
    // delta out), reset the release marks
    for (int base = 0; base < old_entries; base += kThreads * kItems) {
        int blk[kItems];
        EntryWalk w(base + tid, MB);
#pragma unroll
        for (int k = 0; k < kItems; ++k) {
            const int e = base + k * kThreads + tid;
            blk[k] = -1;
            if (e < old_entries && w.pos < s_nb[w.j] && s_nch[w.j] != 1) blk[k] = tab(e);
            w.step(sdj, sdp, MB);
        }
        EntryWalk w2(base + tid, MB);
#pragma unroll
        for (int k = 0; k < kItems; ++k) {
            const int jk = w2.j;
            w2.step(sdj, sdp, MB);
            if (blk[k] >= 0) {
                const int b = blk[k];
                if (s_nch[jk] == 0) p.last_old[b] = -1;
                const int d = atomicExch(&p.delta[b], 0);
                if (ok && d) p.ref[b] += d;
            }
        }
    }
    __syncthreads();

    if (ok) {
        // ---- phase 5: the new tables (parent rows, -1 past the blocks in use)
        for (int base = 0; base < new_entries; base += kThreads * kItems) {
            int v[kItems];
            EntryWalk w(base + tid, MB);
#pragma unroll
            for (int k = 0; k < kItems; ++k) {
                const int e = base + k * kThreads + tid;
                v[k] = -1;
                if (e < new_entries) {
                    const int par = s_par[w.j];
                    if (w.pos < s_nb[par]) v[k] = tab(par * MB + w.pos);
                }
                w.step(sdj, sdp, MB);
            }
#pragma unroll
            for (int k = 0; k < kItems; ++k) {
                const int e = base + k * kThreads + tid;
                if (e < new_entries) q.new_tables[e] = v[k];
            }
        }
        __syncthreads();
        // ---- phase 6: takes, copies, slots
        int tk = 0, cp = 0;
        for (int base = 0; base < n_new; base += kThreads) {
            const int i = base + tid;
            int need = 0, copy = 0, o = -1, t = 0;
            if (i < n_new) {
                const int par = s_par[i];
                t = s_ctx[par];
                if (t % bs == 0) {
                    need = 1;
                } else {
                    o = tab(par * MB + t / bs);
                    copy = (p.ref[o] - p.writers[o] > 0 || p.last_writer[o] != i);
                    need = copy;
                }
            }
            int tt, tc;
            const int k = tk + cta_exclusive_scan(need, warp_sums, &tt);
            const int c = cp + cta_exclusive_scan(copy, warp_sums, &tc);
            tk += tt;
            cp += tc;
            if (i < n_new) {
                int b = o;
                if (need) {
                    b = policy == PA_POOL_FIFO ? p.ring[(head + k) % nb] : p.ring[(head + count + freed - 1 - k) % nb];
                    p.ref[b] = 1;
                    q.new_tables[i * MB + t / bs] = b;
                }
                if (copy) {
                    q.cow_pairs[2 * c] = o;
                    q.cow_pairs[2 * c + 1] = b;
                }
                q.slots[i] = b * bs + t % bs;
                q.new_ctx[i] = t + 1;
            }
        }
        __syncthreads();
        // a copying writer gives up its reference to the old block
        for (int i = tid; i < n_new; i += kThreads) {
            const int par = s_par[i];
            const int t = s_ctx[par];
            if (t % bs) {
                const int o = tab(par * MB + t / bs);
                if (q.new_tables[i * MB + t / bs] != o) atomicSub(&p.ref[o], 1);
            }
        }
    }
    __syncthreads();
    // ---- reset the writer marks; header and outputs
    for (int i = tid; i < n_new; i += kThreads) {
        const int par = s_par[i];
        const int t = s_ctx[par];
        if (t % bs) {
            const int o = tab(par * MB + t / bs);
            p.writers[o] = 0;
            p.last_writer[o] = -1;
        }
        if (!ok) q.slots[i] = -1;
    }
    if (tid == 0) {
        if (ok) {
            p.hdr[3] = policy == PA_POOL_FIFO ? (head + takes) % nb : head;
            p.hdr[4] = count + freed - takes;
            *q.num_cow = copies;
        } else {
            *q.num_cow = 0;
            record_error(q.err, s_bad ? (unsigned)s_bad : PA_DEVERR_POOL);
        }
    }
}

}  // namespace beam

cudaError_t launch_dpool_init(int32_t *state, int num_blocks, int block_size, int policy,
                              const int32_t *free_order, unsigned int *err, cudaStream_t stream) {
    int blocks = (num_blocks + 255) / 256;
    if (blocks > sm_count() * 8) blocks = sm_count() * 8;
    if (blocks < 1) blocks = 1;
    beam::dpool_fill_kernel<<<blocks, 256, 0, stream>>>(state, num_blocks, free_order);
    beam::dpool_seal_kernel<<<1, beam::kThreads, 0, stream>>>(state, num_blocks, block_size, policy,
                                                              free_order ? 1 : 0, err);
    return cudaGetLastError();
}

cudaError_t launch_dpool_load(int32_t *state, int num_blocks, int block_size, int policy, const int32_t *ref_counts,
                              const int32_t *free_list, int num_free, unsigned int *err, cudaStream_t stream) {
    beam::dpool_load_kernel<<<1, beam::kThreads, 0, stream>>>(state, num_blocks, block_size, policy, ref_counts,
                                                              free_list, num_free, err);
    return cudaGetLastError();
}

cudaError_t launch_beam_step(int32_t *state, const int32_t *old_tables, const int32_t *old_ctx, int num_old,
                             const int32_t *parents, int num_new, int32_t *new_tables, int32_t *new_ctx,
                             int max_blocks, int32_t *slots, int64_t *cow_pairs, int32_t *num_cow,
                             int num_blocks, int block_size, unsigned int *err, cudaStream_t stream) {
    beam::StepParams q;
    q.state = state;
    q.old_tables = old_tables;
    q.old_ctx = old_ctx;
    q.parents = parents;
    q.new_tables = new_tables;
    q.new_ctx = new_ctx;
    q.slots = slots;
    q.cow_pairs = cow_pairs;
    q.num_cow = num_cow;
    q.num_old = num_old;
    q.num_new = num_new;
    q.max_blocks = max_blocks;
    q.num_blocks = num_blocks;
    q.block_size = block_size;
    q.err = err;
    const long long base = (3LL * num_old + num_new) * (long long)sizeof(int);
    const long long with_tables = base + (long long)num_old * max_blocks * (long long)sizeof(int);
    static AttrCache attr_done[2];
    cudaError_t e;
    if (with_tables <= beam::kMaxDynBytes) {
        e = ensure_smem_attr(reinterpret_cast<const void *>(beam::beam_step_kernel<true>), beam::kMaxDynBytes,
                             &attr_done[1]);
        if (e != cudaSuccess) return e;
        beam::beam_step_kernel<true><<<1, beam::kThreads, (int)with_tables, stream>>>(q);
    } else {
        e = ensure_smem_attr(reinterpret_cast<const void *>(beam::beam_step_kernel<false>), beam::kMaxStageBytes,
                             &attr_done[0]);
        if (e != cudaSuccess) return e;
        beam::beam_step_kernel<false><<<1, beam::kThreads, (int)base, stream>>>(q);
    }
    return cudaGetLastError();
}

}  // namespace pa
