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
// The launches below reach that sequential result in parallel:
//   * counts: net change per block accumulated with atomics in a scratch
//     array, applied once;
//   * free-list order: a block is freed at its last decrement, the largest
//     flattened (beam, table position) index holding it; per-chunk totals and
//     a scan within each chunk give each freed block its place;
//   * copy-on-write: writer i into block b finds count > 1 unless it is the
//     last writer into b (largest i) and no other new beam holds b, so
//     copies = (not last writer) or (other holders > 0);
//   * takes: a scan of "needs a block" in beam order gives each writer its
//     position in the free list (front for FIFO, back for LIFO).
// Everything is checked before anything changes: on an error the state is
// unchanged, every slot is -1 and the copy count is 0.
#include <algorithm>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {
namespace beam {

constexpr int kThreads = 1024;     // pool set-up kernels
// per-beam values staged in shared memory by each CTA of the step: 3 words
// per old beam, 1 per new beam
constexpr int kMaxStageBytes = PA_BEAM_MAX_STAGED * 4;
constexpr int32_t kMagic = 0x50414250;

struct Pool {
    int32_t *hdr, *ref, *ring, *delta, *last_old, *writers, *last_writer, *tail;
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
    p.tail = p.last_writer + nb;
    return p;
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
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < PA_DPOOL_TAIL_WORDS; i += gridDim.x * blockDim.x)
        p.tail[i] = 0;
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
    for (int i = threadIdx.x; i < PA_DPOOL_TAIL_WORDS; i += kThreads) p.tail[i] = 0;
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
    int chunk;       // old-table entries per CTA
    int num_chunks;  // CTAs of each launch
    unsigned int *err;
};

// ------------------------------------------------------------------ beam step
//
// Four launches over chunks of the old tables' entries (flattened (beam,
// position) index e = j * max_blocks + pos), so that the passes over the
// tables and their atomics spread over the SMs; a kernel boundary is the
// only grid-wide ordering used. Every CTA first stages the per-beam values
// (context length, block count, number of children, parent) in shared
// memory and makes the same argument checks, so all CTAs agree on them
// without a global exchange. Between launches the step keeps a status word
// and per-chunk totals in the state's tail.
//   1. count:  validate each entry in use (block id in range, count > 0);
//              delta[b] += children - 1 for beams without exactly one
//              child; last_old[b] = max e over beams with no child; count
//              the writers into each block (writers, last_writer).
//   2. flags:  an entry frees its block if the block's count reaches 0 and
//              it is the block's last release (last_old[b] == e); per-chunk
//              totals of such entries; blocks whose count stays above 0 get
//              last_old = -2 so that later tests need no count. CTA 0 also
//              totals the blocks the new tokens take.
//   3. apply:  freed blocks go to the back of the free list in entry order
//              (chunk prefix + rank within the chunk); counts take their net
//              change; the new tables get their parents' rows (except the
//              entry each new beam writes into).
//   4. finish: CTA 0 decides, in beam order, the block each new token takes
//              and the copies (scans over the new beams), writes slots,
//              context lengths and pairs, updates the header and clears the
//              status; every CTA clears the release marks of its chunk.
// Everything that changes the pool happens in launch 3 and 4, and only if
// launches 1 and 2 found nothing wrong (status 0) and the free list is long
// enough; otherwise the pool is left as it was, every slot is -1 and the
// copy count is 0.

constexpr int kStepThreads = 256;
constexpr int kMaxChunks = PA_DPOOL_TAIL_WORDS - 4;
// tail words: [0] status bits of this step, [1] blocks taken, [2] copies,
// [4 + c] freed blocks in chunk c

struct Staged {
    int *ctx, *nblk, *nch, *par;
    int bad;  // PA_DEVERR_* bits of the checks every CTA makes alike
};

__device__ __forceinline__ int nblk(int ctx, int bs) { return (ctx + bs - 1) / bs; }

// Stages the per-beam values and checks the header, contexts and parents.
__device__ Staged stage_beams(const StepParams &q, const Pool &p, int *dyn, int *s_bad) {
    Staged st;
    const int n_old = q.num_old, n_new = q.num_new, bs = q.block_size, MB = q.max_blocks;
    st.ctx = dyn;
    st.nblk = dyn + n_old;
    st.nch = dyn + 2 * n_old;
    st.par = dyn + 3 * n_old;
    if (threadIdx.x == 0) {
        *s_bad = 0;
        const int count = p.hdr[4], head = p.hdr[3];
        if (p.hdr[5] != kMagic || p.hdr[0] != q.num_blocks || p.hdr[1] != bs || count < 0 ||
            count > q.num_blocks || head < 0 || head >= q.num_blocks)
            *s_bad = PA_DEVERR_POOL;
    }
    for (int j = threadIdx.x; j < n_old; j += kStepThreads) {
        const int c = __ldg(q.old_ctx + j);
        st.ctx[j] = c;
        st.nblk[j] = c < 0 ? 0 : nblk(c, bs);
        st.nch[j] = 0;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < n_old; j += kStepThreads)
        if (st.ctx[j] < 0 || st.nblk[j] > MB) atomicOr(s_bad, PA_DEVERR_CONTEXT);
    for (int i = threadIdx.x; i < n_new; i += kStepThreads) {
        const int par = __ldg(q.parents + i);
        st.par[i] = par;
        if (par < 0 || par >= n_old) {
            atomicOr(s_bad, PA_DEVERR_CONTEXT);
        } else {
            atomicAdd(&st.nch[par], 1);
            if (st.ctx[par] >= 0 && st.ctx[par] / bs >= MB) atomicOr(s_bad, PA_DEVERR_POOL);  // no room
        }
    }
    __syncthreads();
    st.bad = *s_bad;
    return st;
}

// This CTA's chunk of old-table entries: [e0, e1).
__device__ __forceinline__ void chunk_of(const StepParams &q, int *e0, int *e1) {
    const long long entries = (long long)q.num_old * q.max_blocks;
    const long long b = (long long)blockIdx.x * q.chunk;
    *e0 = (int)min(b, entries);
    *e1 = (int)min(b + q.chunk, entries);
}

__device__ __forceinline__ volatile int *status_word(const Pool &p) { return p.tail; }

// Programmatic dependent launch: launches 2-4 start while the previous one
// runs (each stages the per-beam values, which no launch writes) and wait
// for it to finish, its writes visible, before they read its results. Both
// are no-ops for a launch made without the attribute.
__device__ __forceinline__ void allow_next_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void wait_previous_launch() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__global__ void __launch_bounds__(kStepThreads) beam_count_kernel(const StepParams q) {
    extern __shared__ int dyn[];
    __shared__ int s_bad;
    allow_next_launch();
    const Pool p = views(q.state, q.num_blocks);
    const Staged st = stage_beams(q, p, dyn, &s_bad);
    if (st.bad) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(p.tail, st.bad);
        return;
    }
    const int MB = q.max_blocks, nb = q.num_blocks, bs = q.block_size;
    int e0, e1;
    chunk_of(q, &e0, &e1);
    for (int e = e0 + threadIdx.x; e < e1; e += kStepThreads) {
        const int j = e / MB, pos = e - j * MB;
        if (pos >= st.nblk[j]) continue;
        const int b = __ldg(q.old_tables + e);
        if (b < 0 || b >= nb || p.ref[b] <= 0) {
            atomicOr(p.tail, PA_DEVERR_BLOCK_ID);
            continue;
        }
        const int n = st.nch[j];
        if (n != 1) atomicAdd(&p.delta[b], n - 1);
        if (n == 0) atomicMax(&p.last_old[b], e);
    }
    for (int i = blockIdx.x * kStepThreads + threadIdx.x; i < q.num_new; i += gridDim.x * kStepThreads) {
        const int par = st.par[i];
        const int t = st.ctx[par];
        if (t % bs) {
            const int o = __ldg(q.old_tables + par * MB + t / bs);
            if (o >= 0 && o < nb) {
                atomicAdd(&p.writers[o], 1);
                atomicMax(&p.last_writer[o], i);
            }
        }
    }
}

// Block-wide sum over kStepThreads threads (ends with a barrier).
__device__ __forceinline__ int cta_sum(int v, int *warp_sums) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
    if (lane == 0) warp_sums[warp] = v;
    __syncthreads();
    int t = 0;
#pragma unroll
    for (int w = 0; w < kStepThreads / 32; ++w) t += warp_sums[w];
    __syncthreads();
    return t;
}

// Exclusive scan over kStepThreads threads; *total receives the sum (ends with a barrier).
__device__ __forceinline__ int cta_scan(int v, int *warp_sums, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, d);
        if (lane >= d) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    int before = 0, t = 0;
#pragma unroll
    for (int w = 0; w < kStepThreads / 32; ++w) {
        if (w < warp) before += warp_sums[w];
        t += warp_sums[w];
    }
    __syncthreads();
    *total = t;
    return x - v + before;
}

// Whether new beam i needs a block and whether it copies (counts as the
// sequential order sees them when the new tokens are written: after every
// fork and release). `applied`: the net changes are already in ref.
__device__ __forceinline__ void take_and_copy(const StepParams &q, const Pool &p, const Staged &st, int i,
                                              bool applied, int *need, int *copy, int *o, int *t) {
    const int par = st.par[i];
    *t = st.ctx[par];
    *need = 0;
    *copy = 0;
    *o = -1;
    if (*t % q.block_size == 0) {
        *need = 1;
    } else {
        *o = __ldg(q.old_tables + par * q.max_blocks + *t / q.block_size);
        const int r = applied ? p.ref[*o] : p.ref[*o] + p.delta[*o];
        *copy = (r - p.writers[*o] > 0 || p.last_writer[*o] != i);
        *need = *copy;
    }
}

__global__ void __launch_bounds__(kStepThreads) beam_flags_kernel(const StepParams q) {
    extern __shared__ int dyn[];
    __shared__ int s_bad;
    __shared__ int warp_sums[kStepThreads / 32];
    allow_next_launch();
    const Pool p = views(q.state, q.num_blocks);
    const Staged st = stage_beams(q, p, dyn, &s_bad);
    wait_previous_launch();  // from here on: the previous launch's results
    const bool bad = st.bad || *status_word(p) != 0;
    const int MB = q.max_blocks;
    int e0, e1;
    chunk_of(q, &e0, &e1);
    int cnt = 0;
    if (!bad) {
        for (int e = e0 + threadIdx.x; e < e1; e += kStepThreads) {
            const int j = e / MB, pos = e - j * MB;
            if (pos >= st.nblk[j] || st.nch[j] != 0) continue;
            const int b = __ldg(q.old_tables + e);
            const int r = p.ref[b] + p.delta[b];
            if (r < 0) {
                atomicOr(p.tail, PA_DEVERR_POOL);  // a table holds a block more often than counted
            } else if (r > 0) {
                p.last_old[b] = -2;  // not freed (every entry of b sees the same r)
            } else if (p.last_old[b] == e) {
                ++cnt;
            }
        }
    }
    cnt = cta_sum(cnt, warp_sums);
    if (threadIdx.x == 0) p.tail[4 + blockIdx.x] = cnt;
    if (blockIdx.x == 0) {
        int takes = 0, copies = 0;
        if (!bad) {
            for (int base = 0; base < q.num_new; base += kStepThreads) {
                const int i = base + threadIdx.x;
                int need = 0, copy = 0, o, t;
                if (i < q.num_new) take_and_copy(q, p, st, i, false, &need, &copy, &o, &t);
                takes += need;
                copies += copy;
            }
        }
        takes = cta_sum(takes, warp_sums);
        copies = cta_sum(copies, warp_sums);
        if (threadIdx.x == 0) {
            p.tail[1] = takes;
            p.tail[2] = copies;
        }
    }
}

__global__ void __launch_bounds__(kStepThreads) beam_apply_kernel(const StepParams q) {
    extern __shared__ int dyn[];
    __shared__ int s_bad;
    __shared__ int warp_sums[kStepThreads / 32];
    allow_next_launch();
    const Pool p = views(q.state, q.num_blocks);
    const Staged st = stage_beams(q, p, dyn, &s_bad);
    wait_previous_launch();  // from here on: the previous launch's results
    const int MB = q.max_blocks, nb = q.num_blocks, bs = q.block_size;
    const int head = p.hdr[3], count = p.hdr[4];
    // freed blocks in all chunks and in the chunks before this one
    int before = 0, freed = 0;
    for (int c = threadIdx.x; c < (int)gridDim.x; c += kStepThreads) {
        const int v = p.tail[4 + c];
        freed += v;
        if (c < (int)blockIdx.x) before += v;
    }
    freed = cta_sum(freed, warp_sums);
    before = cta_sum(before, warp_sums);
    const int status = *status_word(p);  // final: launches 1 and 2 are done, this one adds nothing
    const bool ok = !st.bad && status == 0 && p.tail[1] <= count + freed;
    int e0, e1;
    chunk_of(q, &e0, &e1);
    if (!st.bad && status == 0) {  // every entry in use holds a valid block id
        // freed blocks, in entry order: each thread takes a contiguous run of the chunk
        const int per = (q.chunk + kStepThreads - 1) / kStepThreads;
        const int a0 = min(e1, e0 + threadIdx.x * per), a1 = min(e1, a0 + per);
        int mine = 0;
        for (int e = a0; e < a1; ++e) {
            const int j = e / MB, pos = e - j * MB;
            if (pos < st.nblk[j] && st.nch[j] == 0 && p.last_old[__ldg(q.old_tables + e)] == e) ++mine;
        }
        int tot;
        int r = cta_scan(mine, warp_sums, &tot);
        if (ok && mine) {
            for (int e = a0; e < a1; ++e) {
                const int j = e / MB, pos = e - j * MB;
                if (pos >= st.nblk[j] || st.nch[j] != 0) continue;
                const int b = __ldg(q.old_tables + e);
                if (p.last_old[b] == e) p.ring[(head + count + before + r++) % nb] = b;
            }
        }
    }
    if (!st.bad) {  // (with st.bad set, launch 1 changed nothing)
        // net count changes (each block once: whoever swaps its delta out);
        // every delta goes back to 0 whatever the outcome
        for (int e = e0 + threadIdx.x; e < e1; e += kStepThreads) {
            const int j = e / MB, pos = e - j * MB;
            if (pos >= st.nblk[j] || st.nch[j] == 1) continue;
            const int b = __ldg(q.old_tables + e);
            if (b < 0 || b >= nb) continue;
            const int d = atomicExch(&p.delta[b], 0);
            if (ok && d) p.ref[b] += d;
        }
    }
    if (ok) {  // the new tables: parents' rows, -1 past them; each beam's write entry is left to launch 4
        const long long new_entries = (long long)q.num_new * MB;
        for (long long e = (long long)blockIdx.x * kStepThreads + threadIdx.x; e < new_entries;
             e += (long long)gridDim.x * kStepThreads) {
            const int i = (int)(e / MB), pos = (int)(e - (long long)i * MB);
            const int par = st.par[i];
            if (pos == st.ctx[par] / bs) continue;
            q.new_tables[e] = pos < st.nblk[par] ? __ldg(q.old_tables + par * MB + pos) : -1;
        }
    }
}

__global__ void __launch_bounds__(kStepThreads) beam_finish_kernel(const StepParams q) {
    extern __shared__ int dyn[];
    __shared__ int s_bad;
    __shared__ int warp_sums[kStepThreads / 32];
    const Pool p = views(q.state, q.num_blocks);
    const Staged st = stage_beams(q, p, dyn, &s_bad);
    wait_previous_launch();  // from here on: the previous launch's results
    const int MB = q.max_blocks, nb = q.num_blocks, bs = q.block_size;
    if (blockIdx.x == 0) {
        const int policy = p.hdr[2], head = p.hdr[3], count = p.hdr[4];
        int freed = 0;
        for (int c = threadIdx.x; c < q.num_chunks; c += kStepThreads) freed += p.tail[4 + c];
        freed = cta_sum(freed, warp_sums);
        const int status = *status_word(p);
        const int takes = p.tail[1];
        const bool ok = !st.bad && status == 0 && takes <= count + freed;
        if (ok) {
            int tk = 0, cp = 0;
            for (int base = 0; base < q.num_new; base += kStepThreads) {
                const int i = base + threadIdx.x;
                int need = 0, copy = 0, o = -1, t = 0;
                if (i < q.num_new) take_and_copy(q, p, st, i, true, &need, &copy, &o, &t);
                int tt, tc;
                const int k = tk + cta_scan(need, warp_sums, &tt);
                const int c = cp + cta_scan(copy, warp_sums, &tc);
                tk += tt;
                cp += tc;
                if (i < q.num_new) {
                    int b = o;
                    if (need) {
                        b = policy == PA_POOL_FIFO ? p.ring[(head + k) % nb] : p.ring[(head + count + freed - 1 - k) % nb];
                        p.ref[b] = 1;
                    }
                    q.new_tables[(long long)i * MB + t / bs] = b;
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
            for (int i = threadIdx.x; i < q.num_new; i += kStepThreads) {
                const int par = st.par[i];
                const int t = st.ctx[par];
                if (t % bs) {
                    const int o = __ldg(q.old_tables + par * MB + t / bs);
                    if (q.new_tables[(long long)i * MB + t / bs] != o) atomicSub(&p.ref[o], 1);
                }
            }
        }
        __syncthreads();
        // reset the writer marks; outputs of a failed step
        if (!st.bad) {
            for (int i = threadIdx.x; i < q.num_new; i += kStepThreads) {
                const int par = st.par[i];
                const int t = st.ctx[par];
                if (t % bs) {
                    const int o = __ldg(q.old_tables + par * MB + t / bs);
                    if (o >= 0 && o < nb) {
                        p.writers[o] = 0;
                        p.last_writer[o] = -1;
                    }
                }
            }
        }
        if (!ok)
            for (int i = threadIdx.x; i < q.num_new; i += kStepThreads) q.slots[i] = -1;
        if (threadIdx.x == 0) {
            if (ok) {
                p.hdr[3] = policy == PA_POOL_FIFO ? (head + takes) % nb : head;
                p.hdr[4] = count + freed - takes;
                *q.num_cow = p.tail[2];
            } else {
                *q.num_cow = 0;
                const int bits = st.bad | status;
                record_error(q.err, bits ? (unsigned)bits : PA_DEVERR_POOL);
            }
        }
        __syncthreads();  // every thread has read the totals: the step scratch goes back to zero
        for (int i = threadIdx.x; i < 4 + q.num_chunks; i += kStepThreads) p.tail[i] = 0;
    }
    // every CTA: clear the release marks of its chunk
    if (!st.bad) {
        int e0, e1;
        chunk_of(q, &e0, &e1);
        for (int e = e0 + threadIdx.x; e < e1; e += kStepThreads) {
            const int j = e / MB, pos = e - j * MB;
            if (pos >= st.nblk[j] || st.nch[j] != 0) continue;
            const int b = __ldg(q.old_tables + e);
            if (b >= 0 && b < nb) p.last_old[b] = -1;
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
    // chunks of at least one entry per thread, at most kMaxChunks of them
    const long long entries = (long long)num_old * max_blocks;
    long long chunk = beam::kStepThreads;
    while ((entries + chunk - 1) / chunk > beam::kMaxChunks) chunk += beam::kStepThreads;
    q.chunk = (int)chunk;
    q.num_chunks = (int)std::max(1LL, (entries + chunk - 1) / chunk);
    const int smem = (3 * num_old + num_new) * (int)sizeof(int);
    static AttrCache attr_done[4];
    const void *kernels[4] = {reinterpret_cast<const void *>(beam::beam_count_kernel),
                              reinterpret_cast<const void *>(beam::beam_flags_kernel),
                              reinterpret_cast<const void *>(beam::beam_apply_kernel),
                              reinterpret_cast<const void *>(beam::beam_finish_kernel)};
    for (int k = 0; k < 4; ++k) {
        cudaError_t e = ensure_smem_attr(kernels[k], beam::kMaxStageBytes, &attr_done[k]);
        if (e != cudaSuccess) return e;
    }
    const dim3 grid(q.num_chunks), block(beam::kStepThreads);
    beam::beam_count_kernel<<<grid, block, smem, stream>>>(q);  // after all earlier work on the stream
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, beam::beam_flags_kernel, q);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, beam::beam_apply_kernel, q);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, beam::beam_finish_kernel, q);
    return e;
}

}  // namespace pa
