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
    // test hook (pa_beam_step_withhold_arrival; the one-launch form's hook
    // instance only): CTA withhold_cta never arrives at the first grid
    // barrier, and barrier waits give up after barrier_limit_ns
    int withhold_cta = -1;
    unsigned long long barrier_limit_ns = 0;
};

// ------------------------------------------------------------------ beam step
//
// Four phases over chunks of the old tables' entries (flattened (beam,
// position) index e = j * max_blocks + pos), so that the passes over the
// tables and their atomics spread over the SMs. They run as one cooperative
// launch with a grid barrier between phases (at most one CTA per SM, all
// resident at once), or, where a cooperative launch is refused, as four
// launches whose boundaries order them. Every CTA first stages the per-beam values
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
constexpr int kMaxChunks = PA_DPOOL_TAIL_WORDS - 10;  // tail: 4 words, chunk totals, the one-launch words
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
    // contexts and parents are independent loads: one round trip for both
    for (int j = threadIdx.x; j < n_old; j += kStepThreads) {
        const int c = __ldg(q.old_ctx + j);
        st.ctx[j] = c;
        st.nblk[j] = c < 0 ? 0 : nblk(c, bs);
        st.nch[j] = 0;
    }
    for (int i = threadIdx.x; i < n_new; i += kStepThreads) st.par[i] = __ldg(q.parents + i);
    __syncthreads();
    for (int j = threadIdx.x; j < n_old; j += kStepThreads)
        if (st.ctx[j] < 0 || st.nblk[j] > MB) atomicOr(s_bad, PA_DEVERR_CONTEXT);
    for (int i = threadIdx.x; i < n_new; i += kStepThreads) {
        const int par = st.par[i];
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

// ---- phase 1 (count)
__device__ void phase_count(const StepParams &q, const Pool &p, const Staged &st) {
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

// ---- phase 2 (flags)
__device__ void phase_flags(const StepParams &q, const Pool &p, const Staged &st, int *warp_sums) {
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

// ---- phase 3 (apply)
__device__ void phase_apply(const StepParams &q, const Pool &p, const Staged &st, int *warp_sums) {
    const int MB = q.max_blocks, nb = q.num_blocks, bs = q.block_size;
    const int head = p.hdr[3], count = p.hdr[4];
    // freed blocks in all chunks and in the chunks before this one
    int before = 0, freed = 0;
    for (int c = threadIdx.x; c < q.num_chunks; c += kStepThreads) {
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

// ---- phase 4 (finish)
__device__ void phase_finish(const StepParams &q, const Pool &p, const Staged &st, int *warp_sums) {
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


// ---- the four phases as four launches (launches 2-4 by programmatic
// dependent launch)

__global__ void __launch_bounds__(kStepThreads) beam_count_kernel(const StepParams q) {
    extern __shared__ int dyn[];
    __shared__ int s_bad;
    allow_next_launch();
    const Pool p = views(q.state, q.num_blocks);
    const Staged st = stage_beams(q, p, dyn, &s_bad);
    phase_count(q, p, st);
}

#define PA_BEAM_PHASE_KERNEL(NAME, PHASE, ALLOW_NEXT)                                    \
    __global__ void __launch_bounds__(kStepThreads) NAME(const StepParams q) {           \
        extern __shared__ int dyn[];                                                     \
        __shared__ int s_bad;                                                            \
        __shared__ int warp_sums[kStepThreads / 32];                                     \
        if (ALLOW_NEXT) allow_next_launch();                                             \
        const Pool p = views(q.state, q.num_blocks);                                     \
        const Staged st = stage_beams(q, p, dyn, &s_bad);                                \
        wait_previous_launch(); /* from here on: the previous launch's results */        \
        PHASE(q, p, st, warp_sums);                                                      \
    }
PA_BEAM_PHASE_KERNEL(beam_flags_kernel, phase_flags, true)
PA_BEAM_PHASE_KERNEL(beam_apply_kernel, phase_apply, true)
PA_BEAM_PHASE_KERNEL(beam_finish_kernel, phase_finish, false)
#undef PA_BEAM_PHASE_KERNEL

// ---- the four phases in one cooperative launch: every CTA is resident at
// once (the launch guarantees it, or fails), so a CTA may wait for the others
// at a grid barrier between phases. Barrier and exit counters live in the
// pool's tail; each wait is bounded (a CTA that gives up records
// PA_DEVERR_TIMEOUT and the step stops; with every CTA resident that does
// not happen).

// Words of the one-launch form: a status word per epoch parity (the step's
// PA_DEVERR bits; each step clears the next step's), the grid barrier's
// arrival count (it only grows: barrier k of a step waits for base + k * CTAs
// arrivals, base kept in header word 7), and the epoch + 1 of a step whose
// barrier wait gave up. Header word 6 counts the steps (the epoch).
constexpr int kFusedStatus = PA_DPOOL_TAIL_WORDS - 6;  // and - 5
constexpr int kBarArrive = PA_DPOOL_TAIL_WORDS - 3;
constexpr int kBarAbort = PA_DPOOL_TAIL_WORDS - 2;
constexpr uint64_t kBarrierLimitNs = 200ull * 1000ull * 1000ull;  // 200 ms

__device__ __forceinline__ int ld_acquire(const int *a) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
    return v;
}

// Grid barrier: true once `target` arrivals are counted. A wait that gives
// up (or sees that another CTA gave up) leaves the pool unusable: the step
// stopped part way, and later steps refuse the state (PA_DEVERR_POOL).
// limit_ns: the wait bound; arrive false (test hook only): this CTA does not
// count itself.
__device__ bool grid_barrier(const Pool &p, unsigned target, int epoch, unsigned int *err, int *s_go,
                             uint64_t limit_ns = kBarrierLimitNs, bool arrive = true) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();  // this CTA's writes, before its arrival
        if (arrive) atomicAdd(reinterpret_cast<unsigned *>(&p.tail[kBarArrive]), 1u);
        bool ok = true;
        uint64_t t0 = 0;
        for (uint32_t it = 0; (int)((unsigned)ld_acquire(&p.tail[kBarArrive]) - target) < 0; ++it) {
            if ((it & 63u) != 63u) continue;
            if (ld_acquire(&p.tail[kBarAbort]) == epoch + 1) { ok = false; break; }
            const uint64_t t = global_ns();
            if (t0 == 0) t0 = t;
            else if (t - t0 > limit_ns) {
                atomicExch(&p.tail[kBarAbort], epoch + 1);
                p.hdr[5] = 0;
                record_error(err, PA_DEVERR_TIMEOUT);
                ok = false;
                break;
            }
        }
        __threadfence();
        *s_go = ok;
    }
    __syncthreads();
    return *s_go != 0;
}

// Entries of the old tables (contiguous, per thread) and new beams (one per
// thread per round) the fused kernel keeps in registers across its phases.
constexpr int kFusedEntries = 4;
constexpr int kFusedBeams = 4;

template <bool kHook>
__global__ void __launch_bounds__(kStepThreads) beam_step_kernel(const StepParams q) {
    extern __shared__ int dyn[];
    __shared__ int s_bad, s_go;
    __shared__ int warp_sums[kStepThreads / 32];
    const Pool p = views(q.state, q.num_blocks);
    const int MB = q.max_blocks, nb = q.num_blocks, bs = q.block_size;
    const int tid = threadIdx.x;
    const unsigned G = gridDim.x;
    // the header as it stands before the step (only CTA 0 changes it, after
    // every CTA has passed the first barrier)
    const int policy = p.hdr[2], head = p.hdr[3], count = p.hdr[4];
    const int epoch = p.hdr[6];
    const unsigned base = (unsigned)p.hdr[7];
    int *status = p.tail + kFusedStatus + (epoch & 1);
    if (blockIdx.x == 0 && tid == 0) p.tail[kFusedStatus + ((epoch + 1) & 1)] = 0;  // the next step's
    const Staged st = stage_beams(q, p, dyn, &s_bad);

    // ---- phase 1: this thread's entries (contiguous run of the chunk):
    // validate, net count change, last release; writers per block
    int e0, e1;
    chunk_of(q, &e0, &e1);
    const int per = q.chunk / kStepThreads;  // <= kFusedEntries (host check)
    const int ea = e0 + tid * per;
    // eb: block id of entry k; ev: in use and valid (only such entries are
    // ever acted on); ench: children of its beam; eref: its count before the step
    int eb[kFusedEntries], eref[kFusedEntries], ench[kFusedEntries];
    bool euse[kFusedEntries], ev[kFusedEntries], efree[kFusedEntries];
#pragma unroll
    for (int k = 0; k < kFusedEntries; ++k) {
        eb[k] = -1;
        ench[k] = 1;
        euse[k] = ev[k] = efree[k] = false;
        const int e = ea + k;
        if (!st.bad && k < per && e < e1) {
            const int j = e / MB, pos = e - j * MB;
            if (pos < st.nblk[j]) {
                eb[k] = __ldg(q.old_tables + e);
                ench[k] = st.nch[j];
                euse[k] = true;
            }
        }
    }
    // new beam i = round * 256 + tid: CTA 0 keeps its old block (-1 at a block
    // boundary) and context for phases 2-3
    int bo[kFusedBeams], bt[kFusedBeams];
#pragma unroll
    for (int r = 0; r < kFusedBeams; ++r) {
        bo[r] = -1;
        bt[r] = 0;
        const int i = r * kStepThreads + tid;
        if (blockIdx.x == 0 && !st.bad && i < q.num_new) {
            bt[r] = st.ctx[st.par[i]];
            if (bt[r] % bs) bo[r] = __ldg(q.old_tables + st.par[i] * MB + bt[r] / bs);
        }
    }
#pragma unroll
    for (int k = 0; k < kFusedEntries; ++k)
        if (euse[k] && eb[k] >= 0 && eb[k] < nb) eref[k] = p.ref[eb[k]];
#pragma unroll
    for (int k = 0; k < kFusedEntries; ++k) {
        if (!euse[k]) continue;
        const int b = eb[k];
        if (b < 0 || b >= nb || eref[k] <= 0) {
            atomicOr(status, PA_DEVERR_BLOCK_ID);
            continue;
        }
        ev[k] = true;
        if (ench[k] != 1) atomicAdd(&p.delta[b], ench[k] - 1);
        if (ench[k] == 0) atomicMax(&p.last_old[b], ea + k);
    }
    if (blockIdx.x == 0) {
#pragma unroll
        for (int r = 0; r < kFusedBeams; ++r) {
            const int o = bo[r];
            if (o >= 0 && o < nb) {
                atomicAdd(&p.writers[o], 1);
                atomicMax(&p.last_writer[o], r * kStepThreads + tid);
            }
        }
        if (tid == 0 && st.bad) atomicOr(status, st.bad);
    }

    // (hook instance: the bound given, and one CTA that never arrives here)
    const uint64_t blim = kHook && q.barrier_limit_ns ? q.barrier_limit_ns : kBarrierLimitNs;
    bool go = grid_barrier(p, base + G, epoch, q.err, &s_go, blim, !(kHook && (int)blockIdx.x == q.withhold_cta));
    // ---- phase 2: which entries free their block (count reaches 0 at its last
    // release); per-chunk totals; CTA 0 decides each new beam's take and copy.
    // Every load of the phase is issued before the status is tested.
    int bk[kFusedBeams], bc[kFusedBeams];  // CTA 0: take index, copy index (-1: none)
    int takes = 0, copies = 0;
    {
        int dl[kFusedEntries], lo[kFusedEntries];
#pragma unroll
        for (int k = 0; k < kFusedEntries; ++k)
            if (ev[k] && ench[k] == 0) {
                dl[k] = p.delta[eb[k]];
                lo[k] = p.last_old[eb[k]];
            }
        int rr[kFusedBeams], wr[kFusedBeams], lw[kFusedBeams];
        if (blockIdx.x == 0) {
#pragma unroll
            for (int r = 0; r < kFusedBeams; ++r)
                if (bo[r] >= 0 && bo[r] < nb) {
                    rr[r] = p.ref[bo[r]] + p.delta[bo[r]];
                    wr[r] = p.writers[bo[r]];
                    lw[r] = p.last_writer[bo[r]];
                }
        }
        const bool bad2 = !go || st.bad || ld_acquire(status) != 0;
        int cnt = 0;
#pragma unroll
        for (int k = 0; k < kFusedEntries; ++k)
            if (!bad2 && ev[k] && ench[k] == 0) {
                const int r = eref[k] + dl[k];
                if (r < 0) atomicOr(status, PA_DEVERR_POOL);  // a table holds a block more often than counted
                efree[k] = r == 0 && lo[k] == ea + k;
                cnt += efree[k];
            }
        cnt = cta_sum(cnt, warp_sums);
        if (tid == 0) p.tail[4 + blockIdx.x] = cnt;
        if (blockIdx.x == 0) {
#pragma unroll
            for (int r = 0; r < kFusedBeams; ++r) {
                const int i = r * kStepThreads + tid;
                int need = 0, copy = 0;
                if (!bad2 && i < q.num_new) {
                    if (bo[r] < 0) {
                        need = 1;
                    } else {
                        copy = rr[r] - wr[r] > 0 || lw[r] != i;
                        need = copy;
                    }
                }
                int tt, tc;
                const int k = takes + cta_scan(need, warp_sums, &tt);
                const int c = copies + cta_scan(copy, warp_sums, &tc);
                bk[r] = need ? k : -1;
                bc[r] = copy ? c : -1;
                takes += tt;
                copies += tc;
            }
            if (tid == 0) {
                p.tail[1] = takes;
                p.tail[2] = copies;
            }
        }
    }

    go = grid_barrier(p, base + 2 * G, epoch, q.err, &s_go, blim) && go;
    // ---- phase 3: apply. Deltas are swapped out first (their values are
    // needed only once the outcome is known), then freed blocks go to the
    // back of the free list in entry order, counts take their net change, the
    // new tables get their parents' rows; CTA 0 the takes (from the free
    // list's front: FIFO with enough free blocks) or, otherwise, after one
    // more barrier
    int dx[kFusedEntries];
#pragma unroll
    for (int k = 0; k < kFusedEntries; ++k) {
        dx[k] = 0;
        if (ev[k] && ench[k] != 1) dx[k] = atomicExch(&p.delta[eb[k]], 0);
    }
    int freed = 0, before = 0;
    for (int c = tid; c < q.num_chunks; c += kStepThreads) {
        const int v = p.tail[4 + c];
        freed += v;
        if (c < (int)blockIdx.x) before += v;
    }
    takes = p.tail[1];
    copies = p.tail[2];
    const int bits = ld_acquire(status);
    freed = cta_sum(freed, warp_sums);
    before = cta_sum(before, warp_sums);
    const bool ok = go && !st.bad && bits == 0 && takes <= count + freed;
    {
        int mine = 0;
#pragma unroll
        for (int k = 0; k < kFusedEntries; ++k) mine += efree[k];
        int tot;
        int r = before + cta_scan(mine, warp_sums, &tot);
#pragma unroll
        for (int k = 0; k < kFusedEntries; ++k)
            if (ok && efree[k]) p.ring[(head + count + r++) % nb] = eb[k];
    }
#pragma unroll
    for (int k = 0; k < kFusedEntries; ++k) {
        if (ok && dx[k]) atomicAdd(&p.ref[eb[k]], dx[k]);
        if (ev[k] && ench[k] == 0) p.last_old[eb[k]] = -1;
    }
    if (ok) {  // the new tables: parents' rows, -1 past them; each beam's write entry is CTA 0's
        const long long new_entries = (long long)q.num_new * MB;
        for (long long e = (long long)blockIdx.x * kStepThreads + tid; e < new_entries;
             e += (long long)G * kStepThreads) {
            const int i = (int)(e / MB), pos = (int)(e - (long long)i * MB);
            const int par = st.par[i];
            if (pos == st.ctx[par] / bs) continue;
            q.new_tables[e] = pos < st.nblk[par] ? __ldg(q.old_tables + par * MB + pos) : -1;
        }
    }
    const bool early = policy == PA_POOL_FIFO && takes <= count;  // the same in every CTA
    if (!early) go = grid_barrier(p, base + 3 * G, epoch, q.err, &s_go, blim) && go;  // the freed blocks are listed
    if (blockIdx.x == 0) {
        const bool ok4 = ok && go;
#pragma unroll
        for (int r = 0; r < kFusedBeams; ++r) {
            const int i = r * kStepThreads + tid;
            if (!ok4 || i >= q.num_new) continue;
            const int o = bo[r], t = bt[r];
            int b = o;
            if (bk[r] >= 0) {
                const int k = bk[r];
                b = policy == PA_POOL_FIFO ? p.ring[(head + k) % nb] : p.ring[(head + count + freed - 1 - k) % nb];
                p.ref[b] = 1;
            }
            q.new_tables[(long long)i * MB + t / bs] = b;
            if (bc[r] >= 0) {
                q.cow_pairs[2 * bc[r]] = o;
                q.cow_pairs[2 * bc[r] + 1] = b;
                atomicSub(&p.ref[o], 1);  // a copying writer gives up its reference to the old block
            }
            q.slots[i] = b * bs + t % bs;
            q.new_ctx[i] = t + 1;
        }
#pragma unroll
        for (int r = 0; r < kFusedBeams; ++r) {  // writer marks back, failed outputs
            const int i = r * kStepThreads + tid;
            if (bo[r] >= 0 && bo[r] < nb) {
                p.writers[bo[r]] = 0;
                p.last_writer[bo[r]] = -1;
            }
            if (!ok4 && i < q.num_new) q.slots[i] = -1;
        }
        if (tid == 0) {
            if (ok4) {
                p.hdr[3] = policy == PA_POOL_FIFO ? (head + takes) % nb : head;
                p.hdr[4] = count + freed - takes;
                *q.num_cow = copies;
            } else {
                *q.num_cow = 0;
                const int why = st.bad | bits;
                record_error(q.err, why ? (unsigned)why : (go ? PA_DEVERR_POOL : PA_DEVERR_TIMEOUT));
            }
            // the next step's epoch and barrier base (every CTA read them before barrier 1)
            p.hdr[7] = (int)(base + (early ? 2u : 3u) * G);
            p.hdr[6] = epoch + 1;
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
                             int num_blocks, int block_size, unsigned int *err, cudaStream_t stream,
                             int withhold_cta, unsigned long long barrier_limit_ns) {
    const bool hook = withhold_cta >= 0;
    beam::StepParams q;
    q.withhold_cta = withhold_cta;
    q.barrier_limit_ns = barrier_limit_ns;
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
    const long long entries = (long long)num_old * max_blocks;
    const int smem = (3 * num_old + num_new) * (int)sizeof(int);
    const dim3 block(beam::kStepThreads);
    // chunk: a multiple of the CTA size, so that there are at most max_ctas chunks
    auto chunk_for = [&](long long max_ctas) {
        long long c = (entries + max_ctas - 1) / max_ctas;
        c = (c + beam::kStepThreads - 1) / beam::kStepThreads * beam::kStepThreads;
        return std::max<long long>(c, beam::kStepThreads);
    };
    // One cooperative launch, one CTA per chunk and at most one chunk per SM
    // (one such CTA fits on any SM: 256 threads, < 100 KB of shared memory,
    // few registers, so the whole grid can be resident at once).
    const long long fused_chunk = chunk_for(std::min<long long>(sm_count(), beam::kMaxChunks));
    if (fused_chunk <= (long long)beam::kStepThreads * beam::kFusedEntries &&
        num_new <= beam::kStepThreads * beam::kFusedBeams) {
        const long long chunk = fused_chunk;
        q.chunk = (int)chunk;
        q.num_chunks = (int)std::max(1LL, (entries + chunk - 1) / chunk);
        static AttrCache fused_attr[2];
        const void *fused = hook ? reinterpret_cast<const void *>(beam::beam_step_kernel<true>)
                                 : reinterpret_cast<const void *>(beam::beam_step_kernel<false>);
        cudaError_t e = ensure_smem_attr(fused, beam::kMaxStageBytes, &fused_attr[hook ? 1 : 0]);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(q.num_chunks);
        cfg.blockDim = block;
        cfg.dynamicSmemBytes = (size_t)smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = hook ? cudaLaunchKernelEx(&cfg, beam::beam_step_kernel<true>, q)
                 : cudaLaunchKernelEx(&cfg, beam::beam_step_kernel<false>, q);
        if (e == cudaSuccess) return cudaSuccess;
        if (e != cudaErrorCooperativeLaunchTooLarge && e != cudaErrorNotSupported) return e;
        (void)cudaGetLastError();  // not launched: the four launches below instead
    }
    if (hook) return cudaErrorNotSupported;  // the hook is the one-launch form's only
    // Four launches (launches 2-4 by programmatic dependent launch), chunks
    // of at least one entry per thread, at most kMaxChunks of them.
    const long long chunk = chunk_for(beam::kMaxChunks);
    q.chunk = (int)chunk;
    q.num_chunks = (int)std::max(1LL, (entries + chunk - 1) / chunk);
    static AttrCache attr_done[4];
    const void *kernels[4] = {reinterpret_cast<const void *>(beam::beam_count_kernel),
                              reinterpret_cast<const void *>(beam::beam_flags_kernel),
                              reinterpret_cast<const void *>(beam::beam_apply_kernel),
                              reinterpret_cast<const void *>(beam::beam_finish_kernel)};
    for (int k = 0; k < 4; ++k) {
        cudaError_t e = ensure_smem_attr(kernels[k], beam::kMaxStageBytes, &attr_done[k]);
        if (e != cudaSuccess) return e;
    }
    const dim3 grid(q.num_chunks);
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
