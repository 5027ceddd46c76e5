"""Prefix cache ([P4] "PagedAttention 实现细节", §3.2): the oracle's manager
is pinned to the pages' printed demo and to its own rules; the library's C++
cache (pa_prefix_* calls) must make exactly the oracle's decisions (hits, block
ids, use counts, pool state) on random operation sequences, including with a
truncated hash that forces every prompt into a few buckets."""
import os

import numpy as np
import pytest

from oracle.block_pool import BlockPool as OPool, PoolExhausted, Sequence, append_tokens, fork
from oracle.prefix_cache import PrefixCacheManager

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _kv(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return dict(ln.split()[:2] for ln in f if ln.strip() and not ln.startswith("#"))


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_340_b200 import _build
    _build.build()
    import paged_kv_cache_340_b200 as pa
    return pa


def _demo(pool, cache, use_cache):
    """The pages' scenario run through a pool: every request takes the system
    prompt's blocks (from the cache, or its own without it) and its own blocks
    for its user tokens."""
    g = _kv("prefix_cache_demo.txt")
    bs = int(g["block_size"])
    system = list(range(1000, 1000 + int(g["system_prompt_tokens"])))
    n_user = int(g["user_tokens"])
    hits = 0
    for _ in range(int(g["num_requests"])):
        if use_cache:
            _, hit = cache.get_or_create(system)
            hits += hit
        else:
            for _ in range((len(system) + bs - 1) // bs):
                pool.allocate()
        for _ in range((n_user + bs - 1) // bs):
            pool.allocate()
    return g, hits


def _check_demo(g, used_without, used_with, hits):
    assert used_without == int(g["blocks_without_cache"])
    assert used_with == int(g["blocks_with_cache"])
    saved = used_without - used_with
    assert saved == int(g["blocks_saved"])
    assert f"{saved / used_without * 100:.1f}" == g["saving_pct"]
    assert f"{saved * int(g['block_kib']) / 1024:.1f}" == g["saved_mib"]
    assert hits == int(g["num_requests"]) - 1


def test_oracle_manager_reproduces_printed_demo():
    """[P4] §3.2 printed output (300 / 201 / 99 / 33.0% / 12.4 MB), by running
    the manager over a pool rather than by the demo's arithmetic."""
    p0 = OPool(1024, 16, policy="fifo")
    _demo(p0, None, use_cache=False)
    p1 = OPool(1024, 16, policy="fifo")
    c1 = PrefixCacheManager(p1)
    g, hits = _demo(p1, c1, use_cache=True)
    _check_demo(g, 1024 - p0.num_free(), 1024 - p1.num_free(), hits)
    assert c1.ref_count(range(1000, 1009)) == 100


def test_oracle_manager_rules():
    pool = OPool(8, 4, policy="lifo")
    c = PrefixCacheManager(pool)
    ids, hit = c.get_or_create([5, 6, 7, 8, 9])          # 5 tokens at bs 4: two blocks
    assert not hit and ids == [7, 6] and pool.num_free() == 6
    ids2, hit = c.get_or_create([5, 6, 7, 8, 9])
    assert hit and ids2 == ids and pool.num_free() == 6 and c.ref_count([5, 6, 7, 8, 9]) == 2
    _, hit = c.get_or_create([5, 6, 7, 8])               # a different (shorter) prompt: its own entry
    assert not hit and c.num_entries() == 2
    c.release([1, 2, 3])                                 # unknown: ignored
    c.release([5, 6, 7, 8, 9])
    assert c.ref_count([5, 6, 7, 8, 9]) == 1 and pool.num_free() == 5
    c.release([5, 6, 7, 8, 9])                           # last user: blocks back, entry gone
    assert c.ref_count([5, 6, 7, 8, 9]) == 0 and pool.num_free() == 7 and c.num_entries() == 1
    assert pool.free_blocks[-2:] == ids                  # freed in entry order
    with pytest.raises(PoolExhausted):                   # 8 blocks wanted, 7 free: nothing taken
        c.get_or_create(list(range(32)))
    assert pool.num_free() == 7
    ids3, hit = c.get_or_create([])                      # the empty prompt holds no block
    assert ids3 == [] and not hit


def test_oracle_prefix_shared_by_sequences_copies_on_write():
    """A sequence that maps the prefix blocks into its table takes its own
    references (fork), so its first write into the partial last block copies it
    and the cached prefix keeps its bytes ([P4] §3.2 with §3.3)."""
    pool = OPool(32, 16, policy="fifo")
    c = PrefixCacheManager(pool)
    prompt = list(range(20))                             # 20 tokens: blocks [0, 1], block 1 partial
    ids, _ = c.get_or_create(prompt)
    base = Sequence(block_table=list(ids), num_tokens=len(prompt))
    seq = fork(pool, base)
    assert [pool.ref_counts[b] for b in ids] == [2, 2]
    slots, cow = append_tokens(pool, seq, 1)
    assert cow == [(ids[1], 2)] and slots == [2 * 16 + 4]
    assert seq.block_table == [ids[0], 2]


def _random_ops(seed, n_ops=600, n_blocks=96, bs=16):
    rng = np.random.default_rng(seed)
    prompts = [list(rng.integers(0, 50000, size=int(rng.integers(0, 70)))) for _ in range(12)]
    prompts.append(prompts[3][:-1] if len(prompts[3]) > 1 else [7])   # a prefix of another prompt
    prompts.append([])
    ops = []
    for _ in range(n_ops):
        r = rng.random()
        i = int(rng.integers(len(prompts)))
        if r < 0.5:
            ops.append(("get", i))
        elif r < 0.85:
            ops.append(("release", i))
        elif r < 0.95:
            ops.append(("alloc", 0))
        else:
            ops.append(("free", 0))
    return prompts, ops


@pytest.mark.parametrize("hash_bits", [0, 2])
@pytest.mark.parametrize("seed", [1, 2, 3])
def test_library_prefix_cache_matches_oracle(pa, seed, hash_bits):
    bs, nb = 16, 96
    order = np.random.default_rng(seed + 10).permutation(nb).astype(np.int32)
    opool = OPool(nb, bs, policy="fifo", free_order=order.tolist())
    ocache = PrefixCacheManager(opool)
    lpool = pa.BlockPool(nb, bs, pa.PA_POOL_FIFO, order)
    lcache = pa.PrefixCache(lpool, hash_bits=hash_bits)
    prompts, ops = _random_ops(seed)
    held_o, held_l = [], []
    n_exhausted = 0
    for op, i in ops:
        if op == "get":
            try:
                want = ocache.get_or_create(prompts[i])
            except PoolExhausted:
                n_exhausted += 1
                with pytest.raises(pa.PagedAttentionError) as e:
                    lcache.get_or_create(prompts[i])
                assert e.value.status == -11
                continue
            assert lcache.get_or_create(prompts[i]) == want
        elif op == "release":
            ocache.release(prompts[i])
            lcache.release(prompts[i])
        elif op == "alloc" and opool.num_free():
            held_o.append(opool.allocate())
            held_l.append(lpool.allocate())
        elif op == "free" and held_o:
            opool.free(held_o.pop())
            lpool.free(held_l.pop())
        assert lpool.num_free() == opool.num_free()
        assert lcache.num_entries() == ocache.num_entries()
        assert lcache.ref_count(prompts[i]) == ocache.ref_count(prompts[i])
    assert [lpool.ref_count(b) for b in range(nb)] == opool.ref_counts
    assert held_l == held_o


def test_library_demo(pa):
    """The pages' demo through the library's pool and cache: 201 blocks in use."""
    lp0 = pa.BlockPool(1024, 16, pa.PA_POOL_FIFO)
    _demo(lp0, None, use_cache=False)
    lp1 = pa.BlockPool(1024, 16, pa.PA_POOL_FIFO)
    c = pa.PrefixCache(lp1)
    g, hits = _demo(lp1, c, use_cache=True)
    _check_demo(g, 1024 - lp0.num_free(), 1024 - lp1.num_free(), hits)


def test_library_prefix_errors(pa):
    lp = pa.BlockPool(4, 16, pa.PA_POOL_LIFO)
    c = pa.PrefixCache(lp)
    with pytest.raises(pa.PagedAttentionError) as e:
        c.get_or_create(list(range(80)))                 # 5 blocks from a 4-block pool
    assert e.value.status == -11 and lp.num_free() == 4 and c.num_entries() == 0
    ids, _ = c.get_or_create(list(range(17)))
    lp.free(ids[0])                                      # caller freed a cached block behind its back
    with pytest.raises(pa.PagedAttentionError) as e:
        c.release(list(range(17)))
    assert e.value.status == -12 and c.num_entries() == 1
    import ctypes
    ids_buf = np.zeros(1, np.int32)
    n, hit = ctypes.c_int(0), ctypes.c_int(0)
    t = np.arange(40, dtype=np.int32)                    # 3 blocks, room for 1
    rc = pa._lib.pa_prefix_get_or_create(c._h, pa._i32p(t), 40, pa._i32p(ids_buf), 1, ctypes.byref(n),
                                         ctypes.byref(hit))
    assert rc == -13
    assert pa._lib.pa_prefix_cache_create(None, 0) is None
    assert pa._lib.pa_prefix_cache_create(lp._h, 65) is None


def test_oracle_request_flow_hand_worked():
    """Requests over the cache, worked by hand (pool of 8 blocks of 4 tokens,
    FIFO from 0): prompt A = 6 tokens (blocks 0, 1; block 1 partial), B = 3.
    r0 (A + 3): miss, writes A at slots 0..5, copies block 1 -> 2 before its
    first token (slot 10), then 11 and a new block 3 (12). r1 (A + 1): hit,
    copies 1 -> 4 (slot 18). r0 finishes: blocks 2 and 3 return to the free
    list's end (5, 6, 7, 2, 3); block 0 stays (cache and r1). r2 (A + 2): hit,
    copies 1 -> 5 (slots 22, 23). r3 (B + 1): miss, block 6 (slots 24..26),
    copied to 7 before its own token (slot 31)."""
    from oracle.prefix_cache import request_flow
    A = [11, 12, 13, 14, 15, 16]
    B = [21, 22, 23]
    toks = np.zeros((2, 6), np.int32)
    toks[0, :6], toks[1, :3] = A, B
    ops, tables, ctx, live = request_flow([6, 3], toks, [0, 0, 0, 1], [3, 1, 2, 1], 8, list(range(8)), 4, 3,
                                          finish_after={1: [0]})
    assert ops == [("prefix", 0, [0, 1, 2, 3, 4, 5]), ("copy", 0, [[1, 2]]), ("user", 0, [10, 11, 12]),
                   ("copy", 1, [[1, 4]]), ("user", 1, [18]), ("finish", 0, []),
                   ("copy", 2, [[1, 5]]), ("user", 2, [22, 23]),
                   ("prefix", 1, [24, 25, 26]), ("copy", 3, [[6, 7]]), ("user", 3, [31])]
    assert tables.tolist() == [[-1, -1, -1], [0, 4, -1], [0, 5, -1], [7, -1, -1]]
    assert ctx.tolist() == [0, 7, 8, 4] and live.tolist() == [False, True, True, True]


@pytest.mark.parametrize("seed", [0, 1])
def test_library_request_flow_matches_oracle(pa, seed):
    """The library's host flow (its pool and prefix cache) makes the oracle's
    decisions: the same prefix writes, copy pairs, slots, tables and lengths,
    with requests finishing (and prompts released and re-created) mid-flow."""
    from paged_kv_cache_340_b200.batch import prefix_cache_flow
    from paged_kv_cache_340_b200.workloads import SPECS, make_prefix_cache_inputs, scaled
    from oracle.prefix_cache import request_flow
    spec = scaled(SPECS["prefix_cache_fp16"], seed=100 + seed, num_seqs=40, num_heads=2, num_kv_heads=2,
                  head_dim=64, lengths=("prefix", 1, 120), num_prompts=4, prefix_len=120, max_divergent=50)
    inp = make_prefix_cache_inputs(spec)
    rng = np.random.default_rng(seed)
    finish_after, alive = {}, []
    for r in range(40):
        alive.append(r)
        if rng.random() < 0.4 and len(alive) > 1:
            done = [int(x) for x in rng.choice(alive, size=int(rng.integers(1, len(alive))), replace=False)]
            finish_after[r] = done
            alive = [a for a in alive if a not in done]
    ops, tables, ctx, live = prefix_cache_flow(spec, inp, finish_after=finish_after)
    want = request_flow(inp["system_lens"].numpy(), inp["system_tokens"].numpy(), inp["choice"].numpy(),
                        inp["user_lens"].numpy(), int(inp["num_blocks"]), inp["free_order"].numpy(),
                        spec.block_size, tables.shape[1], finish_after)
    assert [(o.kind, o.index) for o in ops] == [(k, i) for k, i, _ in want[0]]
    for o, (_, _, w) in zip(ops, want[0]):
        assert np.array_equal(o.slots.reshape(-1), np.asarray(w, np.int64).reshape(-1))
    assert np.array_equal(tables, want[1]) and np.array_equal(ctx, want[2]) and np.array_equal(live, want[3])
    assert sum(o.kind == "prefix" for o in ops) > spec.num_prompts   # some prompt was released and written again
