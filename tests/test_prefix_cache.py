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
