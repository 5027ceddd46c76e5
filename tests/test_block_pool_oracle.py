"""Pins the oracle's host block pool (reference counts, copy-on-write) to the
pages' worked examples."""
import os

import pytest

from oracle.block_pool import BlockPool, PoolExhausted, Sequence, append_tokens, beam_step, fork, release

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def test_p1_request_mapping():
    """[P1] §2: requests of 32, 16 and 48 tokens take [0,1], [2], [3,4,5]
    from a pool handing out blocks front-first."""
    rows = _rows("p1_request_mapping.txt")
    pool = BlockPool(16, 16, policy="fifo")
    for r in rows:
        if r[0] in ("used", "next_free"):
            continue
        seq = Sequence()
        append_tokens(pool, seq, int(r[1]))
        assert seq.block_table == [int(x) for x in r[2].split(",")]
    used = [int(x) for x in dict((r[0], r[1]) for r in rows)["used"].split(",")]
    assert [b for b in range(16) if pool.ref_counts[b] > 0] == used
    assert pool.free_blocks[0] == int(dict((r[0], r[1]) for r in rows)["next_free"])


def test_lifo_pool_reuses_last_freed():
    """[P2] §4.2: allocate pops the free list's end; free appends at count 0."""
    pool = BlockPool(4, 16, policy="lifo")
    a = pool.allocate()
    b = pool.allocate()
    assert (a, b) == (3, 2)
    pool.free(a)
    assert pool.allocate() == a
    assert pool.num_free() == 2


def test_cow_timeline():
    """[P4] §3.3: A and B share block 5; B writes offset 8 -> copy to a new
    block (42 here), ref(5) 2 -> 1, ref(42) = 1, A keeps 5."""
    g = dict((r[0], r[1]) for r in _rows("cow_timeline.txt"))
    shared = int(g["shared_block"])
    order = [shared, 42] + [b for b in range(64) if b not in (shared, 42)]
    pool = BlockPool(64, 16, policy="fifo", free_order=order)
    a = Sequence()
    append_tokens(pool, a, int(g["write_offset"]))
    assert a.block_table == [shared]
    b = fork(pool, a)
    assert pool.ref_counts[shared] == int(g["ref_before"])
    slots, cow = append_tokens(pool, b, 1)
    assert cow == [(shared, 42)]
    assert slots == [42 * 16 + int(g["write_offset"])]
    assert pool.ref_counts[shared] == int(g["ref_old_after"])
    assert pool.ref_counts[42] == int(g["ref_new_after"])
    assert a.block_table == [shared] and b.block_table == [42]
    # A now owns block 5 alone: its next write goes in place.
    slots, cow = append_tokens(pool, a, 1)
    assert cow == [] and slots == [shared * 16 + 8]


def test_parallel_sampling_geometry():
    """n = 5 branches over a 1000-token prefix at block size 16: 63 prefix
    blocks (62 full + 8 tokens), ref 5 after forking; the first divergent
    token lands at offset 8 of block 62, so branches 0-3 copy it and branch 4
    (ref back to 1 by then) writes in place. [P2] §3.4 (n = 5 sharing);
    [P4] §3.3 (copy on write when ref > 1)."""
    pool = BlockPool(200, 16, policy="fifo")
    root = Sequence()
    append_tokens(pool, root, 1000)
    assert len(root.block_table) == 63
    branches = [root] + [fork(pool, root) for _ in range(4)]
    assert all(pool.ref_counts[b] == 5 for b in root.block_table)
    last = root.block_table[62]
    pairs = []
    for br in branches:
        slots, cow = append_tokens(pool, br, 1)
        pairs += cow
        assert slots[0] % 16 == 8
    assert len(pairs) == 4 and all(src == last for src, _ in pairs)
    # Branches write in list order: the first four copy, the last writes in place.
    assert branches[4].block_table[62] == last
    assert all(br.block_table[62] != last for br in branches[:4])
    assert pool.ref_counts[last] == 1
    assert all(br.block_table[:62] == root.block_table[:62] for br in branches)
    assert all(pool.ref_counts[b] == 5 for b in root.block_table[:62])


def test_release_and_exhaustion():
    pool = BlockPool(3, 4, policy="fifo")
    s = Sequence()
    append_tokens(pool, s, 12)
    with pytest.raises(PoolExhausted):
        append_tokens(pool, s, 1)
    t = fork(pool, s)
    release(pool, s)
    assert pool.num_free() == 0
    release(pool, t)
    assert pool.num_free() == 3
    with pytest.raises(ValueError):
        pool.free(0)


# ------------------------------------------------------------- beam search

def test_beam_step_worked_example():
    """Two beams, both children of beam A ([P2] §3.4 beam search sharing,
    [P4] §3.3 copy on write), block size 4, front-first pool 0..15:
    A = 6 tokens in [0, 1] (block 1 holds 2), B = 3 tokens in [2].
    Fork: counts of 0 and 1 go 1 -> 3. Release A: 3 -> 2; release B: block 2
    reaches 0 and goes to the back of the free list. Child 0 writes token 6
    into block 1 (count 2): copies it to the free list's front, 3, and block
    1 drops to 1. Child 1 then finds count 1 and writes in place."""
    pool = BlockPool(16, 4, policy="fifo")
    a, b = Sequence(), Sequence()
    append_tokens(pool, a, 6)
    append_tokens(pool, b, 3)
    assert (a.block_table, b.block_table) == ([0, 1], [2])
    new, slots, cow = beam_step(pool, [a, b], [0, 0])
    assert [c.block_table for c in new] == [[0, 3], [0, 1]]
    assert [c.num_tokens for c in new] == [7, 7]
    assert slots == [3 * 4 + 2, 1 * 4 + 2]
    assert cow == [(1, 3)]
    assert pool.ref_counts[:5] == [2, 1, 0, 1, 0]
    assert pool.free_blocks == list(range(4, 16)) + [2]


def test_beam_step_identity_is_plain_append():
    """parents = identity: each beam keeps its blocks and appends one token,
    exactly as append_tokens does (a new block at a block boundary)."""
    p1, p2 = BlockPool(64, 16, policy="lifo"), BlockPool(64, 16, policy="lifo")
    beams1, beams2 = [], []
    for n in (15, 16, 17, 1):
        for p, bl in ((p1, beams1), (p2, beams2)):
            s = Sequence()
            append_tokens(p, s, n)
            bl.append(s)
    new, slots, cow = beam_step(p1, beams1, [0, 1, 2, 3])
    want = []
    for s in beams2:
        want += append_tokens(p2, s, 1)[0]
    assert slots == want and cow == []
    assert [c.block_table for c in new] == [s.block_table for s in beams2]
    assert p1.ref_counts == p2.ref_counts and p1.free_blocks == p2.free_blocks


@pytest.mark.parametrize("policy", ["fifo", "lifo"])
def test_beam_step_invariants_random(policy):
    """Over many random steps: every count equals the number of beams whose
    table holds the block; the free list is exactly the blocks of count 0,
    without repeats; the new tokens' slots are distinct; a child's table is
    its parent's except the block it wrote into; the number of copies of a
    block is its writers minus one when no other beam holds it, else its
    writers."""
    import random
    rng = random.Random(7)
    pool = BlockPool(400, 4, policy=policy)
    beams = []
    for n in (5, 9, 12, 1):
        s = Sequence()
        append_tokens(pool, s, n)
        beams.append(s)
    for step in range(60):
        w_new = rng.randint(1, 6)
        parents = [rng.randrange(len(beams)) for _ in range(w_new)]
        before = [(list(b.block_table), b.num_tokens) for b in beams]
        writers = {}
        holders = {}
        for p in parents:
            tab, t = before[p]
            for bid in tab:
                holders[bid] = holders.get(bid, 0) + 1
            if t % 4:
                writers[tab[t // 4]] = writers.get(tab[t // 4], 0) + 1
        new, slots, cow = beam_step(pool, beams, parents)
        counts = {}
        for c in new:
            for bid in c.block_table:
                counts[bid] = counts.get(bid, 0) + 1
        assert all(pool.ref_counts[bid] == counts.get(bid, 0) for bid in range(400))
        assert sorted(pool.free_blocks) == [bid for bid in range(400) if counts.get(bid, 0) == 0]
        assert len(set(slots)) == len(slots)
        for i, (c, p) in enumerate(zip(new, parents)):
            tab, t = before[p]
            assert c.num_tokens == t + 1
            lb = t // 4
            assert c.block_table[:lb] == tab[:lb]
            assert slots[i] == c.block_table[lb] * 4 + t % 4
        for src, n_w in writers.items():
            others = holders[src] - n_w
            assert sum(1 for s_, _ in cow if s_ == src) == (n_w if others else n_w - 1)
        beams = new
