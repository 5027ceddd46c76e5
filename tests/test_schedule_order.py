"""Host-side step decisions for the decode kernels: scheduling orders
(seq_order) must be permutations, longest_first sorts by decreasing context,
the grouped order keeps each prefix-sharing group together; the one-launch
slot write + decode is chosen only when every slot is its sequence's newest."""
import numpy as np

from paged_kv_cache_340_b200.batch import groups_longest_first, longest_first


def test_longest_first_is_a_descending_permutation():
    rng = np.random.default_rng(1)
    ctx = rng.integers(0, 5000, 257).astype(np.int32)
    o = longest_first(ctx)
    assert o.dtype == np.int32 and sorted(o.tolist()) == list(range(257))
    assert np.all(np.diff(ctx[o]) <= 0)


def test_groups_stay_together_and_lead_with_their_longest():
    ctx = np.array([5, 9, 1, 20, 3, 4, 7, 7, 2], np.int32)
    o = groups_longest_first(ctx, 3)
    assert o.tolist() == [3, 5, 4, 1, 0, 2, 6, 7, 8]
    rng = np.random.default_rng(2)
    ctx = rng.integers(1000, 1300, 80).astype(np.int32)
    o = groups_longest_first(ctx, 5)
    assert sorted(o.tolist()) == list(range(80))
    groups = o.reshape(16, 5) // 5
    assert np.all(groups == groups[:, :1])               # each run of 5 is one group
    heads = ctx[o.reshape(16, 5)[:, 0]]
    assert np.all(np.diff(heads) <= 0)                    # groups by their longest member


def test_newest_token_slots_decides_the_one_launch_step():
    """The one-launch slot write + decode applies only when slots[s] is the
    slot of token ctx[s] - 1 as each table gives it."""
    from paged_kv_cache_340_b200.batch import newest_token_slots
    bs = 16
    tables = np.array([[3, 5, -1], [7, -1, -1], [2, 9, 4]], np.int32)
    ctx = np.array([20, 3, 33], np.int32)
    slots = np.array([5 * bs + 3, 7 * bs + 2, 4 * bs + 0], np.int32)
    assert newest_token_slots(tables, ctx, bs, slots)
    assert not newest_token_slots(tables, ctx, bs, slots + np.array([0, 1, 0], np.int32))   # another slot
    assert not newest_token_slots(tables, np.array([20, 3, 0], np.int32), bs, slots)       # an empty sequence
    assert not newest_token_slots(tables, ctx, bs, np.concatenate([slots, slots]))         # more tokens than sequences
    # the decode workloads' batches are built that way (host side only, no device)
    from paged_kv_cache_340_b200.workloads import SPECS, make_decode_inputs, scaled
    spec = scaled(SPECS["llama7b_mha_fp16"], num_seqs=6)
    inp = make_decode_inputs(spec)
    ctx = inp["context_lens"].numpy().astype(np.int32)
    from paged_kv_cache_340_b200 import BlockPool, PA_POOL_FIFO
    pool = BlockPool(int(inp["num_blocks"]), bs, PA_POOL_FIFO, free_order=inp["free_order"].numpy())
    mb = -(-int(ctx.max()) // bs)
    tables = np.full((len(ctx), mb), -1, np.int32)
    slots = np.empty(len(ctx), np.int32)
    for s in range(len(ctx)):
        nt, _, _ = pool.append(tables[s], 0, int(ctx[s]) - 1, want_slots=False)
        _, sl, _ = pool.append(tables[s], nt, 1)
        slots[s] = sl[0]
    assert newest_token_slots(tables, ctx, bs, slots)
