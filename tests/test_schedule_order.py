"""Host scheduling orders handed to the decode kernels (seq_order): they
must be permutations; longest_first sorts by decreasing context; the grouped
order keeps each prefix-sharing group together."""
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
