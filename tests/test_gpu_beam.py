"""Device block pool and beam-search step (pa_dpool_*, pa_beam_step,
pa_copy_blocks_counted) against the oracle pool's beam_step.

The device step must leave exactly the oracle's state: reference counts,
free list (order included), new tables, context lengths, slots and
copy-on-write pairs, bit for bit. Then the K/V data path (counted copy, slot
write, decode) over the device-made tables must match the oracle's caches
bit for bit and its attention within the tolerance."""
import numpy as np
import pytest
import torch

import oracle
from oracle.block_pool import BlockPool as OPool, Sequence, append_tokens, beam_step
from _helpers import assert_attention_close, f64, raw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_340_b200 import _build
    _build.build()
    import paged_kv_cache_340_b200 as pa
    return pa


def _tables(beams, mb):
    t = np.full((max(1, len(beams)), mb), -1, np.int32)[: len(beams)]
    for i, b in enumerate(beams):
        t[i, :len(b.block_table)] = b.block_table
    return t


def _policy(pa, name):
    return pa.PA_POOL_FIFO if name == "fifo" else pa.PA_POOL_LIFO


def _start(pa, nb, bs, policy, lengths, seed):
    """Oracle pool and device pool from one seeded free order, with beams of
    the given lengths: appended through the oracle pool and through the
    library's host pool, whose state is then loaded into the device pool."""
    order = np.random.default_rng(seed).permutation(nb).astype(np.int32)
    opool = OPool(nb, bs, policy=policy, free_order=order.tolist())
    hpool = pa.BlockPool(nb, bs, _policy(pa, policy), free_order=order)
    beams = []
    for n in lengths:
        s = Sequence()
        append_tokens(opool, s, n)
        beams.append(s)
        tab = np.full(nb, -1, np.int32)
        hpool.append(tab, 0, n)
        assert tab[:len(s.block_table)].tolist() == s.block_table
    dpool = pa.DevicePool(nb, bs, _policy(pa, policy), host_pool=hpool)
    return opool, dpool, beams


def _device_step(pa, dpool, beams, parents, mb):
    dev = "cuda"
    old_t = torch.from_numpy(_tables(beams, mb)).to(dev)
    old_c = torch.tensor([b.num_tokens for b in beams], dtype=torch.int32, device=dev)
    par = torch.tensor(parents, dtype=torch.int32, device=dev)
    n = len(parents)
    new_t = torch.full((n, mb), 7777, dtype=torch.int32, device=dev)
    new_c = torch.full((n,), -5, dtype=torch.int32, device=dev)
    slots = torch.full((n,), -5, dtype=torch.int32, device=dev)
    cow = torch.full((n, 2), -5, dtype=torch.int64, device=dev)
    ncow = torch.full((1,), -5, dtype=torch.int32, device=dev)
    pa.pa_beam_step(dpool, old_t, old_c, par, new_t, new_c, slots, cow, ncow)
    torch.cuda.synchronize()
    return new_t.cpu().numpy(), new_c.cpu().numpy(), slots.cpu().numpy(), cow.cpu().numpy(), int(ncow.item())


def _host_copy(pa, opool):
    """A library host pool in the oracle pool's state (same counts and free
    list), built by the pool's own calls: allocate everything in free-list
    order, then free back to the oracle's state."""
    nb = opool.num_blocks
    hp = pa.BlockPool(nb, opool.block_size, pa.PA_POOL_FIFO, free_order=np.arange(nb, dtype=np.int32))
    for _ in range(nb):
        hp.allocate()
    for b in range(nb):                                  # counts: share up to the oracle's count
        for _ in range(opool.ref_counts[b] - 1):
            hp.share(b)
    for b in opool.free_blocks:                          # free in free-list order
        hp.free(b)
    ref, fl = hp.export()
    assert ref.tolist() == opool.ref_counts and fl.tolist() == opool.free_blocks
    return hp


def _assert_same_state(dpool, opool):
    assert dpool.ref.cpu().tolist() == opool.ref_counts
    assert dpool.free_list() == opool.free_blocks


def test_dpool_init(pa):
    order = np.random.default_rng(0).permutation(50).astype(np.int32)
    d = pa.DevicePool(50, 16, pa.PA_POOL_FIFO, free_order=order)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    assert d.ref.cpu().tolist() == [0] * 50
    assert d.free_list() == order.tolist()
    d2 = pa.DevicePool(8, 16, pa.PA_POOL_LIFO)
    assert d2.free_list() == list(range(8))
    bad = order.copy()
    bad[3] = bad[4]                                      # not a permutation
    d3 = pa.DevicePool(50, 16, pa.PA_POOL_FIFO, free_order=bad)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() & pa.PA_DEVERR_POOL
    # a step on the unusable state changes nothing
    t, c, slots, cow, ncow = _device_step(pa, d3, [Sequence([1], 3)], [0], 4)
    assert pa.pa_read_device_errors() & pa.PA_DEVERR_POOL
    assert (slots == -1).all() and ncow == 0


def test_dpool_load_checks_consistency(pa):
    """A free list naming a block still in use, or a block of count 0 left off
    the list, is refused (PA_DEVERR_POOL) and the state is unusable."""
    nb = 16
    ref = torch.zeros(nb, dtype=torch.int32, device="cuda")
    ref[:4] = 1
    good = torch.arange(4, nb, dtype=torch.int32, device="cuda")
    for fl in (torch.arange(3, nb, dtype=torch.int32, device="cuda"),     # block 3 has count 1
               torch.arange(5, nb, dtype=torch.int32, device="cuda"),     # block 4 (count 0) missing
               torch.cat([good[:-1], good[:1]])):                         # a repeat
        st = torch.empty(int(pa._lib.pa_dpool_state_bytes(nb)) // 4, dtype=torch.int32, device="cuda")
        assert pa._lib.pa_dpool_load(st.data_ptr(), nb, 4, 0, ref.data_ptr(), fl.data_ptr(), fl.shape[0],
                                     None) == 0
        torch.cuda.synchronize()
        assert pa.pa_read_device_errors() & pa.PA_DEVERR_POOL
        assert st[5].item() == 0
    st = torch.empty(int(pa._lib.pa_dpool_state_bytes(nb)) // 4, dtype=torch.int32, device="cuda")
    assert pa._lib.pa_dpool_load(st.data_ptr(), nb, 4, 0, ref.data_ptr(), good.data_ptr(), good.shape[0], None) == 0
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0 and st[5].item() != 0


def test_worked_example_on_device(pa):
    """Two beams, both children of beam A (block size 4): the oracle's worked
    example, on the device."""
    opool, dpool, beams = _start(pa, 16, 4, "fifo", [6, 3], seed=0)
    ob = [Sequence(list(b.block_table), b.num_tokens) for b in beams]
    new, slots, cow = beam_step(opool, ob, [0, 0])
    t, c, s, cw, n = _device_step(pa, dpool, beams, [0, 0], 4)
    assert t.tolist() == _tables(new, 4).tolist()
    assert c.tolist() == [7, 7] and s.tolist() == slots
    assert n == len(cow) and [tuple(x) for x in cw[:n].tolist()] == cow
    _assert_same_state(dpool, opool)
    assert pa.pa_read_device_errors() == 0


@pytest.mark.parametrize("policy", ["fifo", "lifo"])
@pytest.mark.parametrize("bs", [4, 16])
@pytest.mark.parametrize("extra", [8, 1600, 5000])
def test_random_beam_search_matches_oracle(pa, policy, bs, extra):
    """60 steps of random beam choices (widths 1-40, some parents chosen many
    times, some beams dropped) from 12 prompts: after every step the device
    state, tables, slots and pairs equal the oracle's. With 5000 spare table
    columns, steps from 30 or more beams have more old-table entries than the
    one-launch form keeps in registers (1024 per SM), so the four-launch form
    runs for those steps and the one-launch form for the others."""
    rng = np.random.default_rng(3 + bs)
    mb = 400 // bs + extra
    lengths = [int(x) for x in rng.integers(1, 300, size=12)]
    opool, dpool, beams = _start(pa, 3000, bs, policy, lengths, seed=bs)
    for step in range(60):
        w = int(rng.integers(1, 41))
        hot = int(rng.integers(len(beams)))
        parents = [hot if rng.random() < 0.4 else int(rng.integers(len(beams))) for _ in range(w)]
        ob = [Sequence(list(b.block_table), b.num_tokens) for b in beams]
        new, slots, cow = beam_step(opool, ob, parents)
        t, c, s, cw, n = _device_step(pa, dpool, beams, parents, mb)
        assert t.tolist() == _tables(new, mb).tolist(), step
        assert c.tolist() == [b.num_tokens for b in new]
        assert s.tolist() == slots
        assert n == len(cow) and [tuple(x) for x in cw[:n].tolist()] == cow
        _assert_same_state(dpool, opool)
        beams = new
    assert pa.pa_read_device_errors() == 0


def _pool_words(pa, dpool):
    """The pool proper: header words 0-5, counts, free-list ring and the
    per-block scratch arrays (words 6-7 and the tail are the device step's
    own bookkeeping, which every step advances)."""
    h, nb = pa.PA_DPOOL_HEADER_WORDS, dpool.num_blocks
    return torch.cat([dpool.state[:6], dpool.state[h:h + 6 * nb]]).clone()


def test_exhausted_pool_applies_nothing(pa):
    """Fewer free blocks than the step needs: state unchanged, slots -1, no pairs."""
    opool, dpool, beams = _start(pa, 12, 4, "fifo", [4, 8], seed=1)   # 3 blocks used, 9 free
    before = _pool_words(pa, dpool)
    # 10 children all at a block boundary (4 and 8 tokens): 10 new blocks wanted, 9 free (+0 freed)
    t, c, s, cw, n = _device_step(pa, dpool, beams, [0] * 5 + [1] * 5, 4)
    assert pa.pa_read_device_errors() & pa.PA_DEVERR_POOL
    assert (s == -1).all() and n == 0
    assert torch.equal(_pool_words(pa, dpool), before)
    # bad parent index
    t, c, s, cw, n = _device_step(pa, dpool, beams, [0, 2], 4)
    assert pa.pa_read_device_errors() & pa.PA_DEVERR_CONTEXT
    assert torch.equal(_pool_words(pa, dpool), before)
    # a table entry that the pool says is free
    bad = [Sequence([beams[0].block_table[0]], 4), Sequence([opool.free_blocks[0]], 2)]
    t, c, s, cw, n = _device_step(pa, dpool, bad, [0, 1], 4)
    assert pa.pa_read_device_errors() & pa.PA_DEVERR_BLOCK_ID
    assert torch.equal(_pool_words(pa, dpool), before)
    # no table room for the new token
    t, c, s, cw, n = _device_step(pa, dpool, beams, [1], 2)
    assert pa.pa_read_device_errors() & pa.PA_DEVERR_POOL
    assert torch.equal(_pool_words(pa, dpool), before)


def _beam_data_case(pa, seed, dtype):
    """Beam search over a paged cache: 6 prompts x 4 beams, 32 query heads
    (8 kv), head dim 128, block size 16. Each step on the device: pa_beam_step,
    counted copy of the copy-on-write blocks, slot write of the new tokens,
    decode over the new tables; the oracle does the same with its pool, byte
    copies and double-precision attention."""
    from oracle.block_pool import fork
    g = torch.Generator().manual_seed(seed)
    Hq, Hkv, D, bs, NB, mb = 32, 8, 128, 16, 640, 24
    prompts = [int(x) for x in torch.randint(20, 200, (6,), generator=g)]
    opool, dpool, roots = _start(pa, NB, bs, "lifo", prompts, seed=seed)
    ob = []
    for r in roots:                                      # 4 beams per prompt share its blocks
        ob += [r] + [fork(opool, r) for _ in range(3)]
    dpool = pa.DevicePool(NB, bs, pa.PA_POOL_LIFO, host_pool=_host_copy(pa, opool))
    W = len(ob)
    k = torch.randn((NB, Hkv, bs, D), generator=g).to(dtype)
    v = torch.randn((NB, Hkv, bs, D), generator=g).to(dtype)
    kd, vd = k.cuda(), v.cuda()
    k_or, v_or = raw(k).copy(), raw(v).copy()
    bufs = [(torch.empty((W, mb), dtype=torch.int32, device="cuda"), torch.empty(W, dtype=torch.int32, device="cuda"))
            for _ in range(2)]
    bufs[0][0].copy_(torch.from_numpy(_tables(ob, mb)))
    bufs[0][1].copy_(torch.tensor([b.num_tokens for b in ob], dtype=torch.int32))
    slots = torch.empty(W, dtype=torch.int32, device="cuda")
    cow = torch.empty((W, 2), dtype=torch.int64, device="cuda")
    ncow = torch.empty(1, dtype=torch.int32, device="cuda")
    out = torch.empty((W, Hq, D), dtype=torch.float32, device="cuda")
    scale = D ** -0.5
    rng = np.random.default_rng(seed)
    for i in range(12):
        # each beam's parent is one of its prompt's 4 beams
        parents = (rng.integers(0, 4, size=W) + (np.arange(W) // 4) * 4).astype(np.int32)
        q = torch.randn((W, Hq, D), generator=g).to(dtype)
        nk = torch.randn((W, Hkv, D), generator=g).to(dtype)
        nv = torch.randn((W, Hkv, D), generator=g).to(dtype)
        src, dst = bufs[i % 2], bufs[(i + 1) % 2]
        pa.pa_beam_step(dpool, src[0], src[1], torch.from_numpy(parents).cuda(), dst[0], dst[1], slots, cow, ncow)
        pa.pa_copy_blocks_counted(kd, vd, cow, ncow)
        pa.pa_reshape_and_cache(nk.cuda(), nv.cuda(), kd, vd, slots)
        pa.pa_decode(out, q.cuda(), kd, vd, dst[0], dst[1], scale)
        torch.cuda.synchronize()
        ob, oslots, ocow = beam_step(opool, ob, parents.tolist())
        if ocow:
            oracle.copy_blocks(k_or, v_or, np.array(ocow, np.int64))
        oracle.reshape_and_cache(k_or, v_or, raw(nk), raw(nv), np.array(oslots))
        assert slots.cpu().tolist() == oslots
        assert dst[0].cpu().numpy().tolist() == _tables(ob, mb).tolist()
        ref = oracle.paged_decode(f64(q), _f64_of(k_or, dtype), _f64_of(v_or, dtype), _tables(ob, mb),
                                  np.array([b.num_tokens for b in ob], np.int32), scale, bs)
        assert_attention_close(out, ref, dtype, f"beam step {i}")
    assert np.array_equal(raw(kd), k_or) and np.array_equal(raw(vd), v_or)
    _assert_same_state(dpool, opool)
    assert pa.pa_read_device_errors() == 0


def _f64_of(bits, dtype):
    return f64(torch.from_numpy(bits).view(dtype))


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_beam_search_data_path(pa, dtype):
    _beam_data_case(pa, 11, dtype)


def test_beam_step_in_cuda_graph(pa):
    """The whole step (beam step, counted copy, slot write, decode) captured in
    a CUDA graph and replayed: same results as eager calls on a twin state."""
    nb, bs, mb, W = 256, 16, 16, 8
    order = np.random.default_rng(4).permutation(nb).astype(np.int32)
    opool = OPool(nb, bs, policy="fifo", free_order=order.tolist())
    beams = []
    for n in [40, 33, 16, 70, 5, 90, 64, 17]:
        s = Sequence()
        append_tokens(opool, s, n)
        beams.append(s)
    pools = [pa.DevicePool(nb, bs, pa.PA_POOL_FIFO, host_pool=_host_copy(pa, opool)) for _ in range(2)]
    Hkv, Hq, D = 4, 16, 128
    g = torch.Generator().manual_seed(9)
    caches = [[torch.randn((nb, Hkv, bs, D), generator=g).half().cuda() for _ in range(2)]]
    caches.append([c.clone() for c in caches[0]])
    t0 = torch.from_numpy(_tables(beams, mb)).cuda()
    c0 = torch.tensor([b.num_tokens for b in beams], dtype=torch.int32, device="cuda")
    par = torch.tensor([0, 0, 3, 3, 3, 5, 6, 6], dtype=torch.int32, device="cuda")
    q = torch.randn((W, Hq, D), generator=g).half().cuda()
    nk = torch.randn((W, Hkv, D), generator=g).half().cuda()
    nv = torch.randn((W, Hkv, D), generator=g).half().cuda()

    def outputs():
        return dict(t=torch.empty((W, mb), dtype=torch.int32, device="cuda"),
                    c=torch.empty(W, dtype=torch.int32, device="cuda"),
                    s=torch.empty(W, dtype=torch.int32, device="cuda"),
                    p=torch.empty((W, 2), dtype=torch.int64, device="cuda"),
                    n=torch.empty(1, dtype=torch.int32, device="cuda"),
                    o=torch.empty((W, Hq, D), dtype=torch.float16, device="cuda"))

    def step(d, kv, o, stream=None):
        pa.pa_beam_step(d, t0, c0, par, o["t"], o["c"], o["s"], o["p"], o["n"], stream=stream)
        pa.pa_copy_blocks_counted(kv[0], kv[1], o["p"], o["n"], stream=stream)
        pa.pa_reshape_and_cache(nk, nv, kv[0], kv[1], o["s"], stream=stream)
        pa.pa_decode(o["o"], q, kv[0], kv[1], o["t"], o["c"], D ** -0.5, stream=stream)

    eager, graphed = outputs(), outputs()
    step(pools[0], caches[0], eager)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            step(pools[1], caches[1], graphed, stream=s)
    graph.replay()
    torch.cuda.synchronize()
    for key in ("t", "c", "s", "n"):
        assert torch.equal(eager[key], graphed[key]), key
    n = int(eager["n"].item())
    assert torch.equal(eager["p"][:n], graphed["p"][:n])
    assert torch.equal(eager["o"].view(torch.int16), graphed["o"].view(torch.int16))
    assert torch.equal(pools[0].state, pools[1].state)
    assert all(torch.equal(a.view(torch.int16), b.view(torch.int16)) for a, b in zip(caches[0], caches[1]))
    assert pa.pa_read_device_errors() == 0


def test_beam_search_workload_full_size(pa):
    """The benchmark's beam-search workload at full size, in its launch
    configuration (run_beam_step): the library host pool's prompt tables
    equal the oracle pool's; over 6 device steps the tables, slots and pairs
    equal the oracle's beam_step; the caches equal the oracle's byte copies;
    the last step's decode (all 128 beams, all heads) matches the oracle."""
    from oracle.block_pool import fork
    from paged_kv_cache_340_b200.batch import build_beam_batch, run_beam_step
    from paged_kv_cache_340_b200.workloads import SPECS, make_beam_inputs
    spec = SPECS["beam_search_fp16"]
    inp = make_beam_inputs(spec)
    b = build_beam_batch(spec, inp)
    P, B, bs = spec.num_prompts, spec.branches, spec.block_size
    mb = b.tables[0].shape[1]
    opool = OPool(b.num_blocks, bs, policy="fifo", free_order=inp["free_order"].tolist())
    ob = []
    for p in range(P):
        root = Sequence()
        append_tokens(opool, root, int(inp["prompt_lens"][p]))
        ob += [root] + [fork(opool, root) for _ in range(B - 1)]
    assert b.host_tables.tolist() == _tables(ob, mb).tolist()
    _assert_same_state(b.pool, opool)
    k_or, v_or = raw(inp["k_pool"]).copy(), raw(inp["v_pool"]).copy()
    for i in range(6):
        run_beam_step(b)
        torch.cuda.synchronize()
        k = i % inp["parents"].shape[0]
        ob, oslots, ocow = beam_step(opool, ob, inp["parents"][k].tolist())
        if ocow:
            oracle.copy_blocks(k_or, v_or, np.array(ocow, np.int64))
        oracle.reshape_and_cache(k_or, v_or, raw(inp["new_key"][k]), raw(inp["new_value"][k]), np.array(oslots))
        dst = (i + 1) % 2
        assert b.tables[dst].cpu().numpy().tolist() == _tables(ob, mb).tolist(), i
        assert b.slot_mapping.cpu().tolist() == oslots
        n = int(b.num_cow.item())
        assert n == len(ocow) and [tuple(x) for x in b.cow_pairs[:n].cpu().tolist()] == ocow
    assert pa.pa_read_device_errors() == 0
    _assert_same_state(b.pool, opool)
    assert np.array_equal(raw(b.k_cache), k_or) and np.array_equal(raw(b.v_cache), v_or)
    ref = oracle.paged_decode(f64(inp["query"][5]), _f64_of(k_or, torch.float16), _f64_of(v_or, torch.float16),
                              _tables(ob, mb), np.array([s.num_tokens for s in ob], np.int32), spec.scale, bs)
    assert_attention_close(b.out, ref, torch.float16, "beam workload decode")


@pytest.mark.parametrize("policy", ["fifo", "lifo"])
def test_beam_step_release_all_and_empty_beams(pa, policy):
    """No new beams (every old beam released: all their blocks return to the
    free list in release order), then new beams from an empty parent (context
    0: the token takes a fresh block)."""
    opool, dpool, beams = _start(pa, 64, 4, policy, [9, 4, 13, 1], seed=5)
    ob = [Sequence(list(b.block_table), b.num_tokens) for b in beams]
    new, slots, cow = beam_step(opool, ob, [])
    dev = "cuda"
    old_t = torch.from_numpy(_tables(beams, 8)).to(dev)
    old_c = torch.tensor([b.num_tokens for b in beams], dtype=torch.int32, device=dev)
    empty_i = torch.empty(0, dtype=torch.int32, device=dev)
    ncow = torch.full((1,), -5, dtype=torch.int32, device=dev)
    pa.pa_beam_step(dpool, old_t, old_c, empty_i, torch.empty((0, 8), dtype=torch.int32, device=dev), empty_i,
                    empty_i, torch.empty((0, 2), dtype=torch.int64, device=dev), ncow)
    torch.cuda.synchronize()
    assert new == [] and int(ncow.item()) == 0
    _assert_same_state(dpool, opool)
    assert dpool.ref.cpu().tolist() == [0] * 64
    # a context-0 beam forked twice: both take a fresh block for position 0
    zero = [Sequence([], 0)]
    ob = [Sequence([], 0)]
    new, slots, cow = beam_step(opool, ob, [0, 0])
    t, c, s_, cw, n = _device_step(pa, dpool, zero, [0, 0], 8)
    assert t.tolist() == _tables(new, 8).tolist() and s_.tolist() == slots and n == 0 == len(cow)
    assert c.tolist() == [1, 1]
    _assert_same_state(dpool, opool)
    assert pa.pa_read_device_errors() == 0


@pytest.mark.parametrize("policy", ["fifo", "lifo"])
def test_many_beams_matches_oracle(pa, policy):
    """Steps with more new beams (1100-1300) than the one-launch form serves
    (1024): the four-launch form, against the oracle, and a step after it
    with few beams (the one-launch form) on the state it left."""
    rng = np.random.default_rng(17)
    bs, mb = 16, 24
    lengths = [int(x) for x in rng.integers(1, 200, size=40)]
    opool, dpool, beams = _start(pa, 6000, bs, policy, lengths, seed=5)
    for step, w in enumerate((1100, 1300, 12, 1200)):
        parents = [int(rng.integers(len(beams))) for _ in range(w)]
        ob = [Sequence(list(b.block_table), b.num_tokens) for b in beams]
        new, slots, cow = beam_step(opool, ob, parents)
        t, c, s, cw, n = _device_step(pa, dpool, beams, parents, mb)
        assert t.tolist() == _tables(new, mb).tolist(), step
        assert c.tolist() == [b.num_tokens for b in new]
        assert s.tolist() == slots
        assert n == len(cow) and [tuple(x) for x in cw[:n].tolist()] == cow
        _assert_same_state(dpool, opool)
        beams = new
    assert pa.pa_read_device_errors() == 0
