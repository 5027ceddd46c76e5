"""The bounded pipeline waits on the GPU. A copy that never lands must not
hang the GPU: the waiting warp gives up after its bound, records
PA_DEVERR_TIMEOUT, waits (again bounded) for the copies it still has in flight
and leaves, and the launch ends. pa_decode_withhold_stage (decode: one 16-token
stage) and pa_prefill_withhold_tile (prefill: one 64-token K tile) plant that
fault from the host, with a bound of a few milliseconds, so the test makes the
wait run out and checks what the host reads back; nothing faults or traps.

After such a launch, every other (sequence, kv head) of a decode, and every
other CTA's rows of a prefill, still match the oracle, and the next normal
call is clean."""
import math
import time

import numpy as np
import pytest
import torch

import oracle
from _helpers import assert_attention_close, f64, oracle_decode_tables

pytestmark = pytest.mark.gpu

LIMIT_NS = 5_000_000  # 5 ms


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_340_b200 import _build
    _build.build()
    import paged_kv_cache_340_b200 as pa
    return pa


def _problem(dtype, Hq, Hkv, D, BS, ctx, seed):
    g = torch.Generator().manual_seed(seed)
    ctx = np.array(ctx, np.int32)
    NB = sum(oracle.blocks_needed(int(c), BS) for c in ctx) + 2
    order = torch.randperm(NB, generator=g).numpy().astype(np.int32)
    tables, _ = oracle_decode_tables(ctx, NB, BS, order)
    k = torch.randn((NB, Hkv, BS, D), generator=g).to(dtype)
    v = torch.randn((NB, Hkv, BS, D), generator=g).to(dtype)
    q = torch.randn((len(ctx), Hq, D), generator=g).to(dtype)
    ref = oracle.paged_decode(f64(q), f64(k), f64(v), tables, ctx, 1.0 / math.sqrt(D), BS)
    dev = dict(q=q.cuda(), k=k.cuda(), v=v.cuda(), bt=torch.from_numpy(tables).cuda(), cl=torch.from_numpy(ctx).cuda())
    return dev, ref


@pytest.mark.parametrize("dtype,Hq,Hkv,D,BS", [(torch.float16, 4, 4, 128, 16),     # CUDA-core consumer
                                               (torch.bfloat16, 8, 2, 128, 32),    # tensor-core consumer
                                               (torch.float32, 2, 2, 64, 16)])
def test_withheld_copy_times_out_and_reports(pa, dtype, Hq, Hkv, D, BS):
    ctx = [300, 129, 70, 1000]
    p, ref = _problem(dtype, Hq, Hkv, D, BS, ctx, seed=7)
    out_dt = torch.float32 if dtype == torch.bfloat16 else dtype
    scale = 1.0 / math.sqrt(D)
    assert pa.pa_read_device_errors() == 0
    seq, kvh = 1, Hkv - 1
    for stage in (0, 5):  # a stage of the prologue, and one reloaded in the loop
        out = torch.full((len(ctx), Hq, D), float("nan"), dtype=out_dt, device="cuda")
        t = time.perf_counter()
        pa.pa_decode_withhold_stage(out, p["q"], p["k"], p["v"], p["bt"], p["cl"], scale, seq, kvh, stage, LIMIT_NS)
        torch.cuda.synchronize()
        wall = time.perf_counter() - t
        assert pa.pa_read_device_errors() == pa.PA_DEVERR_TIMEOUT
        assert wall < 2.0  # two bounded waits of 5 ms, not the default 1 s bound, and never a hang
        G = Hq // Hkv
        mask = np.ones((len(ctx), Hq), bool)
        mask[seq, kvh * G:(kvh + 1) * G] = False
        o = out.double().cpu().numpy()
        assert_attention_close(torch.from_numpy(o[mask]).to(out_dt), ref[mask], dtype, f"stage {stage}")
    # the next normal call on the same context: clean and correct
    out = torch.empty((len(ctx), Hq, D), dtype=out_dt, device="cuda")
    pa.pa_decode(out, p["q"], p["k"], p["v"], p["bt"], p["cl"], scale)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    assert_attention_close(out, ref, dtype, "after the timeouts")


def test_stage_past_the_end_withholds_nothing(pa):
    p, ref = _problem(torch.float16, 4, 2, 128, 16, [40, 17], seed=8)
    out = torch.empty((2, 4, 128), dtype=torch.float16, device="cuda")
    out2 = torch.empty_like(out)
    pa.pa_decode_withhold_stage(out, p["q"], p["k"], p["v"], p["bt"], p["cl"], 0.1, 0, 0, 3, LIMIT_NS)
    pa.pa_decode(out2, p["q"], p["k"], p["v"], p["bt"], p["cl"], 0.1)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    assert torch.equal(out, out2)


def test_hook_arguments_are_checked(pa):
    p, _ = _problem(torch.float16, 4, 2, 128, 16, [40, 17], seed=8)
    out = torch.empty((2, 4, 128), dtype=torch.float16, device="cuda")
    for seq, kvh, stage, lim in ((2, 0, 0, LIMIT_NS), (0, 2, 0, LIMIT_NS), (0, 0, -1, LIMIT_NS), (0, 0, 0, 10),
                                 (0, 0, 0, 2_000_000_000)):
        with pytest.raises(pa.PagedAttentionError) as e:
            pa.pa_decode_withhold_stage(out, p["q"], p["k"], p["v"], p["bt"], p["cl"], 0.1, seq, kvh, stage, lim)
        assert e.value.status == -3


# ---- prefill (the tcgen05 kernel): a withheld K tile

def _prefill_problem(dtype, ctx, qlen, Hq, Hkv, BS, seed, D=128):
    g = torch.Generator().manual_seed(seed)
    S = len(ctx)
    nb = [oracle.blocks_needed(int(c), BS) for c in ctx]
    NB = sum(nb) + 3
    ids = torch.randperm(NB, generator=g).numpy().astype(np.int32)
    tables = np.full((S, max(nb)), -1, np.int32)
    pos = 0
    for s, n in enumerate(nb):
        tables[s, :n] = ids[pos:pos + n]
        pos += n
    k = torch.randn((NB, Hkv, BS, D), generator=g).to(dtype)
    v = torch.randn((NB, Hkv, BS, D), generator=g).to(dtype)
    qs = np.concatenate([[0], np.cumsum(qlen)]).astype(np.int32)
    q = torch.randn((int(qs[-1]), Hq, D), generator=g).to(dtype)
    ctx = np.array(ctx, np.int32)
    scale = 1.0 / math.sqrt(D)
    ref = oracle.paged_prefill(f64(q), qs, f64(k), f64(v), tables, ctx, scale, BS)
    dev = dict(q=q.cuda(), k=k.cuda(), v=v.cuda(), qs=torch.from_numpy(qs).cuda(), bt=torch.from_numpy(tables).cuda(),
               cl=torch.from_numpy(ctx).cuda(), max_q=int(max(qlen)), scale=scale, qs_host=qs)
    return dev, ref


def _cta_rows(qs, seq, kvh, qt, Hq, Hkv):
    """(token rows, heads) of the prefill CTA (sequence, kv head, query tile):
    128 (token, head slot) rows, the head group rounded up to a power of two."""
    G = Hq // Hkv
    slots = 1 << (G - 1).bit_length()
    tok_per_tile = 128 // slots
    t0 = int(qs[seq]) + qt * tok_per_tile
    t1 = min(int(qs[seq + 1]), t0 + tok_per_tile)
    return slice(t0, t1), slice(kvh * G, (kvh + 1) * G)


# query tile qt of sequence 0 (300 new tokens from an empty cache) sees four
# 64-key tiles: tokens 128..255 at head group 1, tokens 192..223 at group 4
@pytest.mark.parametrize("dtype,Hq,Hkv,BS,qt", [(torch.bfloat16, 4, 4, 16, 1),   # group 1: rows staged in shared memory
                                                (torch.float16, 16, 4, 32, 6)])  # group 4: rows stored directly
def test_prefill_withheld_tile_times_out_and_reports(pa, dtype, Hq, Hkv, BS, qt):
    ctx, qlen = [300, 200, 90], [300, 64, 90]
    p, ref = _prefill_problem(dtype, ctx, qlen, Hq, Hkv, BS, seed=11)
    T = int(p["qs_host"][-1])
    assert pa.pa_read_device_errors() == 0
    seq, kvh = 0, Hkv - 1
    for tile in (0, 3):  # a tile of the prologue (S_0), and one loaded in the loop
        out = torch.full((T, Hq, 128), float("nan"), dtype=torch.float32, device="cuda")
        t = time.perf_counter()
        pa.pa_prefill_withhold_tile(out, p["q"], p["qs"], p["max_q"], p["k"], p["v"], p["bt"], p["cl"], p["scale"],
                                    seq, kvh, qt, tile, LIMIT_NS)
        torch.cuda.synchronize()
        wall = time.perf_counter() - t
        assert pa.pa_read_device_errors() == pa.PA_DEVERR_TIMEOUT
        assert wall < 2.0  # a few bounded waits of 5 ms, not the default 1 s bound, and never a hang
        rows, heads = _cta_rows(p["qs_host"], seq, kvh, qt, Hq, Hkv)
        mask = np.ones((T, Hq), bool)
        mask[rows, heads] = False
        o = out.cpu().numpy()
        assert_attention_close(torch.from_numpy(o[mask]), ref[mask], dtype, f"tile {tile}")
    # the next normal call: clean and correct
    out = torch.empty((T, Hq, 128), dtype=torch.float32, device="cuda")
    pa.pa_prefill(out, p["q"], p["qs"], p["max_q"], p["k"], p["v"], p["bt"], p["cl"], p["scale"])
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    assert_attention_close(out, ref, dtype, "prefill after the timeouts")


def test_prefill_tile_past_the_work_withholds_nothing(pa):
    p, _ = _prefill_problem(torch.bfloat16, [300, 64], [300, 64], 8, 4, 16, seed=12)
    T = int(p["qs_host"][-1])
    out = torch.empty((T, 8, 128), dtype=torch.float32, device="cuda")
    out2 = torch.empty_like(out)
    # sequence 1's single query tile covers 64 keys: its tile 1 and a query tile 3 do not exist
    for seq, qt, tile in ((1, 0, 1), (1, 3, 0)):
        pa.pa_prefill_withhold_tile(out, p["q"], p["qs"], p["max_q"], p["k"], p["v"], p["bt"], p["cl"], p["scale"],
                                    seq, 0, qt, tile, LIMIT_NS)
        pa.pa_prefill(out2, p["q"], p["qs"], p["max_q"], p["k"], p["v"], p["bt"], p["cl"], p["scale"])
        torch.cuda.synchronize()
        assert pa.pa_read_device_errors() == 0
        assert torch.equal(out, out2)


def test_prefill_hook_arguments_are_checked(pa):
    p, _ = _prefill_problem(torch.float16, [40, 17], [40, 17], 4, 2, 16, seed=13)
    out = torch.empty((57, 4, 128), dtype=torch.float32, device="cuda")
    for seq, kvh, qt, tile, lim in ((2, 0, 0, 0, LIMIT_NS), (0, 2, 0, 0, LIMIT_NS), (0, 0, -1, 0, LIMIT_NS),
                                    (0, 0, 0, -1, LIMIT_NS), (0, 0, 0, 0, 10), (0, 0, 0, 0, 2_000_000_000)):
        with pytest.raises(pa.PagedAttentionError) as e:
            pa.pa_prefill_withhold_tile(out, p["q"], p["qs"], p["max_q"], p["k"], p["v"], p["bt"], p["cl"],
                                        p["scale"], seq, kvh, qt, tile, lim)
        assert e.value.status == -3
    k32, v32 = p["k"].float(), p["v"].float()
    q32 = p["q"].float()
    with pytest.raises(pa.PagedAttentionError) as e:  # fp32 caches run on the CUDA cores: no hook there
        pa.pa_prefill_withhold_tile(out, q32, p["qs"], p["max_q"], k32, v32, p["bt"], p["cl"], p["scale"],
                                    0, 0, 0, 0, LIMIT_NS)
    assert e.value.status == -2
    p64, _ = _prefill_problem(torch.float16, [40, 17], [40, 17], 4, 2, 16, seed=14, D=64)
    out64 = torch.empty((57, 4, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(pa.PagedAttentionError) as e:  # the hook's instances are head_dim 128 only
        pa.pa_prefill_withhold_tile(out64, p64["q"], p64["qs"], p64["max_q"], p64["k"], p64["v"], p64["bt"], p64["cl"],
                                    p64["scale"], 0, 0, 0, 0, LIMIT_NS)
    assert e.value.status == -5


# ---- beam step (one cooperative launch): a CTA that never reaches the first grid barrier

def _beam_setup(pa, nb, bs, lengths, seed):
    from oracle.block_pool import BlockPool as OPool, Sequence, append_tokens
    order = np.random.default_rng(seed).permutation(nb).astype(np.int32)
    opool = OPool(nb, bs, policy="fifo", free_order=order.tolist())
    hpool = pa.BlockPool(nb, bs, pa.PA_POOL_FIFO, free_order=order)
    beams = []
    for n in lengths:
        s = Sequence()
        append_tokens(opool, s, n)
        beams.append(s)
        tab = np.full(nb, -1, np.int32)
        hpool.append(tab, 0, n)
    return opool, hpool, beams


def _beam_args(beams, parents, mb):
    tabs = np.full((len(beams), mb), -1, np.int32)
    for i, b in enumerate(beams):
        tabs[i, :len(b.block_table)] = b.block_table
    n = len(parents)
    return dict(old_t=torch.from_numpy(tabs).cuda(),
                old_c=torch.tensor([b.num_tokens for b in beams], dtype=torch.int32, device="cuda"),
                par=torch.tensor(parents, dtype=torch.int32, device="cuda"),
                new_t=torch.full((n, mb), 7777, dtype=torch.int32, device="cuda"),
                new_c=torch.full((n,), -5, dtype=torch.int32, device="cuda"),
                slots=torch.full((n,), -5, dtype=torch.int32, device="cuda"),
                cow=torch.full((n, 2), -5, dtype=torch.int64, device="cuda"),
                ncow=torch.full((1,), -5, dtype=torch.int32, device="cuda"))


def test_beam_barrier_wait_times_out_and_marks_the_state(pa):
    from oracle.block_pool import beam_step
    nb, bs, mb = 600, 16, 24
    rng = np.random.default_rng(21)
    lengths = [int(x) for x in rng.integers(1, 300, 40)]          # 40 beams x 24 entries: 4 CTAs of 256
    parents = [int(x) for x in rng.integers(0, 40, 40)]
    opool, hpool, beams = _beam_setup(pa, nb, bs, lengths, seed=21)
    dpool = pa.DevicePool(nb, bs, pa.PA_POOL_FIFO, host_pool=hpool)
    h = pa.PA_DPOOL_HEADER_WORDS
    before = torch.cat([dpool.state[:5], dpool.state[h:h + 6 * nb]]).clone()
    assert int(dpool.state[5].item()) != 0 and pa.pa_read_device_errors() == 0
    a = _beam_args(beams, parents, mb)
    t = time.perf_counter()
    pa.pa_beam_step_withhold_arrival(dpool, a["old_t"], a["old_c"], a["par"], a["new_t"], a["new_c"], a["slots"],
                                     a["cow"], a["ncow"], 2, LIMIT_NS)
    torch.cuda.synchronize()
    wall = time.perf_counter() - t
    assert wall < 2.0  # bounded waits of 5 ms, not the default 200 ms, and never a hang
    assert pa.pa_read_device_errors() & pa.PA_DEVERR_TIMEOUT
    assert (a["slots"].cpu().numpy() == -1).all() and int(a["ncow"].item()) == 0
    # nothing applied; the state is marked unusable (header word 5)
    assert torch.equal(torch.cat([dpool.state[:5], dpool.state[h:h + 6 * nb]]), before)
    assert int(dpool.state[5].item()) == 0
    # reloaded from the host pool, the same step runs clean and matches the oracle
    dpool = pa.DevicePool(nb, bs, pa.PA_POOL_FIFO, host_pool=hpool)
    a = _beam_args(beams, parents, mb)
    pa.pa_beam_step(dpool, a["old_t"], a["old_c"], a["par"], a["new_t"], a["new_c"], a["slots"], a["cow"], a["ncow"])
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    children, slots, cow = beam_step(opool, beams, parents)
    assert a["slots"].cpu().tolist() == slots
    assert int(a["ncow"].item()) == len(cow)
    assert a["cow"].cpu().numpy()[:len(cow)].tolist() == [list(c) for c in cow]
    assert dpool.ref.cpu().tolist() == opool.ref_counts and dpool.free_list() == opool.free_blocks


def test_beam_hook_arguments_are_checked(pa):
    opool, hpool, beams = _beam_setup(pa, 64, 16, [20, 5], seed=22)
    dpool = pa.DevicePool(64, 16, pa.PA_POOL_FIFO, host_pool=hpool)
    a = _beam_args(beams, [0, 1], 4)
    for cta, lim in ((-1, LIMIT_NS), (0, 10), (0, 2_000_000_000)):
        with pytest.raises(pa.PagedAttentionError) as e:
            pa.pa_beam_step_withhold_arrival(dpool, a["old_t"], a["old_c"], a["par"], a["new_t"], a["new_c"],
                                             a["slots"], a["cow"], a["ncow"], cta, lim)
        assert e.value.status == -3
    # a CTA past the launch withholds nothing: the step is pa_beam_step's
    pa.pa_beam_step_withhold_arrival(dpool, a["old_t"], a["old_c"], a["par"], a["new_t"], a["new_c"], a["slots"],
                                     a["cow"], a["ncow"], 50, LIMIT_NS)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    from oracle.block_pool import beam_step
    _, slots, _ = beam_step(opool, beams, [0, 1])
    assert a["slots"].cpu().tolist() == slots
