"""Host-side checks that need no GPU: the shared library loads and exports
every function include/pa.h declares; host argument checks return their
status codes before touching the device; the library's C++ block pool makes
exactly the decisions of the oracle's pool."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_340_b200 import _build
    _build.build()
    import paged_kv_cache_340_b200 as pa
    return pa


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[a-z_ ]*?[\w\s\*]+?\b(pa_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_library_exports_every_declared_function(pa):
    declared = _declared_functions()
    assert len(declared) >= 20
    lib = ctypes.CDLL(pa.LIB_PATH)
    missing = [n for n in declared if not hasattr(lib, n)]
    assert not missing, missing
    assert sorted(pa.EXPORTED) == declared


def test_status_strings(pa):
    for code in range(0, -14, -1):
        s = pa.status_string(code)
        assert s and s != "unknown status"
    assert pa.status_string(-99) == "unknown status"


def test_workspace_layout(pa):
    S, H, D, L, P = 3, 8, 128, 1000, 256
    mp = 4
    off = pa.pa_splitk_acc_offset(S, H, L, P)
    assert off >= S * H * mp * 2 * 4 and off % 256 == 0
    assert pa.pa_splitk_workspace_bytes(S, H, D, L, P) == off + S * H * mp * D * 4


def test_choose_partition(pa):
    import torch
    # many (seq, kv head) items: no split
    assert pa.pa_choose_partition(256, 8, 4096, 16, 128, torch.bfloat16) == 0
    # few long sequences: split, multiple of the block size, shorter than the context
    P = pa.pa_choose_partition(8, 8, 131072, 32, 128, torch.bfloat16)
    assert P > 0 and P % 32 == 0 and P < 131072


A16 = 1 << 20  # a fake 16-byte aligned address; never dereferenced by these calls


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), -5),
    (dict(block_size=8), -6),
    (dict(num_heads=12, num_kv_heads=8), -4),
    (dict(num_heads=16 * 65535, num_kv_heads=65535), -3),   # head group 16: two CTAs per kv head, past gridDim.y
    (dict(kv_dtype=7), -2),
    (dict(out_dtype=1, kv_dtype=2), -2),
    (dict(num_seqs=-1), -3),
    (dict(query=A16 + 8), -7),
    (dict(k_cache=0), -1),
])
def test_decode_host_checks(pa, kw, code):
    args = dict(out=A16, query=A16, k_cache=A16, v_cache=A16, block_tables=A16, max_blocks=4, context_lens=A16,
                num_seqs=2, num_heads=8, num_kv_heads=8, head_dim=128, scale=0.1, block_size=16, num_blocks=8,
                kv_dtype=1, out_dtype=1)
    args.update(kw)
    rc = pa._lib.pa_decode(args["out"], args["query"], args["k_cache"], args["v_cache"], args["block_tables"],
                           args["max_blocks"], args["context_lens"], args["num_seqs"], args["num_heads"],
                           args["num_kv_heads"], args["head_dim"], args["scale"], args["block_size"],
                           args["num_blocks"], args["kv_dtype"], args["out_dtype"], None, None)
    assert rc == code


@pytest.mark.parametrize("new_key,new_value,code", [
    (0, A16, -1),            # no new key rows
    (A16, 0, -1),
    (A16 + 8, A16, -7),      # rows not 16-byte aligned
    (A16, A16 + 4, -7),
])
def test_decode_append_host_checks(pa, new_key, new_value, code):
    rc = pa._lib.pa_decode_append(A16, A16, new_key, new_value, A16, A16, A16, 4, A16, 2, 8, 8, 128, 0.1, 16, 8,
                                  1, 1, None, None)
    assert rc == code
    # the checks of pa_decode apply as well
    assert pa._lib.pa_decode_append(A16, A16, A16, A16, A16, A16, A16, 4, A16, 2, 8, 8, 96, 0.1, 16, 8,
                                    1, 1, None, None) == -5
    # an empty batch needs no rows
    assert pa._lib.pa_decode_append(None, None, None, None, None, None, None, 0, None, 0, 8, 8, 128, 0.1, 16, 0,
                                    1, 1, None, None) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), -5),
    (dict(kv_dtype=0, out_dtype=1), -2),           # fp32 caches prefill into fp32 outputs
    (dict(kv_dtype=0, out_dtype=0, head_dim=96), -5),
    (dict(kv_dtype=0, out_dtype=0, query=A16 + 4), -7),
    (dict(out_dtype=1, kv_dtype=2), -2),
    (dict(block_size=8), -6),
    (dict(num_heads=12, num_kv_heads=8), -4),
    (dict(num_heads=256 * 65535, num_kv_heads=65535), -3),   # two sub-groups of 128 per kv head, past gridDim.y
    (dict(num_seqs=-1), -3),
    (dict(query=0), -1),
    (dict(q_start=A16 + 2), -7),
    (dict(out=A16 + 8), -7),
    (dict(num_blocks=1 << 27, num_kv_heads=8, num_heads=8), -3),   # pool rows past int32
    (dict(max_q_len=1 << 29, num_heads=32, num_kv_heads=4), -3),   # query tile index past int32
    (dict(num_tokens=0), 0),                       # nothing to do
])
def test_prefill_host_checks(pa, kw, code):
    a = dict(out=A16, query=A16, q_start=A16, num_tokens=40, max_q_len=20, k_cache=A16, v_cache=A16,
             block_tables=A16, max_blocks=4, context_lens=A16, num_seqs=2, num_heads=8, num_kv_heads=8,
             head_dim=128, scale=0.1, block_size=16, num_blocks=8, kv_dtype=2, out_dtype=0)
    a.update(kw)
    rc = pa._lib.pa_prefill(a["out"], a["query"], a["q_start"], a["num_tokens"], a["max_q_len"], a["k_cache"],
                            a["v_cache"], a["block_tables"], a["max_blocks"], a["context_lens"], a["num_seqs"],
                            a["num_heads"], a["num_kv_heads"], a["head_dim"], a["scale"], a["block_size"],
                            a["num_blocks"], a["kv_dtype"], a["out_dtype"], None)
    assert rc == code


@pytest.mark.parametrize("kw,code", [
    (dict(q_dtype=0), -2),                         # the query is 16-bit
    (dict(k_scale=0), -1),
    (dict(v_scale=A16 + 4), -7),
    (dict(out_dtype=2), -2),                       # fp16 query, bf16 output
    (dict(head_dim=96), -5),
    (dict(num_seqs=0), 0),
])
def test_decode_q8_host_checks(pa, kw, code):
    a = dict(out=A16, query=A16, q_dtype=1, k_cache=A16, v_cache=A16, k_scale=A16, v_scale=A16, block_tables=A16,
             max_blocks=4, context_lens=A16, num_seqs=2, num_heads=8, num_kv_heads=2, head_dim=128, scale=0.1,
             block_size=16, num_blocks=8, out_dtype=1)
    a.update(kw)
    rc = pa._lib.pa_decode_q8(a["out"], a["query"], a["q_dtype"], a["k_cache"], a["v_cache"], a["k_scale"],
                              a["v_scale"], a["block_tables"], a["max_blocks"], a["context_lens"], a["num_seqs"],
                              a["num_heads"], a["num_kv_heads"], a["head_dim"], a["scale"], a["block_size"],
                              a["num_blocks"], a["out_dtype"], None, None)
    assert rc == code


def test_slot_write_and_copy_host_checks(pa):
    lib = pa._lib
    # pa_reshape_and_cache(key, value, k_cache, v_cache, slots, T, NB, Hkv, D, bs, dtype, stream)
    w = [A16, A16, A16, A16, A16, 4, 8, 2, 128, 16, 1, None]

    def w_(**kw):
        a = list(w)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return lib.pa_reshape_and_cache(*a)
    assert w_(a8=96) == -5 and w_(a9=8) == -6 and w_(a10=7) == -2 and w_(a5=-1) == -3
    assert w_(a4=0) == -1 and w_(a4=A16 + 2) == -7 and w_(a0=A16 + 8) == -7
    assert w_(a6=1 << 27, a9=32) == -3                     # slots past int32
    # pa_reshape_and_cache_q8(key, value, src_dtype, kq, vq, ks, vs, slots, T, NB, Hkv, D, bs, stream)
    q = [A16, A16, 1, A16, A16, A16, A16, A16, 4, 8, 2, 128, 16, None]

    def q_(**kw):
        a = list(q)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return lib.pa_reshape_and_cache_q8(*a)
    assert q_(a2=9) == -2 and q_(a11=32) == -5 and q_(a12=64) == -6
    assert q_(a5=0) == -1 and q_(a6=A16 + 4) == -7 and q_(a8=0) == 0
    # pa_copy_blocks(k_cache, v_cache, pairs, n, NB, Hkv, D, bs, dtype, stream)
    c = [A16, A16, A16, 3, 8, 2, 128, 16, 1, None]

    def c_(**kw):
        a = list(c)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return lib.pa_copy_blocks(*a)
    assert c_(a6=80) == -5 and c_(a7=48) == -6 and c_(a8=5) == -2 and c_(a3=-2) == -3
    assert c_(a2=0) == -1 and c_(a2=A16 + 4) == -7 and c_(a3=0) == 0


def test_empty_batches_are_no_ops(pa):
    assert pa._lib.pa_decode(None, None, None, None, None, 0, None, 0, 8, 8, 128, 0.1, 16, 0, 1, 1, None, None) == 0
    assert pa._lib.pa_reshape_and_cache(None, None, None, None, None, 0, 4, 8, 128, 16, 1, None) == 0
    assert pa._lib.pa_copy_blocks(None, None, None, 0, 4, 8, 128, 16, 1, None) == 0


def test_splitk_host_checks(pa):
    f = pa._lib.pa_decode_splitk
    base = [A16, 1 << 30, A16, A16, A16, A16, 4, A16, 2, 8, 8, 128, 0.1, 16, 8, 64]
    assert f(*(base + [24, 1, None, None])) == -8       # partition not a multiple of the block size
    assert f(*(base + [0, 1, None, None])) == -8
    small = list(base)
    small[1] = 16
    assert f(*(small + [32, 1, None, None])) == -9      # workspace too small
    nows = list(base)
    nows[0] = None
    assert f(*(nows + [32, 1, None, None])) == -9
    assert f(*(base + [32, 1, A16 + 2, None])) == -7    # misaligned schedule


# ------------------------------------------------------ pool vs oracle pool

def _same_pool_state(pool, opool):
    assert pool.num_free() == opool.num_free()
    for b in range(opool.num_blocks):
        assert pool.ref_count(b) == opool.ref_counts[b]


@pytest.mark.parametrize("policy", ["fifo", "lifo"])
def test_pool_matches_oracle_random_ops(pa, policy):
    from oracle.block_pool import BlockPool as OPool, Sequence, append_tokens, fork, release
    rng = np.random.default_rng(5 if policy == "fifo" else 6)
    NB, bs, MB = 96, 16, 24
    order = rng.permutation(NB)
    pol = pa.PA_POOL_FIFO if policy == "fifo" else pa.PA_POOL_LIFO
    pool = pa.BlockPool(NB, bs, pol, free_order=order)
    opool = OPool(NB, bs, policy=policy, free_order=order.tolist())
    seqs = []  # (table, num_tokens, oracle Sequence)
    for step in range(400):
        op = rng.integers(0, 10)
        if op < 5 or not seqs:
            if op < 5 and seqs:
                i = int(rng.integers(len(seqs)))
            else:
                seqs.append([np.full(MB, -1, np.int32), 0, Sequence()])
                i = len(seqs) - 1
            tab, nt, oseq = seqs[i]
            n = int(rng.integers(1, 40))
            if opool.num_free() < n // bs + 2 or nt + n > MB * bs:
                continue
            nt2, slots, cow = pool.append(tab, nt, n)
            oslots, ocow = append_tokens(opool, oseq, n)
            assert nt2 == oseq.num_tokens
            assert slots.tolist() == oslots
            assert [tuple(x) for x in cow.tolist()] == ocow
            assert tab[: len(oseq.block_table)].tolist() == oseq.block_table
            seqs[i][1] = nt2
        elif op < 8:
            i = int(rng.integers(len(seqs)))
            tab, nt, oseq = seqs[i]
            dst = np.full(MB, -1, np.int32)
            pool.fork(tab, nt, dst)
            seqs.append([dst, nt, fork(opool, oseq)])
        else:
            i = int(rng.integers(len(seqs)))
            tab, nt, oseq = seqs.pop(i)
            pool.release(tab, nt)
            release(opool, oseq)
        _same_pool_state(pool, opool)


def test_pool_errors(pa):
    pool = pa.BlockPool(2, 4, pa.PA_POOL_FIFO)
    tab = np.full(4, -1, np.int32)
    nt, _, _ = pool.append(tab, 0, 8)
    with pytest.raises(pa.PagedAttentionError) as e:
        pool.append(tab, nt, 1)
    assert e.value.status == -11
    with pytest.raises(pa.PagedAttentionError):
        pool.free(5)
    with pytest.raises(pa.PagedAttentionError):
        pa.BlockPool(3, 4, pa.PA_POOL_FIFO, free_order=[0, 0, 1])
    small = np.full(1, -1, np.int32)
    pool2 = pa.BlockPool(4, 4, pa.PA_POOL_FIFO)
    with pytest.raises(pa.PagedAttentionError) as e:
        pool2.append(small, 0, 5)
    assert e.value.status == -13


def test_device_pool_host_checks(pa):
    """pa_dpool_* / pa_beam_step / pa_copy_blocks_counted argument checks
    return before any device work (fake device addresses are never touched)."""
    lib = pa._lib
    assert lib.pa_dpool_state_bytes(10) == (pa.PA_DPOOL_HEADER_WORDS + 6 * 10 + pa.PA_DPOOL_TAIL_WORDS) * 4
    assert lib.pa_dpool_state_bytes(0) == 0
    fake = 1 << 40                                       # 16-byte aligned, never dereferenced
    assert lib.pa_dpool_init(None, 10, 16, 0, None, None) == -1
    assert lib.pa_dpool_init(fake, 0, 16, 0, None, None) == -3
    assert lib.pa_dpool_init(fake, 10, 16, 7, None, None) == -3
    assert lib.pa_dpool_init(fake + 4, 10, 16, 0, None, None) == -7
    args = dict(old_t=fake, old_c=fake, par=fake, new_t=fake + 4096, new_c=fake + 8192, slots=fake, cow=fake,
                ncow=fake)

    def step(state=fake, nb=64, bs=16, num_old=2, num_new=2, mb=4, **kw):
        a = dict(args, **kw)
        return lib.pa_beam_step(state, nb, bs, a["old_t"], a["old_c"], num_old, a["par"], num_new, a["new_t"],
                                a["new_c"], mb, a["slots"], a["cow"], a["ncow"], None)
    assert step(state=None) == -1
    assert step(ncow=None) == -1
    assert step(par=None) == -1
    assert step(nb=0) == -3
    assert step(mb=0) == -3
    assert step(num_old=-1) == -3
    assert step(num_old=1 << 12, mb=1 << 18) == -3      # flattened table index past 2^30
    assert step(num_old=20000, num_new=1) == -3           # per-beam values past the shared-memory stage
    assert step(new_t=fake) == -3                        # output tables alias the input tables
    assert step(new_c=fake) == -3                        # output context lengths alias the input ones
    assert step(cow=fake + 4) == -7
    assert lib.pa_copy_blocks_counted(fake, fake, fake, None, 4, 8, 2, 128, 16, 1, None) == -1
    assert lib.pa_copy_blocks_counted(fake, fake, fake, fake, 4, 8, 2, 100, 16, 1, None) == -5
    assert lib.pa_copy_blocks_counted(fake, fake, fake, fake, 0, 8, 2, 128, 16, 1, None) == 0


def test_pool_export_matches_oracle(pa):
    """pa_pool_export returns the counts and the free list (front first) that
    the oracle pool holds after the same operations."""
    from oracle.block_pool import BlockPool as OPool, Sequence, append_tokens, fork, release
    order = np.random.default_rng(5).permutation(40).astype(np.int32)
    for policy, name in ((pa.PA_POOL_FIFO, "fifo"), (pa.PA_POOL_LIFO, "lifo")):
        lp = pa.BlockPool(40, 4, policy, free_order=order)
        op = OPool(40, 4, policy=name, free_order=order.tolist())
        tabs, seqs = [], []
        for n in (9, 4, 13):
            t = np.full(16, -1, np.int32)
            lp.append(t, 0, n)
            s = Sequence()
            append_tokens(op, s, n)
            tabs.append((t, n))
            seqs.append(s)
        child = np.full(16, -1, np.int32)
        lp.fork(tabs[2][0], 13, child)
        fork(op, seqs[2])
        lp.release(tabs[0][0], 9)
        release(op, seqs[0])
        ref, fl = lp.export()
        assert ref.tolist() == op.ref_counts and fl.tolist() == op.free_blocks


def test_host_beam_step_matches_oracle(pa):
    """batch.host_beam_step (the host-pool path the bench compares against)
    makes the oracle's beam_step decisions."""
    from oracle.block_pool import BlockPool as OPool, Sequence, append_tokens, beam_step
    from paged_kv_cache_340_b200.batch import host_beam_step
    rng = np.random.default_rng(8)
    nb, bs, mb = 300, 4, 40
    order = rng.permutation(nb).astype(np.int32)
    lp = pa.BlockPool(nb, bs, pa.PA_POOL_FIFO, free_order=order)
    op = OPool(nb, bs, policy="fifo", free_order=order.tolist())
    beams, tables, ctx = [], np.full((5, mb), -1, np.int32), np.zeros(5, np.int32)
    for i, n in enumerate((7, 12, 1, 30, 9)):
        s = Sequence()
        append_tokens(op, s, n)
        beams.append(s)
        ctx[i], _, _ = lp.append(tables[i], 0, n)
    for _ in range(25):
        parents = rng.integers(0, len(beams), size=int(rng.integers(1, 8))).astype(np.int32)
        beams, slots, cow = beam_step(op, beams, parents.tolist())
        tables, ctx, lslots, lcow = host_beam_step(lp, tables, ctx, parents)
        assert lslots.tolist() == slots and [tuple(x) for x in lcow.tolist()] == cow
        assert ctx.tolist() == [b.num_tokens for b in beams]
        for t, b in zip(tables, beams):
            assert t[:len(b.block_table)].tolist() == b.block_table
    ref, fl = lp.export()
    assert ref.tolist() == op.ref_counts and fl.tolist() == op.free_blocks
