"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

Acceptance: slot writes, block copies, tables and slots bit-exact; attention
max abs error <= 4e-3 and relative L2 <= 1e-3 for fp16/bf16 inputs, max abs
<= 1e-5 for fp32 inputs (bf16 outputs add their own rounding, see
_helpers.assert_attention_close).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from _helpers import assert_attention_close, f64, oracle_decode_tables, raw

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_340_b200 import _build
    _build.build()
    import paged_kv_cache_340_b200 as pa
    torch.cuda.init()
    return pa


def _pool_flow(pa, ctx, NB, BS, order):
    """Tables and newest-token slots from the library's pool (ctx 0 -> no token, slot -1)."""
    mb = max(1, max((int(c) + BS - 1) // BS for c in ctx))
    pool = pa.BlockPool(NB, BS, pa.PA_POOL_FIFO, free_order=order)
    tables = np.full((len(ctx), mb), -1, np.int32)
    slots = np.full(len(ctx), -1, np.int32)
    for s, L in enumerate(ctx):
        if L == 0:
            continue
        nt, _, _ = pool.append(tables[s], 0, int(L) - 1, want_slots=False)
        _, sl, _ = pool.append(tables[s], nt, 1)
        slots[s] = sl[0]
    return tables, slots


class Case:
    """A small decode problem: pools with NaN in every slot no sequence uses,
    a newest token per sequence written by the slot write, and the oracle's
    result."""

    def __init__(self, pa, dtype, S, Hq, Hkv, D, BS, ctx, seed, out_dtype=None, poison=True):
        g = torch.Generator().manual_seed(seed)
        self.dtype, self.BS, self.D, self.Hq, self.Hkv = dtype, BS, D, Hq, Hkv
        self.out_dtype = out_dtype or dtype
        self.ctx = np.array(ctx, np.int32)
        need = sum(oracle.blocks_needed(int(c), BS) for c in ctx)
        self.NB = NB = need + 3
        order = torch.randperm(NB, generator=g).numpy().astype(np.int32)
        kp = torch.randn((NB, Hkv, BS, D), generator=g).to(dtype)
        vp = torch.randn((NB, Hkv, BS, D), generator=g).to(dtype)
        self.q = torch.randn((S, Hq, D), generator=g).to(dtype)
        self.new_k = torch.randn((S, Hkv, D), generator=g).to(dtype)
        self.new_v = torch.randn((S, Hkv, D), generator=g).to(dtype)
        self.scale = 1.0 / math.sqrt(D)
        # oracle side: tables and slots from the oracle pool
        otab = np.full((S, max(1, max(oracle.blocks_needed(int(c), BS) for c in ctx))), -1, np.int32)
        oslots = np.full(S, -1, np.int32)
        live = [s for s in range(S) if ctx[s] > 0]
        if live:
            t, sl = oracle_decode_tables(self.ctx[live], NB, BS, order)
            otab[live, : t.shape[1]] = t
            oslots[live] = sl
        # library side: the same from the library pool -- must agree bit for bit
        tab, slots = _pool_flow(pa, ctx, NB, BS, order)
        assert np.array_equal(tab, otab), "block tables differ from the oracle pool's"
        assert np.array_equal(slots, oslots), "slots differ from the oracle pool's"
        self.tables, self.slots = tab, slots
        if poison:
            used = np.zeros((NB, BS), bool)
            for s, L in enumerate(ctx):
                for t in range(L):
                    used[tab[s, t // BS], t % BS] = True
            nan = torch.tensor(float("nan"), dtype=dtype)
            m = torch.from_numpy(~used)
            kp[m.nonzero(as_tuple=True)[0], :, m.nonzero(as_tuple=True)[1], :] = nan
            vp[m.nonzero(as_tuple=True)[0], :, m.nonzero(as_tuple=True)[1], :] = nan
        self.kp_host, self.vp_host = kp, vp
        # oracle: slot write (bytes) then attention in double
        okp, ovp = raw(kp).copy(), raw(vp).copy()
        oracle.reshape_and_cache(okp, ovp, raw(self.new_k), raw(self.new_v), oslots)
        self.okp, self.ovp = okp, ovp
        self.okp_t = torch.from_numpy(okp).view(dtype)
        self.ovp_t = torch.from_numpy(ovp).view(dtype)
        self.ref = oracle.paged_decode(f64(self.q), self.okp_t.double().numpy(), self.ovp_t.double().numpy(),
                                       tab, self.ctx, self.scale, BS)

    def device(self):
        dev = "cuda"
        return dict(k=self.kp_host.to(dev), v=self.vp_host.to(dev), q=self.q.to(dev),
                    nk=self.new_k.to(dev), nv=self.new_v.to(dev), slots=torch.from_numpy(self.slots).to(dev),
                    bt=torch.from_numpy(self.tables).to(dev), cl=torch.from_numpy(self.ctx).to(dev))


def _run_write_and_decode(pa, c, partition=0):
    d = c.device()
    pa.pa_reshape_and_cache(d["nk"], d["nv"], d["k"], d["v"], d["slots"])
    out = torch.empty((len(c.ctx), c.Hq, c.D), dtype=c.out_dtype, device="cuda")
    if partition:
        mx = int(c.ctx.max())
        ws = torch.empty(pa.pa_splitk_workspace_bytes(len(c.ctx), c.Hq, c.D, mx, partition), dtype=torch.uint8,
                         device="cuda")
        pa.pa_decode_splitk(ws, d["q"], d["k"], d["v"], d["bt"], d["cl"], c.scale, mx, partition)
        pa.pa_splitk_reduce(out, ws, d["cl"], mx, partition)
    else:
        pa.pa_decode(out, d["q"], d["k"], d["v"], d["bt"], d["cl"], c.scale)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    return d, out


SHAPES = [
    # dtype, D, BS, Hq, Hkv
    ("f32", 64, 16, 4, 4),
    ("f32", 128, 32, 8, 2),
    ("f16", 128, 16, 8, 8),
    ("f16", 128, 32, 8, 2),
    ("f16", 64, 16, 8, 1),
    ("f16", 128, 16, 4, 2),
    ("f32", 64, 32, 8, 4),
    ("bf16", 128, 16, 8, 2),
    ("bf16", 128, 32, 16, 4),
    ("bf16", 64, 32, 4, 4),
    ("bf16", 128, 16, 16, 2),
    ("bf16", 64, 32, 8, 4),
]


@pytest.mark.parametrize("dt,D,BS,Hq,Hkv", SHAPES)
@pytest.mark.parametrize("partition", [0, 1, 3])
def test_decode_parity_small(pa, dt, D, BS, Hq, Hkv, partition):
    dtype = DT[dt]
    ctx = [1, BS - 1, BS, BS + 1, 3 * BS + 5, 200, 0, 517]
    c = Case(pa, dtype, len(ctx), Hq, Hkv, D, BS, ctx, seed=7 * D + 3 * BS + Hq + 11 * Hkv + len(dt))
    d, out = _run_write_and_decode(pa, c, partition * BS)
    # slot write: pools bit-exact with the oracle's
    assert np.array_equal(raw(d["k"].cpu()), c.okp)
    assert np.array_equal(raw(d["v"].cpu()), c.ovp)
    assert_attention_close(out, c.ref, dtype, f"{dt} D{D} BS{BS} G{Hq // Hkv} P{partition * BS}")
    assert torch.all(out[6] == 0)  # empty context -> zeros


@pytest.mark.parametrize("dt,out", [("f16", "f32"), ("bf16", "bf16"), ("bf16", "f32")])
def test_output_dtypes(pa, dt, out):
    ctx = [33, 64, 150]
    c = Case(pa, DT[dt], 3, 8, 4, 128, 16, ctx, seed=11, out_dtype=DT[out])
    _, o = _run_write_and_decode(pa, c)
    assert o.dtype == DT[out]
    assert_attention_close(o, c.ref, DT[dt], f"{dt}->{out}")


def test_context_one_is_exact_value_fp32(pa):
    c = Case(pa, torch.float32, 3, 4, 4, 64, 16, [1, 1, 1], seed=3)
    _, out = _run_write_and_decode(pa, c)
    # one token: the weight is exactly 1, so out is that token's value
    assert torch.equal(out.cpu(), c.new_v)


def test_permutation_of_physical_ids_is_bit_invariant(pa):
    ctx = [40, 97, 300, 16]
    c = Case(pa, torch.bfloat16, 4, 8, 2, 128, 16, ctx, seed=4)
    d, out = _run_write_and_decode(pa, c)
    perm = torch.randperm(c.NB, generator=torch.Generator().manual_seed(9))
    k2 = torch.empty_like(d["k"])
    v2 = torch.empty_like(d["v"])
    k2[perm.cuda()] = d["k"]
    v2[perm.cuda()] = d["v"]
    bt2 = torch.where(d["bt"] >= 0, perm.cuda().to(torch.int32)[d["bt"].clamp(min=0).long()], d["bt"])
    out2 = torch.empty_like(out)
    pa.pa_decode(out2, d["q"], k2, v2, bt2.contiguous(), d["cl"], c.scale)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


@pytest.mark.parametrize("partition", [0, 64])
def test_schedule_order_changes_nothing(pa, partition):
    """seq_order only reorders the work: any permutation gives bit-identical
    outputs; an entry outside [0, num_seqs) is skipped and flagged."""
    ctx = [40, 700, 3, 129, 0, 260]
    c = Case(pa, torch.bfloat16, len(ctx), 8, 2, 128, 16, ctx, seed=21, out_dtype=torch.float32)
    d, out = _run_write_and_decode(pa, c, partition)
    for perm in ([5, 4, 3, 2, 1, 0], [1, 5, 3, 0, 2, 4]):
        order = torch.tensor(perm, dtype=torch.int32, device="cuda")
        out2 = torch.empty_like(out)
        if partition:
            mx = int(c.ctx.max())
            ws = torch.empty(pa.pa_splitk_workspace_bytes(len(ctx), 8, 128, mx, partition), dtype=torch.uint8,
                             device="cuda")
            pa.pa_decode_splitk(ws, d["q"], d["k"], d["v"], d["bt"], d["cl"], c.scale, mx, partition,
                                seq_order=order)
            pa.pa_splitk_reduce(out2, ws, d["cl"], mx, partition)
        else:
            pa.pa_decode(out2, d["q"], d["k"], d["v"], d["bt"], d["cl"], c.scale, seq_order=order)
        torch.cuda.synchronize()
        assert pa.pa_read_device_errors() == 0
        assert torch.equal(out, out2)
    if not partition:
        bad = torch.tensor([0, 1, 2, 3, 4, 9], dtype=torch.int32, device="cuda")
        out3 = torch.full_like(out, 7.0)
        pa.pa_decode(out3, d["q"], d["k"], d["v"], d["bt"], d["cl"], c.scale, seq_order=bad)
        assert pa.pa_read_device_errors() & pa.PA_DEVERR_CONTEXT
        assert torch.equal(out3[:5], out[:5]) and torch.all(out3[5] == 7.0)


def test_splitk_partials_match_oracle(pa):
    ctx = [100, 1000, 31, 64]
    P = 128
    c = Case(pa, torch.bfloat16, 4, 8, 2, 128, 32, ctx, seed=5)
    d = c.device()
    pa.pa_reshape_and_cache(d["nk"], d["nv"], d["k"], d["v"], d["slots"])
    mx = int(c.ctx.max())
    ws = torch.zeros(pa.pa_splitk_workspace_bytes(4, 8, 128, mx, P), dtype=torch.uint8, device="cuda")
    pa.pa_decode_splitk(ws, d["q"], d["k"], d["v"], d["bt"], d["cl"], c.scale, mx, P)
    torch.cuda.synchronize()
    ml, acc = pa.splitk_views(ws, 4, 8, 128, mx, P)
    mp = -(-mx // P)
    om, ol, oacc = oracle.splitk_partials(f64(c.q), c.okp_t.double().numpy(), c.ovp_t.double().numpy(), c.tables,
                                          c.ctx, c.scale, 32, P, mp)
    ml, acc = ml.double().cpu().numpy(), acc.double().cpu().numpy()
    for s in range(4):
        n = -(-int(ctx[s]) // P)
        np.testing.assert_allclose(ml[s, :, :n, 0], om[s, :, :n], rtol=0, atol=2e-4)
        np.testing.assert_allclose(ml[s, :, :n, 1], ol[s, :, :n], rtol=2e-4, atol=0)
        np.testing.assert_allclose(acc[s, :, :n], oacc[s, :, :n], rtol=0,
                                   atol=2e-4 * np.abs(oacc[s, :, :n]).max() + 1e-6)


def test_splitk_reduce_on_oracle_partials(pa):
    """The merge kernel alone, fed the oracle's partials (cast to fp32),
    against the oracle's closed-form merge."""
    rng = np.random.default_rng(6)
    S, H, D, P = 3, 4, 128, 64
    ctx = np.array([1, 130, 640], np.int32)
    mx = int(ctx.max())
    mp = -(-mx // P)
    m = rng.normal(size=(S, H, mp)) * 3
    l = rng.uniform(0.5, 40, size=(S, H, mp))
    acc = rng.normal(size=(S, H, mp, D)) * l[..., None]
    m32, l32, acc32 = m.astype(np.float32), l.astype(np.float32), acc.astype(np.float32)
    ref = oracle.splitk_merge(m32.astype(np.float64), l32.astype(np.float64), acc32.astype(np.float64), ctx, P)
    ws = torch.zeros(pa.pa_splitk_workspace_bytes(S, H, D, mx, P), dtype=torch.uint8, device="cuda")
    wml, wacc = pa.splitk_views(ws, S, H, D, mx, P)
    wml[..., 0] = torch.from_numpy(m32).cuda()
    wml[..., 1] = torch.from_numpy(l32).cuda()
    wacc.copy_(torch.from_numpy(acc32).cuda())
    out = torch.empty((S, H, D), dtype=torch.float32, device="cuda")
    pa.pa_splitk_reduce(out, ws, torch.from_numpy(ctx).cuda(), mx, P)
    torch.cuda.synchronize()
    np.testing.assert_allclose(f64(out), ref, rtol=2e-6, atol=2e-6)


def test_splitk_reduce_many_partitions_rising_max(pa):
    """The merge over hundreds of partitions per head, with the partitions'
    maxima rising along the sequence (a random walk with drift) and also
    falling in places, so each warp of the merge kernel folds several batches
    and raises its running maximum between them; against the oracle's
    closed-form merge."""
    rng = np.random.default_rng(61)
    S, H, D, P = 2, 3, 64, 16
    ctx = np.array([P * 300 - 5, P * 97 + 1], np.int32)
    mx = int(ctx.max())
    mp = -(-mx // P)
    m = np.cumsum(rng.normal(0.05, 1.5, size=(S, H, mp)), axis=-1)
    l = rng.uniform(0.5, 40, size=(S, H, mp))
    acc = rng.normal(size=(S, H, mp, D)) * l[..., None]
    m32, l32, acc32 = m.astype(np.float32), l.astype(np.float32), acc.astype(np.float32)
    ref = oracle.splitk_merge(m32.astype(np.float64), l32.astype(np.float64), acc32.astype(np.float64), ctx, P)
    ws = torch.zeros(pa.pa_splitk_workspace_bytes(S, H, D, mx, P), dtype=torch.uint8, device="cuda")
    wml, wacc = pa.splitk_views(ws, S, H, D, mx, P)
    wml[..., 0] = torch.from_numpy(m32).cuda()
    wml[..., 1] = torch.from_numpy(l32).cuda()
    wacc.copy_(torch.from_numpy(acc32).cuda())
    out = torch.empty((S, H, D), dtype=torch.float32, device="cuda")
    pa.pa_splitk_reduce(out, ws, torch.from_numpy(ctx).cuda(), mx, P)
    torch.cuda.synchronize()
    np.testing.assert_allclose(f64(out), ref, rtol=2e-6, atol=2e-6)


def test_partition_covering_context_equals_unsplit(pa):
    ctx = [300, 17, 999]
    c = Case(pa, torch.float16, 3, 8, 8, 128, 16, ctx, seed=7, out_dtype=torch.float32)
    _, o1 = _run_write_and_decode(pa, c)
    _, o2 = _run_write_and_decode(pa, c, partition=1024)
    assert torch.allclose(o1, o2, rtol=1e-6, atol=1e-6)


def test_copy_blocks_bitwise(pa):
    g = torch.Generator().manual_seed(8)
    NB, Hkv, BS, D = 40, 4, 16, 128
    k = torch.randn((NB, Hkv, BS, D), generator=g).to(torch.bfloat16)
    v = torch.randn((NB, Hkv, BS, D), generator=g).to(torch.bfloat16)
    pairs = np.array([[3, 10], [3, 11], [7, 0], [39, 38], [12, 13]], np.int64)
    ok, ov = raw(k).copy(), raw(v).copy()
    oracle.copy_blocks(ok, ov, pairs)
    kd, vd = k.cuda(), v.cuda()
    pa.pa_copy_blocks(kd, vd, torch.from_numpy(pairs).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(raw(kd.cpu()), ok) and np.array_equal(raw(vd.cpu()), ov)
    assert pa.pa_read_device_errors() == 0


def _bits(t):
    return t.view(torch.int32 if t.element_size() == 4 else torch.int16)


@pytest.mark.parametrize("dt,D,BS,Hq,Hkv", SHAPES)
def test_decode_append_equals_write_then_decode(pa, dt, D, BS, Hq, Hkv):
    """pa_decode_append gives, bit for bit, the pools and the output of
    pa_reshape_and_cache of the newest tokens followed by pa_decode. Its side
    starts with NaN in the newest tokens' slots, so attention that read the
    pool's copy of a newest row instead of the new one would show NaN."""
    ctx = [1, 17, 45, 100, 16, 33, 0, 64]
    c = Case(pa, DT[dt], len(ctx), Hq, Hkv, D, BS, ctx, seed=41 + D + BS + Hq)
    d1, out1 = _run_write_and_decode(pa, c)
    d2 = c.device()
    for s, L in enumerate(ctx):
        if L:
            b, o = divmod(int(c.slots[s]), BS)
            d2["k"][b, :, o, :] = float("nan")
            d2["v"][b, :, o, :] = float("nan")
    from paged_kv_cache_340_b200.batch import longest_first
    order = torch.from_numpy(longest_first(c.ctx)).cuda()
    out2 = torch.empty_like(out1)
    pa.pa_decode_append(out2, d2["q"], d2["nk"], d2["nv"], d2["k"], d2["v"], d2["bt"], d2["cl"], c.scale,
                        seq_order=order)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    assert torch.equal(_bits(d2["k"]), _bits(d1["k"])) and torch.equal(_bits(d2["v"]), _bits(d1["v"]))
    assert torch.isfinite(out2.float()).all()
    assert torch.equal(out2, out1)
    assert_attention_close(out2, c.ref, DT[dt], "decode_append")


def test_decode_append_skips_a_bad_block(pa):
    """A table entry out of range at a sequence's newest token: that block is
    skipped (nothing written, error flagged); the other sequences match."""
    c = Case(pa, torch.bfloat16, 3, 8, 2, 128, 16, [40, 40, 40], seed=43, poison=False)
    d = c.device()
    bt = d["bt"].clone()
    bt[1, 2] = c.NB + 7                                      # holds token 39 of sequence 1
    k0 = d["k"].clone()
    pa.pa_read_device_errors()
    out = torch.empty((3, 8, 128), dtype=torch.bfloat16, device="cuda")
    pa.pa_decode_append(out, d["q"], d["nk"], d["nv"], d["k"], d["v"], bt, d["cl"], c.scale)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() & pa.PA_DEVERR_BLOCK_ID
    b1, o1 = divmod(int(c.slots[1]), 16)
    assert torch.equal(_bits(d["k"][b1, :, o1]), _bits(k0[b1, :, o1]))   # sequence 1's newest row not written
    assert_attention_close(out[[0, 2]], c.ref[[0, 2]], torch.bfloat16, "unaffected sequences")


def test_device_errors_are_recorded_not_faulted(pa):
    c = Case(pa, torch.float16, 3, 4, 4, 128, 16, [40, 40, 40], seed=12, poison=False)
    d = c.device()
    pa.pa_read_device_errors()
    # a table entry out of range in sequence 1: its block is skipped, others unaffected
    bt = d["bt"].clone()
    bt[1, 1] = c.NB + 5
    out = torch.empty((3, 4, 128), dtype=torch.float16, device="cuda")
    pa.pa_decode(out, d["q"], d["k"], d["v"], bt, d["cl"], c.scale)
    assert pa.pa_read_device_errors() & pa.PA_DEVERR_BLOCK_ID
    assert torch.isfinite(out.float()).all()
    ref = oracle.paged_decode(f64(c.q), f64(c.kp_host), f64(c.vp_host), c.tables, c.ctx, c.scale, 16)
    assert_attention_close(out[[0, 2]], ref[[0, 2]], torch.float16, "unaffected sequences")
    # a slot past the pool: nothing written, flag set
    k0 = d["k"].clone()
    bad = torch.tensor([c.NB * 16, -1, 3], dtype=torch.int32, device="cuda")
    pa.pa_reshape_and_cache(d["nk"], d["nv"], d["k"], d["v"], bad)
    assert pa.pa_read_device_errors() & pa.PA_DEVERR_SLOT
    assert torch.equal(d["k"][1:], k0[1:]) and torch.equal(d["k"][0, :, 3], d["nk"][2])
    # a context longer than its table row: clamped, flagged
    cl = d["cl"].clone()
    cl[0] = 16 * d["bt"].shape[1] + 1
    pa.pa_decode(out, d["q"], d["k"], d["v"], d["bt"], cl, c.scale)
    assert pa.pa_read_device_errors() & pa.PA_DEVERR_CONTEXT
    # a copy pair out of range: skipped, flagged
    pa.pa_copy_blocks(d["k"], d["v"], torch.tensor([[0, c.NB]], dtype=torch.int64, device="cuda"))
    assert pa.pa_read_device_errors() & pa.PA_DEVERR_PAIR
    assert pa.pa_read_device_errors() == 0


def test_largest_batch_grid(pa):
    """65,535 sequences (the most one launch covers), contexts 0..40: every
    sequence's output matches the oracle; a 65,536th is refused on the host."""
    g = torch.Generator().manual_seed(31)
    S, H, D, BS = 65535, 1, 64, 16
    ctx = torch.randint(0, 41, (S,), generator=g).to(torch.int32)
    nb = [(int(c) + BS - 1) // BS for c in ctx]
    NB = sum(nb)
    ids = torch.randperm(NB, generator=g).to(torch.int32)
    tables = torch.full((S, 3), -1, dtype=torch.int32)
    pos = 0
    for s, n in enumerate(nb):
        tables[s, :n] = ids[pos:pos + n]
        pos += n
    k = torch.randn((NB, H, BS, D), generator=g).to(torch.float16)
    v = torch.randn((NB, H, BS, D), generator=g).to(torch.float16)
    q = torch.randn((S, H, D), generator=g).to(torch.float16)
    out = torch.empty((S, H, D), dtype=torch.float32, device="cuda")
    pa.pa_decode(out, q.cuda(), k.cuda(), v.cuda(), tables.cuda(), ctx.cuda(), 0.125)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    ref = oracle.paged_decode(f64(q), f64(k), f64(v), tables.numpy(), ctx.numpy(), 0.125, BS)
    assert_attention_close(out, ref, torch.float16, "65535 sequences")
    big = torch.empty((S + 1, H, D), dtype=torch.float32, device="cuda")
    with pytest.raises(pa.PagedAttentionError):
        pa.pa_decode(big, big.to(torch.float16), k.cuda(), v.cuda(), torch.cat([tables, tables[:1]]).cuda(),
                     torch.cat([ctx, ctx[:1]]).cuda(), 0.125)


# (dtype, Hkv, D, block_size, tokens): 16-byte vectors per token Hkv * D * elt / 16
# at most 256 (several tokens per CTA round; 256 not always a multiple of it)
# and above 256 (a token in rounds of 256 vectors, the last one partial), with
# token counts that span many rounds of the grid and end mid-round.
SLOT_WRITE_SHAPES = [
    ("f16", 3, 128, 16, 3001),    # 48 vectors a token: 5 tokens a round, 16 threads idle
    ("f32", 1, 64, 32, 777),      # 16 vectors
    ("bf16", 24, 128, 16, 2500),  # 384 vectors: rounds of 256 and 128
    ("f32", 8, 128, 32, 1500),    # 256 vectors: exactly one round
    ("f32", 32, 128, 16, 9000),   # 1024 vectors: four rounds, and more tokens than the grid
]


@pytest.mark.parametrize("dt,Hkv,D,BS,T", SLOT_WRITE_SHAPES)
def test_slot_write_shapes_bitwise(pa, dt, Hkv, D, BS, T):
    """pa_reshape_and_cache against the oracle's byte copies: every pool byte
    equal, including rows no slot names (left as they were) and tokens whose
    slot is -1 (skipped)."""
    dtype = DT[dt]
    g = torch.Generator().manual_seed(1000 + Hkv * 7 + T)
    NB = -(-T // BS) + 5
    kp = torch.randn((NB, Hkv, BS, D), generator=g).to(dtype)
    vp = torch.randn((NB, Hkv, BS, D), generator=g).to(dtype)
    nk = torch.randn((T, Hkv, D), generator=g).to(dtype)
    nv = torch.randn((T, Hkv, D), generator=g).to(dtype)
    rng = np.random.default_rng(T)
    slots = rng.permutation(NB * BS)[:T].astype(np.int32)  # distinct slots, any block and offset
    slots[rng.random(T) < 0.05] = -1                        # padding tokens
    okp, ovp = raw(kp).copy(), raw(vp).copy()
    oracle.reshape_and_cache(okp, ovp, raw(nk), raw(nv), slots)
    dk, dv = kp.cuda(), vp.cuda()
    pa.pa_reshape_and_cache(nk.cuda(), nv.cuda(), dk, dv, torch.from_numpy(slots).cuda())
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    assert np.array_equal(raw(dk), okp)
    assert np.array_equal(raw(dv), ovp)
