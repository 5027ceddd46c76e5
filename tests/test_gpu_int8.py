"""int8 KV cache on the GPU (pa_reshape_and_cache_q8, pa_decode_q8,
pa_decode_splitk_q8, pa_copy_blocks_q8) against the oracle.

The quantizing slot write must give the oracle's codes and scales bit for bit
(the integer decision is taken in fp32 on both sides). Attention over the int8
cache must match the oracle's attention over the dequantized cache within the
16-bit bound (max abs 4e-3, relative L2 1e-3). Unused slots hold random codes
and NaN scales, so a read past a context or a missed mask shows up."""
import math

import numpy as np
import pytest
import torch

import oracle
from _helpers import assert_attention_close, f64, raw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_340_b200 import _build
    _build.build()
    import paged_kv_cache_340_b200 as pa
    return pa


def _f32(t):
    return t.float().numpy()


@pytest.mark.parametrize("src", [torch.float16, torch.bfloat16, torch.float32])
@pytest.mark.parametrize("D", [64, 128])
def test_quantizing_slot_write_is_bit_exact(pa, src, D):
    g = torch.Generator().manual_seed(D + 3)
    NB, Hkv, bs, T = 9, 3, 16, 40
    key = (torch.randn((T, Hkv, D), generator=g) * torch.rand((T, Hkv, 1), generator=g) * 10).to(src)
    val = torch.randn((T, Hkv, D), generator=g).to(src)
    key[3] = 0.0                                            # zero rows: codes 0, scale 0
    key[4, 0, :4] = torch.tensor([254.0, 1.0, -1.0, 3.0])   # ties to even
    key[4, 0, 4:] = 0.0
    val[5, 1, 0] = -0.0
    if src == torch.float32:
        key[6, 2] *= 1e30
        val[6, 2] *= 1e-30
    slots = torch.randperm(NB * bs, generator=g)[:T].to(torch.int32)
    slots[7] = -1
    kc = torch.randint(-127, 128, (NB, Hkv, bs, D), generator=g, dtype=torch.int8)
    vc = kc.clone()
    ks = torch.rand((NB, Hkv, bs), generator=g)
    vs = ks.clone()
    kd, vd, ksd, vsd = kc.cuda(), vc.cuda(), ks.cuda(), vs.cuda()
    pa.pa_reshape_and_cache_q8(key.cuda(), val.cuda(), kd, vd, ksd, vsd, slots.cuda())
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    kn, vn, ksn, vsn = kc.numpy().copy(), vc.numpy().copy(), ks.numpy().copy(), vs.numpy().copy()
    oracle.reshape_and_cache_q8(kn, vn, ksn, vsn, _f32(key), _f32(val), slots.numpy())
    assert np.array_equal(kd.cpu().numpy(), kn) and np.array_equal(vd.cpu().numpy(), vn)
    assert np.array_equal(raw(ksd), ksn.view(np.int32)) and np.array_equal(raw(vsd), vsn.view(np.int32))


class Q8Case:
    """int8 pools quantized by the oracle from random fp32 rows (every slot),
    then NaN scales on every slot no sequence uses; random tables."""

    def __init__(self, S, Hq, Hkv, D, bs, ctx, seed):
        rng = np.random.default_rng(seed)
        self.ctx = np.array(ctx, np.int32)
        nbk = [-(-int(c) // bs) for c in ctx]
        self.NB = NB = sum(nbk) + 4
        perm = rng.permutation(NB)
        self.tables = np.full((S, max(1, max(nbk))), -1, np.int32)
        pos = 0
        used = np.zeros((NB, bs), bool)
        for s, n in enumerate(nbk):
            self.tables[s, :n] = perm[pos:pos + n]
            pos += n
            for t in range(int(ctx[s])):
                used[self.tables[s, t // bs], t % bs] = True
        kf = rng.normal(size=(NB, Hkv, bs, D)).astype(np.float32) * rng.uniform(0.1, 3, size=(NB, Hkv, bs, 1))
        vf = rng.normal(size=(NB, Hkv, bs, D)).astype(np.float32)
        self.kq, self.ks = oracle.quantize_rows(kf.astype(np.float32))
        self.vq, self.vs = oracle.quantize_rows(vf)
        bi, oi = np.nonzero(~used)
        self.ks[bi, :, oi] = np.nan
        self.vs[bi, :, oi] = np.nan
        self.q = torch.from_numpy(rng.normal(size=(S, Hq, D)).astype(np.float32))
        self.scale = 1.0 / math.sqrt(D)
        self.bs = bs

    def device(self):
        return [torch.from_numpy(a).cuda() for a in (self.kq, self.vq, self.ks, self.vs)]

    def ref(self, qdt):
        ctx_ok = np.where(self.ctx > 0, self.ctx, 0)
        ks = np.nan_to_num(self.ks, nan=0.0)   # the oracle never reads unused slots; keep it NaN-free
        vs = np.nan_to_num(self.vs, nan=0.0)
        return oracle.paged_decode_q8(f64(self.q.to(qdt)), self.kq, self.vq, ks, vs, self.tables, ctx_ok,
                                      self.scale, self.bs)


SHAPES = [
    # (S, Hq, Hkv, D, bs, ctx)
    (4, 8, 8, 128, 16, [1, 17, 45, 300]),
    (3, 16, 4, 128, 32, [33, 64, 200]),
    (5, 16, 2, 64, 16, [15, 16, 1, 90, 257]),
    (2, 32, 4, 128, 16, [1000, 7]),
    (3, 8, 8, 64, 32, [31, 32, 129]),
    (4, 8, 4, 128, 16, [2, 16, 33, 517]),   # head group 2 (two heads, one per lane)
]


@pytest.mark.parametrize("qdt", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("case", range(len(SHAPES)))
def test_decode_q8_matches_oracle(pa, qdt, case):
    S, Hq, Hkv, D, bs, ctx = SHAPES[case]
    c = Q8Case(S, Hq, Hkv, D, bs, ctx, seed=30 + case)
    kq, vq, ks, vs = c.device()
    out = torch.full((S, Hq, D), float("nan"), device="cuda")
    pa.pa_decode_q8(out, c.q.to(qdt).cuda(), kq, vq, ks, vs, torch.from_numpy(c.tables).cuda(),
                    torch.from_numpy(c.ctx).cuda(), c.scale)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    assert_attention_close(out, c.ref(qdt), torch.float16, f"q8 case {case} {qdt}")


def test_decode_q8_16bit_output_and_ctx1(pa):
    c = Q8Case(4, 8, 8, 128, 16, [1, 17, 45, 300], seed=41)
    kq, vq, ks, vs = c.device()
    for qdt in (torch.float16, torch.bfloat16):
        out = torch.empty((4, 8, 128), dtype=qdt, device="cuda")
        pa.pa_decode_q8(out, c.q.to(qdt).cuda(), kq, vq, ks, vs, torch.from_numpy(c.tables).cuda(),
                        torch.from_numpy(c.ctx).cuda(), c.scale)
        torch.cuda.synchronize()
        assert_attention_close(out, c.ref(qdt), qdt, f"q8 {qdt} out")
    # one token: the dequantized V row (one fp32 product), whatever the query
    out = torch.empty((4, 8, 128), device="cuda")
    pa.pa_decode_q8(out, c.q.half().cuda(), kq, vq, ks, vs, torch.from_numpy(c.tables).cuda(),
                    torch.from_numpy(c.ctx).cuda(), c.scale)
    b = c.tables[0, 0]
    want = c.vq[b, :, 0].astype(np.float32) * c.vs[b, :, 0, None]
    np.testing.assert_allclose(out[0].cpu().numpy(), want, rtol=2e-7, atol=0)


@pytest.mark.parametrize("P", [32, 64, 512])
def test_decode_splitk_q8(pa, P):
    S, Hq, Hkv, D, bs, ctx = 3, 16, 4, 128, 16, [700, 33, 1]
    c = Q8Case(S, Hq, Hkv, D, bs, ctx, seed=50 + P)
    kq, vq, ks, vs = c.device()
    L = int(max(ctx))
    ws = torch.empty(pa.pa_splitk_workspace_bytes(S, Hq, D, L, P), dtype=torch.uint8, device="cuda")
    out = torch.empty((S, Hq, D), device="cuda")
    tab, cl = torch.from_numpy(c.tables).cuda(), torch.from_numpy(c.ctx).cuda()
    pa.pa_decode_splitk_q8(ws, c.q.half().cuda(), kq, vq, ks, vs, tab, cl, c.scale, L, P)
    pa.pa_splitk_reduce(out, ws, cl, L, P)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    assert_attention_close(out, c.ref(torch.float16), torch.float16, f"q8 split P={P}")


def test_copy_blocks_q8(pa):
    g = torch.Generator().manual_seed(61)
    NB, Hkv, bs, D = 12, 2, 16, 128
    kc = torch.randint(-127, 128, (NB, Hkv, bs, D), generator=g, dtype=torch.int8)
    vc = torch.randint(-127, 128, (NB, Hkv, bs, D), generator=g, dtype=torch.int8)
    ks, vs = torch.rand((NB, Hkv, bs), generator=g), torch.rand((NB, Hkv, bs), generator=g)
    pairs = np.array([[3, 7], [0, 11], [5, 2]], np.int64)
    d = [t.cuda() for t in (kc, vc, ks, vs)]
    pa.pa_copy_blocks_q8(*d, torch.from_numpy(pairs).cuda())
    torch.cuda.synchronize()
    want = [t.numpy().copy() for t in (kc, vc, ks, vs)]
    for s_, t_ in pairs:
        for w in want:
            w[t_] = w[s_]
    for got, w in zip(d, want):
        assert np.array_equal(got.cpu().numpy(), w)
    assert pa.pa_read_device_errors() == 0


def test_decode_q8_bad_block_id_is_recorded(pa):
    c = Q8Case(2, 8, 8, 128, 16, [40, 20], seed=71)
    kq, vq, ks, vs = c.device()
    tab = c.tables.copy()
    tab[0, 1] = c.NB + 5
    out = torch.empty((2, 8, 128), device="cuda")
    pa.pa_decode_q8(out, c.q.half().cuda(), kq, vq, ks, vs, torch.from_numpy(tab).cuda(),
                    torch.from_numpy(c.ctx).cuda(), c.scale)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() & pa.PA_DEVERR_BLOCK_ID
    ref = c.ref(torch.float16)
    assert_attention_close(out[1:], ref[1:], torch.float16, "the other sequence")


@pytest.mark.parametrize("name", ["llama7b_mha_int8", "gqa_int8"])
def test_int8_workloads_full_size(pa, name):
    """The benchmark's int8 workloads at full size, in its launch
    configuration: the whole pool quantized by the library equals the
    oracle's codes and scales; after the step (quantizing slot write of the
    newest tokens, decode) the caches still equal the oracle's; every
    sequence's attention matches the oracle over the dequantized cache."""
    from paged_kv_cache_340_b200.batch import build_decode_batch, run_step
    from paged_kv_cache_340_b200.workloads import SPECS, make_decode_inputs
    from _helpers import oracle_decode_tables
    spec = SPECS[name]
    inp = make_decode_inputs(spec)
    b = build_decode_batch(spec, inp)
    ctx = inp["context_lens"].numpy()
    otab, oslots = oracle_decode_tables(ctx, inp["num_blocks"], spec.block_size, inp["free_order"].numpy())
    assert np.array_equal(b.host_tables, otab) and np.array_equal(b.host_slots, oslots)
    kq, ks = oracle.quantize_rows(inp["k_pool"].float().numpy())
    vq, vs = oracle.quantize_rows(inp["v_pool"].float().numpy())
    assert np.array_equal(b.k_cache.cpu().numpy(), kq) and np.array_equal(b.v_cache.cpu().numpy(), vq)
    assert np.array_equal(raw(b.k_scale), ks.view(np.int32)) and np.array_equal(raw(b.v_scale), vs.view(np.int32))
    run_step(b)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    oracle.reshape_and_cache_q8(kq, vq, ks, vs, inp["new_key"].float().numpy(), inp["new_value"].float().numpy(),
                                oslots)
    assert np.array_equal(b.k_cache.cpu().numpy(), kq) and np.array_equal(b.v_cache.cpu().numpy(), vq)
    assert np.array_equal(raw(b.k_scale), ks.view(np.int32)) and np.array_equal(raw(b.v_scale), vs.view(np.int32))
    out = b.out.cpu()
    q = inp["query"]
    for s in range(spec.num_seqs):
        L = int(ctx[s])
        nb = oracle.blocks_needed(L, spec.block_size)
        ids = b.host_tables[s, :nb]
        tab = np.arange(nb, dtype=np.int32)[None, :]
        ref = oracle.paged_decode_q8(f64(q[s:s + 1]), kq[ids], vq[ids], ks[ids], vs[ids], tab,
                                     np.array([L], np.int32), spec.scale, spec.block_size)
        assert_attention_close(out[s:s + 1], ref, torch.float16, f"{name} seq {s}")


def test_decode_splitk_q8_head_dim_64_with_schedule(pa):
    """Split-K over an int8 cache with head_dim 64 and a GQA group of 8, with a
    longest-first schedule: same result as the oracle."""
    S, Hq, Hkv, D, bs, ctx = 4, 16, 2, 64, 32, [900, 1, 300, 64]
    c = Q8Case(S, Hq, Hkv, D, bs, ctx, seed=81)
    kq, vq, ks, vs = c.device()
    L, P = 900, 128
    ws = torch.empty(pa.pa_splitk_workspace_bytes(S, Hq, D, L, P), dtype=torch.uint8, device="cuda")
    out = torch.empty((S, Hq, D), device="cuda")
    tab, cl = torch.from_numpy(c.tables).cuda(), torch.from_numpy(c.ctx).cuda()
    order = torch.tensor([0, 2, 3, 1], dtype=torch.int32, device="cuda")
    pa.pa_decode_splitk_q8(ws, c.q.to(torch.bfloat16).cuda(), kq, vq, ks, vs, tab, cl, c.scale, L, P,
                           seq_order=order)
    pa.pa_splitk_reduce(out, ws, cl, L, P)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    assert_attention_close(out, c.ref(torch.bfloat16), torch.float16, "q8 split D=64")
