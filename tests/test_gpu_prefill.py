"""GPU parity of paged prefill (tcgen05 tensor-core kernel) against the oracle.

Each sequence's new query tokens attend causally over its paged cache.
Unused pool slots hold NaN so a read past a context or a missing mask shows
up. Acceptance as for decode: max abs <= 4e-3 and relative L2 <= 1e-3 for
16-bit inputs (bf16 outputs add their own rounding)."""
import math

import numpy as np
import pytest
import torch

import oracle
from _helpers import assert_attention_close, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_340_b200 import _build
    _build.build()
    import paged_kv_cache_340_b200 as pa
    return pa


def _case(seed, ctx, qlen, Hq, Hkv, BS, dtype, D=128, poison=True):
    g = torch.Generator().manual_seed(seed)
    S = len(ctx)
    nb = [(c + BS - 1) // BS for c in ctx]
    NB = sum(nb) + 5
    ids = torch.randperm(NB, generator=g).to(torch.int32)
    tables = torch.full((S, max(1, max(nb))), -1, dtype=torch.int32)
    pos = 0
    for s, n in enumerate(nb):
        tables[s, :n] = ids[pos:pos + n]
        pos += n
    k = torch.randn((NB, Hkv, BS, D), generator=g).to(dtype)
    v = torch.randn((NB, Hkv, BS, D), generator=g).to(dtype)
    if poison:
        used = torch.zeros((NB, BS), dtype=torch.bool)
        for s, L in enumerate(ctx):
            for t in range(L):
                used[tables[s, t // BS], t % BS] = True
        bi, oi = (~used).nonzero(as_tuple=True)
        k[bi, :, oi, :] = float("nan")
        v[bi, :, oi, :] = float("nan")
    qs = torch.tensor(np.concatenate([[0], np.cumsum(qlen)]), dtype=torch.int32)
    q = torch.randn((int(qs[-1]), Hq, D), generator=g).to(dtype)
    return dict(k=k, v=v, q=q, qs=qs, tables=tables, ctx=torch.tensor(ctx, dtype=torch.int32), BS=BS,
                scale=1.0 / math.sqrt(D), max_q=max(qlen))


def _run(pa, c, out_dtype):
    T, Hq, D = c["q"].shape
    out = torch.full((T, Hq, D), float("nan"), dtype=out_dtype, device="cuda")
    pa.pa_prefill(out, c["q"].cuda(), c["qs"].cuda(), c["max_q"], c["k"].cuda(), c["v"].cuda(),
                  c["tables"].cuda(), c["ctx"].cuda(), c["scale"])
    torch.cuda.synchronize()
    return out


def _ref(c):
    return oracle.paged_prefill(f64(c["q"]), c["qs"].numpy(), f64(c["k"]), f64(c["v"]), c["tables"].numpy(),
                                c["ctx"].numpy(), c["scale"], c["BS"])


CASES = [
    # (ctx, q_len, Hq, Hkv, BS)
    ([64, 1, 300, 77], [64, 1, 300, 20], 8, 8, 16),          # MHA: prefill from empty, decode-like, long, chunked
    ([200, 129, 40], [130, 129, 3], 8, 8, 32),                # crossing the 128-row tile, bs 32
    ([96, 513, 17], [96, 100, 17], 16, 4, 16),                # GQA G = 4
    ([250, 64], [250, 33], 16, 2, 32),                        # GQA G = 8
    ([700, 300, 1], [640, 300, 1], 16, 8, 16),                # GQA G = 2, several query tiles per sequence
    ([64, 30, 100], [10, 0, 50], 8, 4, 16),                   # a sequence with no new tokens in the middle
]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_prefill_matches_oracle(pa, dtype, case):
    ctx, qlen, Hq, Hkv, BS = CASES[case]
    c = _case(100 + case, ctx, qlen, Hq, Hkv, BS, dtype)
    out = _run(pa, c, torch.float32)
    assert pa.pa_read_device_errors() == 0
    assert_attention_close(out, _ref(c), dtype, f"prefill case {case} {dtype}")


@pytest.mark.parametrize("Hkv", [8, 4, 2])  # head groups 1, 2 (rows staged in shared memory), 4 (rows stored directly)
def test_prefill_16bit_output(pa, Hkv):
    c = _case(7, [150, 60], [150, 10], 8, Hkv, 16, torch.bfloat16)
    out = _run(pa, c, torch.bfloat16)
    assert_attention_close(out, _ref(c), torch.bfloat16, "bf16 out")
    c = _case(8, [150, 60], [150, 10], 8, Hkv, 16, torch.float16)
    out = _run(pa, c, torch.float16)
    assert_attention_close(out, _ref(c), torch.float16, "fp16 out")


def test_prefill_of_single_tokens_equals_decode(pa):
    """q_len = 1 everywhere: the prefill kernel must give pa_decode's answer."""
    ctx = [1, 63, 64, 65, 400]
    c = _case(9, ctx, [1] * len(ctx), 16, 4, 16, torch.bfloat16)
    out = _run(pa, c, torch.float32)
    dec = torch.empty_like(out)
    pa.pa_decode(dec, c["q"].cuda(), c["k"].cuda(), c["v"].cuda(), c["tables"].cuda(), c["ctx"].cuda(), c["scale"])
    torch.cuda.synchronize()
    assert_attention_close(out, f64(dec), torch.bfloat16, "prefill vs decode")
    assert_attention_close(out, _ref(c), torch.bfloat16, "prefill vs oracle")


@pytest.mark.parametrize("G", [1, 2, 4])
def test_prefill_repeated_runs_are_bitwise_identical(pa, G):
    """The kernel's arithmetic order is fixed (same MMAs, same per-row softmax),
    so every run on the same input gives the same bits. A hand-off between the
    load, MMA and softmax warps that lets one warp's tile overtake another's
    shows up here as a run that differs, or as NaN from the poisoned slots."""
    c = _case(11 + G, [1500, 700, 300], [1400, 640, 300], 8 * G, 8, 16, torch.bfloat16)
    pa.pa_read_device_errors()  # clear what earlier tests left
    first = _run(pa, c, torch.float32)
    assert torch.isfinite(first).all()
    for _ in range(8):
        again = _run(pa, c, torch.float32)
        assert torch.equal(again, first)
    assert pa.pa_read_device_errors() == 0
    assert_attention_close(first, _ref(c), torch.bfloat16, f"G = {G}")


def test_prefill_rejects_queries_longer_than_context(pa):
    c = _case(10, [30, 50], [30, 10], 8, 8, 16, torch.float16, poison=False)
    c["ctx"] = torch.tensor([20, 50], dtype=torch.int32)   # sequence 0: 30 queries over 20 tokens
    out = _run(pa, c, torch.float32)
    assert pa.pa_read_device_errors() & pa.PA_DEVERR_CONTEXT
    ok = c["qs"][1].item()
    ref = oracle.paged_prefill(f64(c["q"][ok:]), np.array([0, 10], np.int32), f64(c["k"]), f64(c["v"]),
                               c["tables"].numpy()[1:], np.array([50], np.int32), c["scale"], 16)
    assert_attention_close(out[ok:], ref, torch.float16, "valid sequence")
    assert torch.isnan(out[:ok]).all()                       # the skipped sequence is left untouched


@pytest.mark.parametrize("Hkv", [8, 4, 2])  # head groups 1, 2 (staged rows), 4 (direct rows)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_prefill_writes_no_row_past_a_partial_tile(pa, Hkv, out_dtype):
    """Sequence 0 ends inside its query tile; the rows after it belong to
    sequence 1, which the kernel skips (more queries than context). They must
    keep the NaN they were filled with."""
    c = _case(12, [40, 50], [10, 30], 8, Hkv, 16, torch.bfloat16, poison=False)
    c["ctx"] = torch.tensor([40, 20], dtype=torch.int32)     # sequence 1: 30 queries over 20 tokens
    pa.pa_read_device_errors()
    out = _run(pa, c, out_dtype)
    assert pa.pa_read_device_errors() & pa.PA_DEVERR_CONTEXT
    ref = oracle.paged_prefill(f64(c["q"][:10]), np.array([0, 10], np.int32), f64(c["k"]), f64(c["v"]),
                               c["tables"].numpy()[:1], np.array([40], np.int32), c["scale"], 16)
    assert_attention_close(out[:10], ref, torch.bfloat16, "sequence 0")
    assert torch.isnan(out[10:].float()).all()


@pytest.mark.parametrize("name", ["prefill_llama7b_mha_bf16", "chunked_prefill_gqa_bf16"])
def test_prefill_workloads_full_size(pa, name):
    """The benchmark's prefill workloads at full size, in its launch
    configuration (slot write of the new tokens, then prefill). Tables and
    slots from the library pool match the oracle pool; for the first and the
    last sequence, every query row of the first and the last kv head (all
    query tiles, all heads of the group) matches the oracle."""
    from oracle.block_pool import BlockPool as OPool, Sequence, append_tokens
    from paged_kv_cache_340_b200.batch import build_prefill_batch, run_prefill_step
    from paged_kv_cache_340_b200.workloads import SPECS, make_prefill_inputs
    from _helpers import compact_for, raw
    spec = SPECS[name]
    inp = make_prefill_inputs(spec)
    b = build_prefill_batch(spec, inp)
    ctx = inp["context_lens"].numpy()
    opool = OPool(int(inp["num_blocks"]), spec.block_size, policy="fifo", free_order=inp["free_order"].tolist())
    oslots = []
    for s, L in enumerate(ctx):
        seq = Sequence()
        append_tokens(opool, seq, int(L) - spec.q_len)
        sl, _ = append_tokens(opool, seq, spec.q_len)
        oslots += sl
        assert list(b.host_tables[s, :len(seq.block_table)]) == seq.block_table
    assert np.array_equal(b.host_slots, np.array(oslots, np.int32))
    run_prefill_step(b)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    k_host, v_host = inp["k_pool"], inp["v_pool"]
    oracle.reshape_and_cache(raw(k_host), raw(v_host), raw(inp["new_key"]), raw(inp["new_value"]), np.array(oslots))
    out = b.out.cpu()
    q = inp["query"]
    G = spec.num_heads // spec.num_kv_heads
    Q = spec.q_len
    for s in (0, len(ctx) - 1):
        L = int(ctx[s])
        for kvh in (0, spec.num_kv_heads - 1):
            kp, vp, tab = compact_for(k_host, v_host, b.host_tables[s], L, spec.block_size, kv_heads=[kvh])
            qh = q[s * Q:(s + 1) * Q, kvh * G:(kvh + 1) * G]
            ref = oracle.paged_prefill(f64(qh), np.array([0, Q], np.int32), kp, vp, tab, np.array([L], np.int32),
                                       spec.scale, spec.block_size)
            got = out[s * Q:(s + 1) * Q, kvh * G:(kvh + 1) * G]
            assert_attention_close(got, ref, spec.torch_kv_dtype, f"{name} seq {s} kv head {kvh}")
