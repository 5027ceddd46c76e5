"""Prefix cache on the GPU ([P4] "PagedAttention 实现细节", §3.2 Prefix
Caching, with §3.3's copy-on-write): requests share a few system prompts'
blocks through the library's prefix cache; a prompt's K/V are written once,
on the miss that took its blocks; each request maps the blocks into its own
table (its own reference to each), appends its user tokens (the first write
into the shared partial block copies it) and is decoded over the shared
blocks. Finished requests release their prompt and blocks mid-flow, so later
requests re-create a released prompt in reused blocks.

Checked against the oracle's flow (its pool and prefix-cache manager): every
table, slot and copy pair bit for bit, both pools bit for bit after the same
device steps, and every live request's attention within the tolerance."""
import numpy as np
import pytest
import torch

import oracle
from _helpers import assert_attention_close, f64, oracle_prefix_cache_flow, raw
from paged_kv_cache_340_b200.workloads import SPECS, make_prefix_cache_inputs, scaled

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_340_b200 import _build
    _build.build()
    import paged_kv_cache_340_b200 as pa
    return pa


def _run(pa, spec, finish_after=None, poison=True):
    from paged_kv_cache_340_b200.batch import prefix_cache_flow, shared_prefix_order
    inp = make_prefix_cache_inputs(spec)
    ops, tables, ctx, live = prefix_cache_flow(spec, inp, finish_after=finish_after)
    want_ops, want_tables, want_ctx, want_live = oracle_prefix_cache_flow(
        inp, spec.block_size, spec.prefix_len, spec.max_divergent, finish_after)
    # host decisions: bit for bit
    assert [(o.kind, o.index) for o in ops] == [(k, i) for k, i, _ in want_ops]
    for o, (_, _, w) in zip(ops, want_ops):
        assert np.array_equal(o.slots.reshape(-1), np.asarray(w, np.int64).reshape(-1)), o.kind
    assert np.array_equal(tables, want_tables) and np.array_equal(ctx, want_ctx)
    assert np.array_equal(live, want_live)
    # device steps in the host's order; the oracle repeats them on byte copies
    dt = spec.torch_kv_dtype
    NB, Hkv, bs, D = int(inp["num_blocks"]), spec.num_kv_heads, spec.block_size, spec.head_dim
    init = torch.full((NB, Hkv, bs, D), float("nan"), dtype=dt) if poison else torch.zeros((NB, Hkv, bs, D), dtype=dt)
    kd, vd = init.cuda(), init.cuda()
    okc, ovc = raw(init).copy(), raw(init).copy()
    lens = inp["system_lens"].numpy()
    ustart = np.concatenate([[0], np.cumsum(inp["user_lens"].numpy())]).astype(np.int64)
    for o in ops:
        if o.kind == "prefix":
            L0 = int(lens[o.index])
            key, val = inp["prefix_key"][o.index, :L0].contiguous(), inp["prefix_value"][o.index, :L0].contiguous()
        elif o.kind == "user":
            key = inp["user_key"][ustart[o.index]:ustart[o.index + 1]]
            val = inp["user_value"][ustart[o.index]:ustart[o.index + 1]]
        if o.kind in ("prefix", "user"):
            pa.pa_reshape_and_cache(key.cuda(), val.cuda(), kd, vd, torch.from_numpy(o.slots).cuda())
            oracle.reshape_and_cache(okc, ovc, raw(key), raw(val), o.slots)
        elif o.kind == "copy":
            pa.pa_copy_blocks(kd, vd, torch.from_numpy(o.slots).cuda())
            oracle.copy_blocks(okc, ovc, o.slots)
    rows = np.nonzero(live)[0]
    S = rows.shape[0]
    q = inp["query"][torch.from_numpy(rows)].contiguous()
    out = torch.full((S, spec.num_heads, D), float("nan"), dtype=spec.torch_out_dtype, device="cuda")
    order = shared_prefix_order(ctx[rows], inp["choice"].numpy()[rows])
    pa.pa_decode(out, q.cuda(), kd, vd, torch.from_numpy(tables[rows]).cuda(), torch.from_numpy(ctx[rows]).cuda(),
                 spec.scale, seq_order=torch.from_numpy(order).cuda())
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    assert np.array_equal(raw(kd), okc) and np.array_equal(raw(vd), ovc)
    kf = torch.from_numpy(okc).view(dt)
    vf = torch.from_numpy(ovc).view(dt)
    ref = oracle.paged_decode(f64(q), kf.double().numpy(), vf.double().numpy(), tables[rows], ctx[rows], spec.scale,
                              bs)
    assert_attention_close(out, ref, dt, spec.name)
    return ops


@pytest.mark.parametrize("dtype,Hq,Hkv,D,bs", [("f16", 4, 4, 128, 16), ("bf16", 8, 2, 64, 32),
                                               ("f32", 4, 2, 64, 16)])
def test_prefix_cache_flow_with_releases(pa, dtype, Hq, Hkv, D, bs):
    out_dt = {"f16": "f16", "bf16": "f32", "f32": "f32"}[dtype]
    spec = scaled(SPECS["prefix_cache_fp16"], name=f"prefix_{dtype}", num_seqs=24, num_heads=Hq, num_kv_heads=Hkv,
                  head_dim=D, block_size=bs, kv_dtype=dtype, out_dtype=out_dt, lengths=("prefix", 20, 300),
                  num_prompts=3, prefix_len=300, max_divergent=40)
    choice = make_prefix_cache_inputs(spec)["choice"].numpy()
    p0 = int(choice[0])
    # after request 9: every request so far with prompt p0 finishes, so the
    # cache drops p0 and a later p0 request must write it again elsewhere
    finish_after = {9: [r for r in range(10) if choice[r] == p0], 15: [11, 13]}
    ops = _run(pa, spec, finish_after)
    kinds = [(o.kind, o.index) for o in ops]
    assert kinds.count(("prefix", p0)) >= 2, "the released prompt was never written again"
    assert any(o.kind == "copy" for o in ops)


def test_prefix_cache_workload_full_size(pa):
    """The bench workload (96 requests over 4 system prompts of 500-2000
    tokens, 32 heads, fp16), as the bench builds it, against the oracle."""
    _run(pa, SPECS["prefix_cache_fp16"], poison=False)
