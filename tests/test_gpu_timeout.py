"""The bounded pipeline waits on the GPU. A copy that never lands must not
hang the GPU: the waiting warp gives up after its bound, records
PA_DEVERR_TIMEOUT, waits (again bounded) for the copies it still has in flight
and leaves, and the launch ends. pa_decode_withhold_stage plants that fault
from the host (one stage's copy is never issued) with a bound of a few
milliseconds, so the test makes the wait run out and checks what the host
reads back; nothing faults or traps.

After such a launch, every (sequence, kv head) other than the one with the
withheld stage still matches the oracle, and the next normal call is clean."""
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
