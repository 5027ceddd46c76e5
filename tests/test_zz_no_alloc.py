"""pa_decode_splitk_static: split-K decode for callers that cannot allocate.

Some callers cannot call cudaMalloc while they run: a serving loop that gave
nearly all of HBM to its KV-cache pool at start-up, a plug-in whose host
framework forbids allocation inside its execute callback, or a caller with no
device allocator. pa_decode_splitk_static takes its split-K workspace from a
fixed array inside the library instead of from the caller.

Here it is called through the C ABI and compared with the existing entry
points (pa_decode_splitk + pa_splitk_reduce on a caller workspace) on two
calls in a row with different inputs. Both run the same kernels on the same
inputs, so the outputs must be equal bit for bit: a wrong offset into the
shared array, or partials left over from the first call, would show. The file
name makes pytest collect it last.
"""
import math

import pytest
import torch


pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_340_b200 import _build
    _build.build()
    import paged_kv_cache_340_b200 as pa
    return pa


def _problem(seed, S, ctx_lo, ctx_hi, Hq=32, Hkv=8, D=128, BS=32, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    ctx = torch.randint(ctx_lo, ctx_hi + 1, (S,), generator=g).to(torch.int32)
    nblk = [(int(c) + BS - 1) // BS for c in ctx]
    NB = sum(nblk) + 7
    ids = torch.randperm(NB, generator=g).to(torch.int32)
    tables = torch.full((S, max(nblk)), -1, dtype=torch.int32)
    used = 0
    for s, n in enumerate(nblk):
        tables[s, :n] = ids[used:used + n]
        used += n
    k = torch.randn((NB, Hkv, BS, D), generator=g).to(dtype)
    v = torch.randn((NB, Hkv, BS, D), generator=g).to(dtype)
    q = torch.randn((S, Hq, D), generator=g).to(dtype)
    dev = "cuda"
    return dict(q=q.to(dev), k=k.to(dev), v=v.to(dev), bt=tables.to(dev), cl=ctx.to(dev),
                max_ctx=int(ctx.max()), scale=1.0 / math.sqrt(D))


def _with_workspace(pa, p, P):
    S, Hq, D = p["q"].shape
    ws = torch.empty(pa.pa_splitk_workspace_bytes(S, Hq, D, p["max_ctx"], P), dtype=torch.uint8, device="cuda")
    out = torch.empty((S, Hq, D), dtype=torch.float32, device="cuda")
    pa.pa_decode_splitk(ws, p["q"], p["k"], p["v"], p["bt"], p["cl"], p["scale"], p["max_ctx"], P)
    pa.pa_splitk_reduce(out, ws, p["cl"], p["max_ctx"], P)
    return out


def test_static_scratch_matches_workspace_path(pa):
    # An empty call only loads the array and looks up its address (the warm-up
    # a caller makes before sizing its KV pool); it touches no pointer.
    rc = pa._lib.pa_decode_splitk_static(None, None, None, None, None, 0, None, 0, 32, 8, 128, 0.1, 32, 0, 0, 1024,
                                         pa.PA_BF16, pa.PA_F32, None)
    assert rc == 0
    cases = [(1, 6, 3000, 20000, 1024), (2, 3, 100, 9000, 512)]
    for seed, S, lo, hi, P in cases:  # two calls in a row, different inputs and sizes
        p = _problem(seed, S, lo, hi)
        S_, Hq, D = p["q"].shape
        assert pa.pa_splitk_workspace_bytes(S_, Hq, D, p["max_ctx"], P) <= pa.PA_STATIC_SCRATCH_BYTES
        ref = _with_workspace(pa, p, P)
        out = torch.full_like(ref, float("nan"))
        pa.pa_decode_splitk_static(out, p["q"], p["k"], p["v"], p["bt"], p["cl"], p["scale"], p["max_ctx"], P)
        torch.cuda.synchronize()
        assert pa.pa_read_device_errors() == 0
        assert torch.isfinite(out).all()
        assert torch.equal(out, ref)


def test_static_scratch_refuses_bad_output_up_front(pa):
    """A NULL output or an unknown output type is refused with the reduce's
    status (all other inputs valid, so nothing could go wrong on the device
    even if the refusal came late)."""
    p = _problem(3, 2, 100, 600)
    S, Hq, D = p["q"].shape
    NB, Hkv, BS, _ = p["k"].shape
    args = (p["q"].data_ptr(), p["k"].data_ptr(), p["v"].data_ptr(), p["bt"].data_ptr(), p["bt"].shape[1],
            p["cl"].data_ptr(), S, Hq, Hkv, D, p["scale"], BS, NB, p["max_ctx"], 256, pa.PA_BF16)
    out = torch.empty((S, Hq, D), dtype=torch.float32, device="cuda")
    assert pa._lib.pa_decode_splitk_static(None, *args, pa.PA_F32, None) == -1       # PA_ERR_NULL
    assert pa._lib.pa_decode_splitk_static(out.data_ptr(), *args, 7, None) == -2    # PA_ERR_DTYPE
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0


def test_static_scratch_rejects_oversize(pa):
    """A request whose workspace would exceed the array is refused on the host
    (PA_ERR_WORKSPACE) before any device work; the pointers are never read."""
    S, Hq, Hkv, D, BS, max_ctx, P = 64, 32, 8, 128, 32, 131072, 512
    assert pa.pa_splitk_workspace_bytes(S, Hq, D, max_ctx, P) > pa.PA_STATIC_SCRATCH_BYTES
    fake = 1 << 20
    rc = pa._lib.pa_decode_splitk_static(fake, fake, fake, fake, fake, 4096, fake, S, Hq, Hkv, D, 0.1, BS, 100000,
                                         max_ctx, P, pa.PA_BF16, pa.PA_F32, None)
    assert rc == -9
