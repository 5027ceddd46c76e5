"""Head groups outside the compiled sizes 1, 2, 4, 8 on the GPU, against the
oracle. Any multiple num_heads = G * num_kv_heads is accepted: a group below 8
runs in the next compiled size with padding heads whose outputs are never
written; a group above 8 runs as sub-groups of 8 heads, one CTA each. The
oracle maps query head h to kv head h / G ([P3] §10 leaves GQA open; the
contiguous-group reading). Covers decode, split-K, the fused slot write +
decode, the int8 cache and prefill (tensor-core path for 16-bit caches,
CUDA-core path for fp32 caches)."""
import math

import numpy as np
import pytest
import torch

import oracle
from _helpers import assert_attention_close, f64, raw
from test_gpu_int8 import Q8Case
from test_gpu_parity import Case, _run_write_and_decode
from test_gpu_prefill import _case as prefill_case, _ref as prefill_ref, _run as prefill_run

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}

GROUPS = [
    # dtype, D, BS, Hq, Hkv  (group)
    ("bf16", 128, 16, 24, 8),    # 3
    ("f16", 128, 32, 48, 8),     # 6
    ("bf16", 128, 16, 28, 4),    # 7
    ("f16", 64, 16, 32, 2),      # 16: two sub-groups
    ("bf16", 128, 32, 10, 2),    # 5
    ("f16", 128, 16, 36, 3),     # 12: a full sub-group and a padded one
    ("f32", 64, 16, 6, 2),       # 3 on the CUDA cores
    ("f32", 128, 32, 24, 2),     # 12 on the CUDA cores
    ("bf16", 64, 16, 3, 1),      # 3, one kv head (the padding head reads past the query rows' group)
]


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_340_b200 import _build
    _build.build()
    import paged_kv_cache_340_b200 as pa
    return pa


@pytest.mark.parametrize("dt,D,BS,Hq,Hkv", GROUPS)
@pytest.mark.parametrize("partition", [0, 2])
def test_decode_any_group(pa, dt, D, BS, Hq, Hkv, partition):
    ctx = [1, BS + 1, 3 * BS + 5, 200, 0, 517]
    c = Case(pa, DT[dt], len(ctx), Hq, Hkv, D, BS, ctx, seed=Hq * 31 + Hkv + D,
             out_dtype=torch.float32 if dt == "bf16" else None)
    d, out = _run_write_and_decode(pa, c, partition * BS)
    assert np.array_equal(raw(d["k"].cpu()), c.okp) and np.array_equal(raw(d["v"].cpu()), c.ovp)
    assert_attention_close(out, c.ref, DT[dt], f"{dt} G{Hq // Hkv} P{partition * BS}")
    assert torch.all(out[4] == 0)


@pytest.mark.parametrize("dt,D,BS,Hq,Hkv", [g for g in GROUPS if g[0] != "f32"][:6])
def test_decode_append_any_group(pa, dt, D, BS, Hq, Hkv):
    """The fused slot write + decode gives the two calls' pools and output bit
    for bit (a group above 8: one sub-group's CTA writes the pool)."""
    ctx = [5, BS, 70, 333]
    c = Case(pa, DT[dt], len(ctx), Hq, Hkv, D, BS, ctx, seed=Hq + 7 * Hkv)
    d, out = _run_write_and_decode(pa, c)
    d2 = c.device()
    out2 = torch.empty_like(out)
    pa.pa_decode_append(out2, d2["q"], d2["nk"], d2["nv"], d2["k"], d2["v"], d2["bt"], d2["cl"], c.scale)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    assert torch.equal(out, out2)
    # raw bits (the unused slots hold NaN)
    assert np.array_equal(raw(d["k"]), raw(d2["k"])) and np.array_equal(raw(d["v"]), raw(d2["v"]))


@pytest.mark.parametrize("Hq,Hkv,D,bs", [(24, 8, 128, 16), (12, 2, 64, 32), (32, 2, 128, 16), (3, 1, 128, 32)])
@pytest.mark.parametrize("partition", [0, 64])
def test_decode_q8_any_group(pa, Hq, Hkv, D, bs, partition):
    ctx = [1, 45, 300, 129]
    c = Q8Case(len(ctx), Hq, Hkv, D, bs, ctx, seed=Hq + Hkv)
    kq, vq, ks, vs = c.device()
    S = len(ctx)
    out = torch.full((S, Hq, D), float("nan"), device="cuda")
    q = c.q.to(torch.bfloat16).cuda()
    bt, cl = torch.from_numpy(c.tables).cuda(), torch.from_numpy(c.ctx).cuda()
    if partition:
        mx = int(c.ctx.max())
        ws = torch.empty(pa.pa_splitk_workspace_bytes(S, Hq, D, mx, partition), dtype=torch.uint8, device="cuda")
        pa.pa_decode_splitk_q8(ws, q, kq, vq, ks, vs, bt, cl, c.scale, mx, partition)
        pa.pa_splitk_reduce(out, ws, cl, mx, partition)
    else:
        pa.pa_decode_q8(out, q, kq, vq, ks, vs, bt, cl, c.scale)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    assert_attention_close(out, c.ref(torch.bfloat16), torch.bfloat16, f"int8 G{Hq // Hkv}")


PREFILL = [
    # (ctx, q_len, Hq, Hkv, BS, D)
    ([200, 129, 40], [130, 129, 3], 24, 8, 16, 128),     # 3
    ([300, 64], [300, 33], 12, 2, 32, 128),              # 6
    ([150, 90], [150, 40], 28, 4, 16, 64),               # 7, head_dim 64
    ([140, 33], [140, 33], 32, 2, 16, 128),              # 16: 8 tokens per 128-row tile
    ([100, 50], [60, 50], 36, 3, 32, 64),                # 12
    ([64, 1, 300, 77], [64, 1, 300, 20], 8, 8, 16, 64),  # MHA, head_dim 64
    ([250, 64], [250, 33], 16, 2, 32, 64),               # 8, head_dim 64
    ([70, 30], [70, 30], 256, 1, 16, 64),                # 256: two sub-groups of 128 head slots
]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("case", range(len(PREFILL)))
def test_prefill_any_group(pa, dtype, case):
    ctx, qlen, Hq, Hkv, BS, D = PREFILL[case]
    c = prefill_case(300 + case, ctx, qlen, Hq, Hkv, BS, dtype, D=D)
    pa.pa_read_device_errors()
    out = prefill_run(pa, c, torch.float32)
    assert pa.pa_read_device_errors() == 0
    assert_attention_close(out, prefill_ref(c), dtype, f"prefill G{Hq // Hkv} D{D} {dtype}")
    out16 = prefill_run(pa, c, dtype)  # 16-bit output rows, staged (groups 1, 2) or direct
    assert_attention_close(out16, prefill_ref(c), dtype, f"prefill G{Hq // Hkv} D{D} {dtype} out")


@pytest.mark.parametrize("Hq,Hkv,D,BS", [(4, 4, 64, 16), (6, 2, 128, 32), (16, 1, 64, 16)])
def test_prefill_fp32_cache(pa, Hq, Hkv, D, BS):
    """fp32 caches prefill on the CUDA cores (each query token attends to its
    causal prefix in exact fp32 arithmetic): within 1e-5 of the oracle."""
    c = prefill_case(400 + Hq, [70, 1, 200, 33], [70, 1, 90, 0], Hq, Hkv, BS, torch.float32, D=D)
    pa.pa_read_device_errors()
    out = prefill_run(pa, c, torch.float32)
    assert pa.pa_read_device_errors() == 0
    assert_attention_close(out, prefill_ref(c), torch.float32, f"fp32 prefill G{Hq // Hkv}")


def test_prefill_fp32_skips_a_sequence_with_too_many_queries(pa):
    c = prefill_case(410, [30, 50], [30, 10], 4, 2, 16, torch.float32, poison=False, D=64)
    c["ctx"] = torch.tensor([20, 50], dtype=torch.int32)
    pa.pa_read_device_errors()
    out = prefill_run(pa, c, torch.float32)
    assert pa.pa_read_device_errors() & pa.PA_DEVERR_CONTEXT
    ref = oracle.paged_prefill(f64(c["q"][30:]), np.array([0, 10], np.int32), f64(c["k"]), f64(c["v"]),
                               c["tables"].numpy()[1:], np.array([50], np.int32), c["scale"], 16)
    assert_attention_close(out[30:], ref, torch.float32, "valid sequence")
    assert torch.isnan(out[:30]).all()
