"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times (the same batch builder, partition choice and step).

Tables, slots and copy-on-write pairs from the library's pool are compared
bit for bit with the oracle's pool; the caches after the step are compared
bit for bit with the oracle's byte copies; attention outputs are compared
with the oracle on every sequence (per kv head for the long-context workload,
whose sequences are too long to widen whole to float64)."""
import numpy as np
import pytest
import torch

import oracle
from _helpers import assert_attention_close, compact_for, f64, oracle_decode_tables, oracle_sampling_flow, raw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_340_b200 import _build
    _build.build()
    import paged_kv_cache_340_b200 as pa
    return pa


def _pools_equal(dev: torch.Tensor, host: torch.Tensor) -> bool:
    step = max(1, (256 << 20) // (host[0].numel() * host.element_size()))
    for i in range(0, host.shape[0], step):
        if not torch.equal(dev[i:i + step].cpu().view(torch.int16 if host.element_size() == 2 else torch.int32),
                           host[i:i + step].view(torch.int16 if host.element_size() == 2 else torch.int32)):
            return False
    return True


def _check_sequences(batch, k_host, v_host, seqs, kv_heads_per_seq=None):
    spec = batch.spec
    G = spec.num_heads // spec.num_kv_heads
    out = batch.out.cpu()
    q = batch.query.cpu()
    for s in seqs:
        L = int(batch.host_context_lens[s])
        heads = range(spec.num_kv_heads) if kv_heads_per_seq is None else kv_heads_per_seq(s)
        if kv_heads_per_seq is None:
            kp, vp, tab = compact_for(k_host, v_host, batch.host_tables[s], L, spec.block_size)
            ref = oracle.paged_decode(f64(q[s:s + 1]), kp, vp, tab, np.array([L], np.int32), spec.scale,
                                      spec.block_size)
            assert_attention_close(out[s:s + 1], ref, spec.torch_kv_dtype, f"{spec.name} seq {s}")
        else:
            for h in heads:
                kp, vp, tab = compact_for(k_host, v_host, batch.host_tables[s], L, spec.block_size, kv_heads=[h])
                qh = q[s:s + 1, h * G:(h + 1) * G]
                ref = oracle.paged_decode(f64(qh), kp, vp, tab, np.array([L], np.int32), spec.scale,
                                          spec.block_size)
                assert_attention_close(out[s:s + 1, h * G:(h + 1) * G], ref, spec.torch_kv_dtype,
                                       f"{spec.name} seq {s} kv head {h}")


def _decode_workload(pa, name, partition_size=None, per_head=None):
    from paged_kv_cache_340_b200.batch import build_decode_batch, run_step
    from paged_kv_cache_340_b200.workloads import SPECS, make_decode_inputs
    spec = SPECS[name]
    inputs = make_decode_inputs(spec)
    batch = build_decode_batch(spec, inputs, partition_size=partition_size)
    ctx = inputs["context_lens"].numpy()
    otab, oslots = oracle_decode_tables(ctx, inputs["num_blocks"], spec.block_size, inputs["free_order"].numpy())
    assert np.array_equal(batch.host_tables, otab)
    assert np.array_equal(batch.host_slots, oslots)
    run_step(batch)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    k_host, v_host = inputs["k_pool"], inputs["v_pool"]
    oracle.reshape_and_cache(raw(k_host), raw(v_host), raw(inputs["new_key"]), raw(inputs["new_value"]), oslots)
    assert _pools_equal(batch.k_cache, k_host) and _pools_equal(batch.v_cache, v_host)
    _check_sequences(batch, k_host, v_host, range(spec.num_seqs), per_head)
    return batch


def test_tiny_fp32_mha(pa):
    b = _decode_workload(pa, "tiny_fp32_mha")
    assert b.host_context_lens.tolist() == [1, 17, 45, 100]


def test_tiny_fp32_mha_split(pa):
    _decode_workload(pa, "tiny_fp32_mha", partition_size=32)


def test_llama7b_mha_fp16(pa):
    _decode_workload(pa, "llama7b_mha_fp16")


def test_llama7b_mha_fp16_split(pa):
    _decode_workload(pa, "llama7b_mha_fp16", partition_size=512)


def test_gqa_bf16(pa):
    _decode_workload(pa, "gqa_bf16")


def test_long_splitk_bf16(pa):
    b = _decode_workload(pa, "long_splitk_bf16", per_head=lambda s: [s % 8, (s * 5 + 3) % 8])
    assert b.partition_size > 0 and 2 * b.num_blocks * 32 * 8 * 128 * 2 > 2 ** 31  # K+V pools past 2 GiB


def test_parallel_sampling_fp16(pa):
    from paged_kv_cache_340_b200.batch import build_parallel_sampling_batch, run_step, write_prefix
    from paged_kv_cache_340_b200.workloads import SPECS, make_parallel_sampling_inputs
    spec = SPECS["parallel_sampling_fp16"]
    inp = make_parallel_sampling_inputs(spec)
    batch = build_parallel_sampling_batch(spec, inp)
    div = inp["divergent_lens"].numpy()
    otab, opre, oslots, ocow, octx, opool = oracle_sampling_flow(div, spec.prefix_len, inp["num_blocks"],
                                                                spec.block_size, inp["free_order"].numpy())
    assert np.array_equal(batch.host_tables, otab)
    assert np.array_equal(batch.host_prefix_slots, opre)
    assert np.array_equal(batch.host_slots, oslots)
    assert np.array_equal(batch.host_cow, ocow)
    assert np.array_equal(batch.host_context_lens, octx)
    assert len(ocow) == 4 * spec.num_prompts  # four copies of each prompt's partial prefix block
    write_prefix(batch)
    run_step(batch)
    torch.cuda.synchronize()
    assert pa.pa_read_device_errors() == 0
    NB, Hkv, bs, D = batch.k_cache.shape
    k_host = torch.zeros((NB, Hkv, bs, D), dtype=torch.float16)
    v_host = torch.zeros_like(k_host)
    P, L0 = spec.num_prompts, spec.prefix_len
    oracle.reshape_and_cache(raw(k_host), raw(v_host), raw(inp["prefix_key"].reshape(P * L0, Hkv, D)),
                             raw(inp["prefix_value"].reshape(P * L0, Hkv, D)), opre)
    oracle.copy_blocks(raw(k_host), raw(v_host), ocow)
    oracle.reshape_and_cache(raw(k_host), raw(v_host), raw(inp["divergent_key"]), raw(inp["divergent_value"]),
                             oslots)
    assert _pools_equal(batch.k_cache, k_host) and _pools_equal(batch.v_cache, v_host)
    _check_sequences(batch, k_host, v_host, range(spec.num_seqs))
    # A second step repeats the copies and writes. Branch 4 wrote into the
    # source block in place, so the re-copy changes bytes past the shorter
    # branches' contexts; every sequence's output stays bit-identical.
    out1 = batch.out.clone()
    run_step(batch)
    torch.cuda.synchronize()
    assert torch.equal(out1, batch.out)


def test_host_buffer_pipeline_matches_the_plain_step(pa):
    """HostStepPipeline (inputs from pinned host memory, output back to host,
    copies overlapping neighbouring steps) returns exactly what the plain
    device-resident step computes."""
    from paged_kv_cache_340_b200.batch import HostStepPipeline, build_decode_batch, run_step
    from paged_kv_cache_340_b200.workloads import SPECS, make_decode_inputs, scaled
    spec = scaled(SPECS["gqa_bf16"], num_seqs=32)
    b = build_decode_batch(spec, make_decode_inputs(spec))
    run_step(b)
    torch.cuda.synchronize()
    ref = b.out.cpu()
    pipe = HostStepPipeline(b)
    outs = [pipe.step() for _ in range(5)]
    pipe.drain()
    torch.cuda.synchronize()
    for o in outs[-2:]:
        assert torch.equal(o, ref)
    assert pipe.h2d_bytes > 0 and pipe.d2h_bytes == ref.numel() * ref.element_size()
