"""Helpers shared by the GPU parity tests: the oracle-side flow (tables from
the oracle's pool, caches updated by the oracle's byte copies, attention in
double) and the acceptance checks."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from oracle.block_pool import BlockPool as OPool, Sequence, append_tokens, fork

# Acceptance (fp16/bf16 inputs with fp32 accumulation; fp32 inputs).
TOL_16 = dict(max_abs=4e-3, rel_l2=1e-3)
TOL_32 = dict(max_abs=1e-5)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def raw(t: torch.Tensor) -> np.ndarray:
    """Bit-exact integer numpy view of a tensor's elements (shares memory for
    a contiguous CPU tensor, so in-place oracle writes land in the tensor)."""
    t = t.detach().to("cpu").contiguous()
    return t.view({8: torch.int64, 4: torch.int32, 2: torch.int16, 1: torch.int8}[t.element_size()]).numpy()


def assert_attention_close(out: torch.Tensor, ref: np.ndarray, kv_dtype: torch.dtype, what: str = "") -> None:
    o = f64(out)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    err = np.abs(o - ref)
    if kv_dtype == torch.float32:
        assert err.max() <= TOL_32["max_abs"], f"{what}: max abs {err.max():.3g}"
        return
    extra = 0.0
    rel_bound = TOL_16["rel_l2"]
    if out.dtype == torch.bfloat16:
        # bf16 output rounding (half an ulp, 2^-9 relative) on top of the bound
        extra = np.abs(ref) * 2.0 ** -8
        rel_bound = 3e-3
    assert np.all(err <= TOL_16["max_abs"] + extra), f"{what}: max abs {err.max():.3g}"
    denom = np.linalg.norm(ref)
    if denom > 0:
        rel = np.linalg.norm(o - ref) / denom
        assert rel <= rel_bound, f"{what}: rel L2 {rel:.3g}"


def oracle_decode_tables(ctx: np.ndarray, num_blocks: int, block_size: int, free_order, policy="fifo"):
    """Tables and newest-token slots from the oracle's pool (same rule, same order)."""
    pool = OPool(num_blocks, block_size, policy=policy, free_order=list(np.asarray(free_order)))
    mb = max(1, oracle.blocks_needed(int(ctx.max()), block_size))
    tables = np.full((len(ctx), mb), -1, np.int32)
    slots = np.empty(len(ctx), np.int32)
    for s, L in enumerate(ctx):
        seq = Sequence()
        append_tokens(pool, seq, int(L) - 1)
        sl, cow = append_tokens(pool, seq, 1)
        assert not cow
        slots[s] = sl[0]
        tables[s, :len(seq.block_table)] = seq.block_table
    return tables, slots


def oracle_sampling_flow(div: np.ndarray, prefix_len: int, num_blocks: int, block_size: int, free_order):
    """Oracle-side parallel-sampling flow: tables, prefix slots, divergent
    slots, copy-on-write pairs and context lengths."""
    P, B = div.shape
    pool = OPool(num_blocks, block_size, policy="fifo", free_order=list(np.asarray(free_order)))
    mb = oracle.blocks_needed(prefix_len + int(div.max()), block_size)
    seqs = []
    prefix_slots = []
    for p in range(P):
        root = Sequence()
        sl, cow = append_tokens(pool, root, prefix_len)
        assert not cow
        prefix_slots += sl
        seqs.append(root)
        for _ in range(1, B):
            seqs.append(fork(pool, root))
    slots, cows, ctx = [], [], []
    for i, seq in enumerate(seqs):
        sl, cow = append_tokens(pool, seq, int(div[i // B, i % B]))
        slots += sl
        cows += cow
        ctx.append(seq.num_tokens)
    tables = np.full((len(seqs), mb), -1, np.int32)
    for i, seq in enumerate(seqs):
        tables[i, :len(seq.block_table)] = seq.block_table
    return (tables, np.array(prefix_slots, np.int32), np.array(slots, np.int32),
            np.array(cows, np.int64).reshape(-1, 2), np.array(ctx, np.int32), pool)


def compact_for(k_pool: torch.Tensor, v_pool: torch.Tensor, table_row: np.ndarray, L: int, block_size: int,
                kv_heads=None):
    """The blocks one sequence uses, renumbered 0..nb-1 (results do not depend
    on physical ids, a pinned property of the oracle), optionally restricted
    to some kv heads, as float64 numpy pools plus the renumbered table."""
    nb = oracle.blocks_needed(L, block_size)
    ids = torch.from_numpy(table_row[:nb].astype(np.int64))
    kp = k_pool.index_select(0, ids)
    vp = v_pool.index_select(0, ids)
    if kv_heads is not None:
        h = torch.as_tensor(kv_heads, dtype=torch.int64)
        kp, vp = kp.index_select(1, h), vp.index_select(1, h)
    return kp.double().numpy(), vp.double().numpy(), np.arange(max(nb, 1), dtype=np.int32)[None, :]



def oracle_prefix_cache_flow(inputs: dict, block_size: int, prefix_len: int, max_user: int, finish_after=None):
    """The oracle's prefix-cache request flow on a workload's inputs."""
    from oracle.prefix_cache import request_flow
    return request_flow(inputs["system_lens"].numpy(), inputs["system_tokens"].numpy(), inputs["choice"].numpy(),
                        inputs["user_lens"].numpy(), int(inputs["num_blocks"]), inputs["free_order"].numpy(),
                        block_size, oracle.blocks_needed(prefix_len + max_user, block_size), finish_after)
