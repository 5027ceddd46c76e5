"""Host flow of one decode step, on the library's own block pool.

An engine allocates blocks as sequences grow, writes each new token's K/V
through its slot, copies shared blocks before a sequence writes into them,
then runs decode. These helpers do that for the synthetic workloads: the pool
(``BlockPool``, the C++ pa_pool_* calls) hands out blocks in the workload's
seeded order and yields the block tables, slot mappings and copy-on-write
pairs; the device calls go through the C ABI.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

from . import (PA_POOL_FIFO, BlockPool, DevicePool, PrefixCache, pa_beam_step, pa_choose_partition, pa_copy_blocks,
               pa_copy_blocks_counted, pa_copy_blocks_q8, pa_decode, pa_decode_append, pa_decode_q8, pa_decode_splitk,
               pa_decode_splitk_q8, pa_prefill, pa_reshape_and_cache, pa_reshape_and_cache_q8, pa_splitk_reduce,
               pa_splitk_workspace_bytes)
from .workloads import Spec


@dataclass
class DecodeBatch:
    spec: Spec
    num_blocks: int
    k_cache: torch.Tensor       # device [NB, Hkv, bs, D]
    v_cache: torch.Tensor
    query: torch.Tensor         # device [S, Hq, D]
    out: torch.Tensor           # device [S, Hq, D] of spec.out_dtype
    block_tables: torch.Tensor  # device int32 [S, MB]
    context_lens: torch.Tensor  # device int32 [S]
    new_key: torch.Tensor       # device [T, Hkv, D], the tokens written this step
    new_value: torch.Tensor
    slot_mapping: torch.Tensor  # device int32 [T]
    cow_pairs: torch.Tensor     # device int64 [n, 2] (n may be 0)
    seq_order: torch.Tensor     # device int32 [S]: sequences longest first (scheduling order)
    max_context_len: int
    partition_size: int         # 0 = unpartitioned
    workspace: Optional[torch.Tensor]
    host_tables: np.ndarray
    host_slots: np.ndarray
    host_cow: np.ndarray
    host_context_lens: np.ndarray
    k_scale: Optional[torch.Tensor] = None  # int8 caches: device float32 [NB, Hkv, bs] row scales
    v_scale: Optional[torch.Tensor] = None
    # the step writes exactly each sequence's newest token, into the slot its
    # table gives, and decodes unpartitioned from a 16- or 32-bit cache: the
    # slot write and decode then run as one launch (pa_decode_append)
    fused_append: bool = False


def _blocks(n: int, bs: int) -> int:
    return (n + bs - 1) // bs


def longest_first(ctx: np.ndarray) -> np.ndarray:
    """Sequence indices by decreasing context length (ties in index order):
    the scheduling order that keeps a long sequence from starting last."""
    return np.argsort(-ctx.astype(np.int64), kind="stable").astype(np.int32)


def groups_longest_first(ctx: np.ndarray, group: int) -> np.ndarray:
    """Like longest_first, but sequences that share a prefix (consecutive
    groups of `group`) stay together, so the shared blocks are read while they
    are still in L2: groups by their longest member, members longest first."""
    g = ctx.reshape(-1, group).astype(np.int64)
    order = []
    for gi in np.argsort(-g.max(axis=1), kind="stable"):
        order += [gi * group + j for j in np.argsort(-g[gi], kind="stable")]
    return np.array(order, np.int32)


def build_decode_batch(spec: Spec, inputs: dict, device="cuda", partition_size: Optional[int] = None,
                       pool_policy: int = PA_POOL_FIFO) -> DecodeBatch:
    """Decode step of a non-sampling workload: every sequence already holds
    context_lens - 1 tokens; its newest token is written through its slot,
    then all sequences attend over context_lens tokens."""
    bs = spec.block_size
    ctx = inputs["context_lens"].numpy().astype(np.int32)
    S = ctx.shape[0]
    nb = int(inputs["num_blocks"])
    mb = max(1, _blocks(int(ctx.max()), bs))
    pool = BlockPool(nb, bs, pool_policy, free_order=inputs["free_order"].numpy())
    tables = np.full((S, mb), -1, np.int32)
    slots = np.empty(S, np.int32)
    for s in range(S):
        nt, _, cow = pool.append(tables[s], 0, int(ctx[s]) - 1, want_slots=False)
        nt, sl, cow2 = pool.append(tables[s], nt, 1)
        assert cow.size == 0 and cow2.size == 0
        slots[s] = sl[0]
    dev = torch.device(device)
    max_ctx = int(ctx.max())
    if partition_size is None:
        partition_size = spec.partition_size or pa_choose_partition(S, spec.num_kv_heads, max_ctx, bs, spec.head_dim,
                                                                    spec.torch_q_dtype)
    ws = None
    if partition_size:
        nbytes = pa_splitk_workspace_bytes(S, spec.num_heads, spec.head_dim, max_ctx, partition_size)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    if spec.kv_dtype == "i8":
        kc, vc, ks, vs = quantized_pool(inputs["k_pool"], inputs["v_pool"], dev)
    else:
        kc, vc, ks, vs = inputs["k_pool"].to(dev), inputs["v_pool"].to(dev), None, None
    return DecodeBatch(
        spec=spec, num_blocks=nb, k_cache=kc, v_cache=vc, k_scale=ks, v_scale=vs,
        query=inputs["query"].to(dev),
        out=torch.empty((S, spec.num_heads, spec.head_dim), dtype=spec.torch_out_dtype, device=dev),
        block_tables=torch.from_numpy(tables).to(dev), context_lens=torch.from_numpy(ctx).to(dev),
        new_key=inputs["new_key"].to(dev), new_value=inputs["new_value"].to(dev),
        slot_mapping=torch.from_numpy(slots).to(dev),
        cow_pairs=torch.empty((0, 2), dtype=torch.int64, device=dev),
        seq_order=torch.from_numpy(longest_first(ctx)).to(dev),
        max_context_len=max_ctx, partition_size=int(partition_size), workspace=ws,
        host_tables=tables, host_slots=slots, host_cow=np.empty((0, 2), np.int64), host_context_lens=ctx,
        fused_append=bool(partition_size == 0 and spec.kv_dtype != "i8" and newest_token_slots(tables, ctx, bs, slots)))


def newest_token_slots(tables: np.ndarray, ctx: np.ndarray, bs: int, slots: np.ndarray) -> bool:
    """Whether slots[s] is the slot of token ctx[s] - 1 of every sequence (as
    its table gives it), the case pa_decode_append covers."""
    if slots.shape[0] != ctx.shape[0] or (ctx < 1).any():
        return False
    pos = ctx.astype(np.int64) - 1
    blk = tables[np.arange(ctx.shape[0]), pos // bs].astype(np.int64)
    return bool(np.array_equal(blk * bs + pos % bs, slots.astype(np.int64)))


@dataclass
class SamplingBatch(DecodeBatch):
    prefix_key: torch.Tensor = None     # device [P * prefix_len, Hkv, D]
    prefix_value: torch.Tensor = None
    prefix_slots: torch.Tensor = None   # device int32 [P * prefix_len]
    host_prefix_slots: np.ndarray = None


def build_parallel_sampling_batch(spec: Spec, inputs: dict, device="cuda", partition_size: int = 0,
                                  pool_policy: int = PA_POOL_FIFO) -> SamplingBatch:
    """Parallel sampling: each prompt's prefix is written once, the prompt is
    forked into `branches` sequences sharing its blocks, and every branch
    appends its own tokens (the first write into the shared partial block
    copies it). Branches are processed in (prompt, branch) order."""
    bs = spec.block_size
    P, B, L0 = spec.num_prompts, spec.branches, spec.prefix_len
    div = inputs["divergent_lens"].numpy().astype(np.int32)
    nb = int(inputs["num_blocks"])
    mb = _blocks(L0 + int(div.max()), bs)
    pool = BlockPool(nb, bs, pool_policy, free_order=inputs["free_order"].numpy())
    S = P * B
    tables = np.full((S, mb), -1, np.int32)
    prefix_slots = np.empty(P * L0, np.int32)
    for p in range(P):
        root = p * B
        _, sl, cow = pool.append(tables[root], 0, L0)
        assert cow.size == 0
        prefix_slots[p * L0:(p + 1) * L0] = sl
        for b in range(1, B):
            pool.fork(tables[root], L0, tables[root + b])
    slots = np.empty(int(div.sum()), np.int32)
    cows = []
    ctx = np.empty(S, np.int32)
    pos = 0
    for p in range(P):
        for b in range(B):
            s = p * B + b
            n = int(div[p, b])
            nt, sl, cow = pool.append(tables[s], L0, n)
            slots[pos:pos + n] = sl
            pos += n
            cows.append(cow)
            ctx[s] = nt
    cow_all = np.concatenate(cows).astype(np.int64) if cows else np.empty((0, 2), np.int64)
    dev = torch.device(device)
    NB, Hkv, D = nb, spec.num_kv_heads, spec.head_dim
    dt = spec.torch_kv_dtype
    max_ctx = int(ctx.max())
    ws = None
    if partition_size:
        ws = torch.empty(pa_splitk_workspace_bytes(S, spec.num_heads, D, max_ctx, partition_size),
                         dtype=torch.uint8, device=dev)
    return SamplingBatch(
        spec=spec, num_blocks=nb,
        k_cache=torch.zeros((NB, Hkv, bs, D), dtype=dt, device=dev),
        v_cache=torch.zeros((NB, Hkv, bs, D), dtype=dt, device=dev),
        query=inputs["query"].to(dev),
        out=torch.empty((S, spec.num_heads, D), dtype=spec.torch_out_dtype, device=dev),
        block_tables=torch.from_numpy(tables).to(dev), context_lens=torch.from_numpy(ctx).to(dev),
        new_key=inputs["divergent_key"].to(dev), new_value=inputs["divergent_value"].to(dev),
        slot_mapping=torch.from_numpy(slots).to(dev), cow_pairs=torch.from_numpy(cow_all).to(dev),
        seq_order=torch.from_numpy(groups_longest_first(ctx, B)).to(dev),
        max_context_len=max_ctx, partition_size=int(partition_size), workspace=ws,
        host_tables=tables, host_slots=slots, host_cow=cow_all, host_context_lens=ctx,
        prefix_key=inputs["prefix_key"].reshape(P * L0, Hkv, D).to(dev),
        prefix_value=inputs["prefix_value"].reshape(P * L0, Hkv, D).to(dev),
        prefix_slots=torch.from_numpy(prefix_slots).to(dev), host_prefix_slots=prefix_slots)


def shared_prefix_order(ctx: np.ndarray, group_of: np.ndarray) -> np.ndarray:
    """Scheduling order for sequences that share prefixes: sequences of one
    group (same prefix) stay together, so the shared blocks are read while
    they are still in L2; groups by their longest member, members longest
    first."""
    ctx = ctx.astype(np.int64)
    groups = np.unique(group_of)
    longest = np.array([ctx[group_of == g].max() for g in groups])
    order = []
    for gi in np.argsort(-longest, kind="stable"):
        members = np.nonzero(group_of == groups[gi])[0]
        order += members[np.argsort(-ctx[members], kind="stable")].tolist()
    return np.array(order, np.int32)


@dataclass
class PrefixOp:
    """One device step of the prefix-cache flow, in the order the host took it."""
    kind: str          # "prefix": write system prompt `index`'s K/V; "copy": copy-on-write pairs;
                       # "user": request `index`'s own tokens; "finish": request `index` is done
    index: int
    slots: np.ndarray  # int32 slots ("prefix", "user") or int64 [n, 2] pairs ("copy"); empty for "finish"


def prefix_cache_flow(spec: Spec, inputs: dict, finish_after: Optional[dict] = None,
                      pool_policy: int = PA_POOL_FIFO):
    """Host side of requests that share system prompts through the prefix
    cache ([P4] "PagedAttention 实现细节" §3.2, with the copy-on-write rule of
    §3.3). For request r in order: get_or_create its system prompt's blocks
    (a miss is followed by the write of the prompt's K/V into them); fork them
    into the request's own table row (its own reference to each block); append
    its user tokens (the first write into the shared partial last block
    copies it). finish_after maps r to requests that finish once r is set up:
    the cache releases their prompt and the pool their blocks, which later
    requests may then be handed. Returns (ops in order, tables [R, MB], ctx
    [R], live [R] bool)."""
    bs = spec.block_size
    lens = inputs["system_lens"].numpy().astype(np.int64)
    toks = inputs["system_tokens"].numpy()
    choice = inputs["choice"].numpy().astype(np.int64)
    ulens = inputs["user_lens"].numpy().astype(np.int64)
    R = choice.shape[0]
    mb = _blocks(spec.prefix_len + spec.max_divergent, bs)
    pool = BlockPool(int(inputs["num_blocks"]), bs, pool_policy, free_order=inputs["free_order"].numpy())
    cache = PrefixCache(pool)
    tables = np.full((R, mb), -1, np.int32)
    ctx = np.zeros(R, np.int32)
    live = np.zeros(R, bool)
    ops = []
    for r in range(R):
        p = int(choice[r])
        L0 = int(lens[p])
        ids, hit = cache.get_or_create(toks[p, :L0])
        ids = np.array(ids, np.int32)
        if not hit:  # the prompt's K/V go into the blocks the cache just took
            t = np.arange(L0, dtype=np.int64)
            ops.append(PrefixOp("prefix", p, (ids[t // bs].astype(np.int64) * bs + t % bs).astype(np.int32)))
        pool.fork(ids, L0, tables[r])
        nt, sl, cow = pool.append(tables[r], L0, int(ulens[r]), cow_capacity=4)
        if cow.shape[0]:
            ops.append(PrefixOp("copy", r, cow))
        ops.append(PrefixOp("user", r, sl))
        ctx[r] = nt
        live[r] = True
        for j in (finish_after or {}).get(r, ()):
            assert live[j]
            cache.release(toks[int(choice[j]), :int(lens[int(choice[j])])])
            pool.release(tables[j], int(ctx[j]))
            tables[j] = -1
            ctx[j] = 0
            live[j] = False
            ops.append(PrefixOp("finish", j, np.empty(0, np.int32)))
    return ops, tables, ctx, live


def build_prefix_cache_batch(spec: Spec, inputs: dict, device="cuda", pool_policy: int = PA_POOL_FIFO
                             ) -> SamplingBatch:
    """The prefix-cache workload as a decode step: every system prompt the
    requests use is written once (set-up, write_prefix); a step copies the
    shared partial blocks each request writes into, writes the requests' own
    tokens and decodes every request."""
    ops, tables, ctx, _ = prefix_cache_flow(spec, inputs, pool_policy=pool_policy)
    dev = torch.device(device)
    Hkv, D, bs = spec.num_kv_heads, spec.head_dim, spec.block_size
    R = ctx.shape[0]
    pre = [o for o in ops if o.kind == "prefix"]
    lens = inputs["system_lens"].numpy()
    prefix_key = torch.cat([inputs["prefix_key"][o.index, :int(lens[o.index])] for o in pre])
    prefix_value = torch.cat([inputs["prefix_value"][o.index, :int(lens[o.index])] for o in pre])
    prefix_slots = np.concatenate([o.slots for o in pre]).astype(np.int32)
    cows = [o.slots for o in ops if o.kind == "copy"]
    cow_all = np.concatenate(cows).astype(np.int64) if cows else np.empty((0, 2), np.int64)
    slots = np.concatenate([o.slots for o in ops if o.kind == "user"]).astype(np.int32)
    nb = int(inputs["num_blocks"])
    dt = spec.torch_kv_dtype
    return SamplingBatch(
        spec=spec, num_blocks=nb,
        k_cache=torch.zeros((nb, Hkv, bs, D), dtype=dt, device=dev),
        v_cache=torch.zeros((nb, Hkv, bs, D), dtype=dt, device=dev),
        query=inputs["query"].to(dev),
        out=torch.empty((R, spec.num_heads, D), dtype=spec.torch_out_dtype, device=dev),
        block_tables=torch.from_numpy(tables).to(dev), context_lens=torch.from_numpy(ctx).to(dev),
        new_key=inputs["user_key"].to(dev), new_value=inputs["user_value"].to(dev),
        slot_mapping=torch.from_numpy(slots).to(dev), cow_pairs=torch.from_numpy(cow_all).to(dev),
        seq_order=torch.from_numpy(shared_prefix_order(ctx, inputs["choice"].numpy())).to(dev),
        max_context_len=int(ctx.max()), partition_size=0, workspace=None,
        host_tables=tables, host_slots=slots, host_cow=cow_all, host_context_lens=ctx,
        prefix_key=prefix_key.to(dev), prefix_value=prefix_value.to(dev),
        prefix_slots=torch.from_numpy(prefix_slots).to(dev), host_prefix_slots=prefix_slots)


def write_prefix(batch: SamplingBatch, stream=None) -> None:
    """Writes every prompt's prefix into the pool (set-up, once)."""
    pa_reshape_and_cache(batch.prefix_key, batch.prefix_value, batch.k_cache, batch.v_cache, batch.prefix_slots,
                         stream=stream)


def quantized_pool(k_pool: torch.Tensor, v_pool: torch.Tensor, device, chunk_blocks: int = 4096):
    """int8 codes and row scales of whole K/V pools [NB, Hkv, bs, D] (values of
    a 16- or 32-bit type), made by the library's quantizing slot write with
    every slot written once (slot b * bs + o <- pool row (b, :, o))."""
    NB, Hkv, bs, D = k_pool.shape
    dev = torch.device(device)
    kc = torch.empty((NB, Hkv, bs, D), dtype=torch.int8, device=dev)
    vc = torch.empty_like(kc)
    ks = torch.empty((NB, Hkv, bs), dtype=torch.float32, device=dev)
    vs = torch.empty_like(ks)
    for b0 in range(0, NB, chunk_blocks):
        b1 = min(NB, b0 + chunk_blocks)
        kk = k_pool[b0:b1].to(dev).permute(0, 2, 1, 3).reshape(-1, Hkv, D).contiguous()
        vv = v_pool[b0:b1].to(dev).permute(0, 2, 1, 3).reshape(-1, Hkv, D).contiguous()
        slots = torch.arange(b0 * bs, b1 * bs, dtype=torch.int32, device=dev)
        pa_reshape_and_cache_q8(kk, vv, kc, vc, ks, vs, slots)
    return kc, vc, ks, vs


def run_step(batch: DecodeBatch, stream=None) -> None:
    """One pass of the hot path: copy-on-write block copies (if any), the slot
    write of this step's tokens, then decode (split-K + reduce when the batch
    has a partition size). int8 caches quantize at the slot write. When the
    step writes only each sequence's newest token (fused_append), the slot
    write and decode are one launch."""
    q8 = batch.k_scale is not None
    if batch.cow_pairs.shape[0]:
        if q8:
            pa_copy_blocks_q8(batch.k_cache, batch.v_cache, batch.k_scale, batch.v_scale, batch.cow_pairs,
                              stream=stream)
        else:
            pa_copy_blocks(batch.k_cache, batch.v_cache, batch.cow_pairs, stream=stream)
    if batch.fused_append:
        pa_decode_append(batch.out, batch.query, batch.new_key, batch.new_value, batch.k_cache, batch.v_cache,
                         batch.block_tables, batch.context_lens, batch.spec.scale, seq_order=batch.seq_order,
                         stream=stream)
        return
    if q8:
        pa_reshape_and_cache_q8(batch.new_key, batch.new_value, batch.k_cache, batch.v_cache, batch.k_scale,
                                batch.v_scale, batch.slot_mapping, stream=stream)
    else:
        pa_reshape_and_cache(batch.new_key, batch.new_value, batch.k_cache, batch.v_cache, batch.slot_mapping,
                             stream=stream)
    run_decode(batch, stream)


def run_decode(batch: DecodeBatch, stream=None) -> None:
    spec = batch.spec
    if batch.k_scale is not None:
        if batch.partition_size:
            pa_decode_splitk_q8(batch.workspace, batch.query, batch.k_cache, batch.v_cache, batch.k_scale,
                                batch.v_scale, batch.block_tables, batch.context_lens, spec.scale,
                                batch.max_context_len, batch.partition_size, seq_order=batch.seq_order, stream=stream)
            pa_splitk_reduce(batch.out, batch.workspace, batch.context_lens, batch.max_context_len,
                             batch.partition_size, stream=stream)
        else:
            pa_decode_q8(batch.out, batch.query, batch.k_cache, batch.v_cache, batch.k_scale, batch.v_scale,
                         batch.block_tables, batch.context_lens, spec.scale, seq_order=batch.seq_order, stream=stream)
        return
    if batch.partition_size:
        pa_decode_splitk(batch.workspace, batch.query, batch.k_cache, batch.v_cache, batch.block_tables,
                         batch.context_lens, spec.scale, batch.max_context_len, batch.partition_size,
                         seq_order=batch.seq_order, stream=stream)
        pa_splitk_reduce(batch.out, batch.workspace, batch.context_lens, batch.max_context_len,
                         batch.partition_size, stream=stream)
    else:
        pa_decode(batch.out, batch.query, batch.k_cache, batch.v_cache, batch.block_tables, batch.context_lens,
                  spec.scale, seq_order=batch.seq_order, stream=stream)


class HostStepPipeline:
    """Decode steps driven from pinned host buffers, with the copies of one
    step overlapping the kernels of its neighbours.

    Each step copies its inputs (query, new K/V, slots, block tables, context
    lengths, schedule and copy-on-write pairs) host -> device, runs the hot
    path (run_step) and copies the output back. Device inputs and outputs are
    double-buffered: step i's host->device copies run on a copy stream while
    step i-1 computes, and step i-1's output returns on a second copy stream
    while step i computes. The KV pools stay resident on the device.
    """

    _IN = ("query", "new_key", "new_value", "slot_mapping", "block_tables", "context_lens", "seq_order",
           "cow_pairs")

    def __init__(self, batch: DecodeBatch):
        import copy
        self.batch = batch
        self.names = [n for n in self._IN if getattr(batch, n).numel()]
        self.host_in = {n: getattr(batch, n).cpu().pin_memory() for n in self.names}
        self.host_out = [torch.empty(batch.out.shape, dtype=batch.out.dtype, pin_memory=True) for _ in range(2)]
        self.views = []
        for _ in range(2):
            v = copy.copy(batch)
            for n in self.names:
                setattr(v, n, torch.empty_like(getattr(batch, n)))
            v.out = torch.empty_like(batch.out)
            if batch.workspace is not None:
                v.workspace = torch.empty_like(batch.workspace)
            self.views.append(v)
        self.h2d = torch.cuda.Stream()
        self.d2h = torch.cuda.Stream()
        self.in_ready = [torch.cuda.Event() for _ in range(2)]
        self.in_free = [torch.cuda.Event() for _ in range(2)]
        self.out_ready = [torch.cuda.Event() for _ in range(2)]
        self.out_free = [torch.cuda.Event() for _ in range(2)]
        self.i = 0

    @property
    def h2d_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.host_in.values())

    @property
    def d2h_bytes(self) -> int:
        return self.host_out[0].numel() * self.host_out[0].element_size()

    def start(self, stream=None) -> None:
        """Orders the copy streams after everything already on `stream` (e.g.
        a timing event), so that no copy of the next step starts before it."""
        comp = stream or torch.cuda.current_stream()
        self.h2d.wait_stream(comp)
        self.d2h.wait_stream(comp)

    def step(self, stream=None) -> torch.Tensor:
        """Enqueues one step; returns the pinned host tensor that will hold its
        output once the stream work completes."""
        comp = stream or torch.cuda.current_stream()
        j = self.i & 1
        v = self.views[j]
        if self.i >= 2:
            self.h2d.wait_event(self.in_free[j])
        with torch.cuda.stream(self.h2d):
            for n in self.names:
                getattr(v, n).copy_(self.host_in[n], non_blocking=True)
            self.in_ready[j].record(self.h2d)
        comp.wait_event(self.in_ready[j])
        if self.i >= 2:
            comp.wait_event(self.out_free[j])
        run_step(v, stream=comp)
        self.in_free[j].record(comp)
        self.out_ready[j].record(comp)
        self.d2h.wait_event(self.out_ready[j])
        with torch.cuda.stream(self.d2h):
            self.host_out[j].copy_(v.out, non_blocking=True)
            self.out_free[j].record(self.d2h)
        self.i += 1
        return self.host_out[j]

    def drain(self, stream=None) -> None:
        """Makes `stream` wait for every copy enqueued so far."""
        comp = stream or torch.cuda.current_stream()
        for j in range(2):
            if self.i > j:
                comp.wait_event(self.out_free[j])


@dataclass
class PrefillBatch:
    spec: Spec
    num_blocks: int
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    query: torch.Tensor         # device [T, Hq, D], sequence-major
    out: torch.Tensor           # device [T, Hq, D]
    q_start: torch.Tensor       # device int32 [S + 1]
    block_tables: torch.Tensor
    context_lens: torch.Tensor
    new_key: torch.Tensor       # device [T, Hkv, D]
    new_value: torch.Tensor
    slot_mapping: torch.Tensor  # device int32 [T]
    max_q_len: int
    host_tables: np.ndarray
    host_slots: np.ndarray
    host_context_lens: np.ndarray
    host_q_start: np.ndarray


def build_prefill_batch(spec: Spec, inputs: dict, device="cuda", pool_policy: int = PA_POOL_FIFO) -> PrefillBatch:
    """Prefill step: every sequence holds context_lens - q_len tokens and
    appends q_len new ones; their K/V go in through their slots, then their
    queries attend causally over the cache."""
    bs = spec.block_size
    ctx = inputs["context_lens"].numpy().astype(np.int32)
    S, ql = ctx.shape[0], spec.q_len
    nb = int(inputs["num_blocks"])
    pool = BlockPool(nb, bs, pool_policy, free_order=inputs["free_order"].numpy())
    tables = np.full((S, max(1, _blocks(int(ctx.max()), bs))), -1, np.int32)
    slots = np.empty(S * ql, np.int32)
    for s in range(S):
        nt, _, _ = pool.append(tables[s], 0, int(ctx[s]) - ql, want_slots=False)
        _, sl, _ = pool.append(tables[s], nt, ql)
        slots[s * ql:(s + 1) * ql] = sl
    q_start = (np.arange(S + 1) * ql).astype(np.int32)
    dev = torch.device(device)
    return PrefillBatch(
        spec=spec, num_blocks=nb, k_cache=inputs["k_pool"].to(dev), v_cache=inputs["v_pool"].to(dev),
        query=inputs["query"].to(dev),
        out=torch.empty((S * ql, spec.num_heads, spec.head_dim), dtype=spec.torch_out_dtype, device=dev),
        q_start=torch.from_numpy(q_start).to(dev), block_tables=torch.from_numpy(tables).to(dev),
        context_lens=torch.from_numpy(ctx).to(dev), new_key=inputs["new_key"].to(dev),
        new_value=inputs["new_value"].to(dev), slot_mapping=torch.from_numpy(slots).to(dev), max_q_len=ql,
        host_tables=tables, host_slots=slots, host_context_lens=ctx, host_q_start=q_start)


def run_prefill_step(batch: PrefillBatch, stream=None) -> None:
    """The new tokens' K/V through their slots, then causal attention."""
    pa_reshape_and_cache(batch.new_key, batch.new_value, batch.k_cache, batch.v_cache, batch.slot_mapping,
                         stream=stream)
    pa_prefill(batch.out, batch.query, batch.q_start, batch.max_q_len, batch.k_cache, batch.v_cache,
               batch.block_tables, batch.context_lens, batch.spec.scale, stream=stream)


def prefill_flops(spec: Spec, ctx: np.ndarray) -> int:
    """Causal attention FLOPs of a prefill step: query token i of a sequence
    sees pos + 1 keys, 4 * head_dim FLOPs per key (QK^T and PV), per head."""
    ql = spec.q_len
    total = 0
    for L in ctx.astype(np.int64):
        first = int(L) - ql + 1                     # keys seen by the first new token
        keys = ql * (2 * first + ql - 1) // 2       # sum over the q_len tokens
        total += 4 * spec.head_dim * keys * spec.num_heads
    return total


@dataclass
class BeamBatch:
    spec: Spec
    num_blocks: int
    pool: DevicePool
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    tables: list                # two device int32 [W, MB] buffers: step i reads [i % 2], writes [(i + 1) % 2]
    context_lens: list          # two device int32 [W]
    parents: torch.Tensor       # device int32 [steps, W]
    query: torch.Tensor         # device [steps, W, Hq, D]
    new_key: torch.Tensor       # device [steps, W, Hkv, D]
    new_value: torch.Tensor
    slot_mapping: torch.Tensor  # device int32 [W]
    cow_pairs: torch.Tensor     # device int64 [W, 2]
    num_cow: torch.Tensor       # device int32 [1]
    out: torch.Tensor           # device [W, Hq, D]
    host_prompt_lens: np.ndarray
    host_pool: BlockPool        # the host pool the prompts were written with (state before step 0)
    host_tables: np.ndarray     # [W, MB] before step 0
    steps_done: int = 0


def build_beam_batch(spec: Spec, inputs: dict, device="cuda", pool_policy: int = PA_POOL_FIFO) -> BeamBatch:
    """Beam search start: each prompt's tokens go into blocks of the host pool
    (a prefill), the prompt is forked into `branches` beams sharing them, and
    the pool's state is loaded into a device pool for the device beam steps."""
    bs, B, P = spec.block_size, spec.branches, spec.num_prompts
    W = P * B
    lens = inputs["prompt_lens"].numpy().astype(np.int32)
    nb = int(inputs["num_blocks"])
    mb = _blocks(int(lens.max()) + spec.max_divergent, bs) + 1
    pool = BlockPool(nb, bs, pool_policy, free_order=inputs["free_order"].numpy())
    tables = np.full((W, mb), -1, np.int32)
    for p in range(P):
        pool.append(tables[p * B], 0, int(lens[p]), want_slots=False)
        for b in range(1, B):
            pool.fork(tables[p * B], int(lens[p]), tables[p * B + b])
    dev = torch.device(device)
    ctx = np.repeat(lens, B).astype(np.int32)
    dpool = DevicePool(nb, bs, pool_policy, device=dev, host_pool=pool)
    tb = [torch.from_numpy(tables).to(dev), torch.empty((W, mb), dtype=torch.int32, device=dev)]
    cl = [torch.from_numpy(ctx).to(dev), torch.empty(W, dtype=torch.int32, device=dev)]
    return BeamBatch(
        spec=spec, num_blocks=nb, pool=dpool, k_cache=inputs["k_pool"].to(dev), v_cache=inputs["v_pool"].to(dev),
        tables=tb, context_lens=cl, parents=inputs["parents"].to(dev), query=inputs["query"].to(dev),
        new_key=inputs["new_key"].to(dev), new_value=inputs["new_value"].to(dev),
        slot_mapping=torch.empty(W, dtype=torch.int32, device=dev),
        cow_pairs=torch.empty((W, 2), dtype=torch.int64, device=dev),
        num_cow=torch.zeros(1, dtype=torch.int32, device=dev),
        out=torch.empty((W, spec.num_heads, spec.head_dim), dtype=spec.torch_out_dtype, device=dev),
        host_prompt_lens=lens, host_pool=pool, host_tables=tables)


def run_beam_step(b: BeamBatch, stream=None, events=None) -> None:
    """One beam-search decode step, all on the device: beam step (fork,
    release, copy-on-write decisions), counted block copy, then the slot
    write of the new tokens and decode over the new tables as one launch
    (each new token is its beam's newest, in a block that beam alone holds
    after the copy-on-write). events (optional, 5 CUDA events) are recorded
    between the launches (the fourth right after the third)."""
    i = b.steps_done
    k = i % b.parents.shape[0]
    src, dst = i % 2, (i + 1) % 2

    def mark(j):
        if events is not None:
            events[j].record(stream if stream is not None else torch.cuda.current_stream())

    mark(0)
    pa_beam_step(b.pool, b.tables[src], b.context_lens[src], b.parents[k], b.tables[dst], b.context_lens[dst],
                 b.slot_mapping, b.cow_pairs, b.num_cow, stream=stream)
    mark(1)
    pa_copy_blocks_counted(b.k_cache, b.v_cache, b.cow_pairs, b.num_cow, stream=stream)
    mark(2)
    mark(3)
    pa_decode_append(b.out, b.query[k], b.new_key[k], b.new_value[k], b.k_cache, b.v_cache, b.tables[dst],
                     b.context_lens[dst], b.spec.scale, stream=stream)
    mark(4)
    b.steps_done = i + 1


def beam_decode_bytes(b: BeamBatch, step: int) -> int:
    """Algorithmic bytes of the decode of beam step `step` (0-based): every
    beam of prompt p holds prompt_lens[p] + step + 1 tokens after it (beams of
    one prompt grow together)."""
    s = b.spec
    elt = s.torch_kv_dtype.itemsize
    ctx = (b.host_prompt_lens.astype(np.int64) + step + 1).repeat(s.branches)
    nblk = (ctx + s.block_size - 1) // s.block_size
    W = ctx.shape[0]
    return int(ctx.sum() * 2 * s.num_kv_heads * s.head_dim * elt + W * s.num_heads * s.head_dim *
               (elt + s.torch_out_dtype.itemsize) + 4 * nblk.sum() + 4 * W)


def host_beam_step(pool: BlockPool, tables: np.ndarray, ctx: np.ndarray, parents: np.ndarray):
    """The same step on the host pool (the path without the device pool):
    fork every chosen parent, release the old beams, append one token to each
    new beam. Returns (new tables, new context lengths, slots, copy pairs)."""
    W_new, mb = parents.shape[0], tables.shape[1]
    new_t = np.full((W_new, mb), -1, np.int32)
    for i, p in enumerate(parents):
        pool.fork(tables[p], int(ctx[p]), new_t[i])
    for j in range(tables.shape[0]):
        pool.release(tables[j], int(ctx[j]))
    new_c = np.empty(W_new, np.int32)
    slots = np.empty(W_new, np.int32)
    pairs = []
    for i, p in enumerate(parents):
        nt, sl, cow = pool.append(new_t[i], int(ctx[p]), 1)
        new_c[i] = nt
        slots[i] = sl[0]
        pairs.append(cow)
    cow = np.concatenate(pairs).astype(np.int64) if pairs else np.empty((0, 2), np.int64)
    return new_t, new_c, slots, cow
