"""Seeded synthetic inputs for paged decode.

This module only draws random numbers and shapes. It holds none of the
method's arithmetic (no slot or block indexing, no attention): block tables
and slot mappings come from a block pool (the library's, or the oracle's in
tests), which is handed the seeded free-block order drawn here.

Every tensor is created on the CPU with ``torch.Generator`` seeded per
workload, already rounded to its storage dtype.

Workloads (shapes follow LLaMA-style decode layers):
  tiny_fp32_mha        4 seqs, 4 heads, head_dim 64, block 16, lengths {1,17,45,100},
                       64-block pool; q/k/v ~ N(0,1); scale 1/8
  llama7b_mha_fp16     64 seqs, 32 heads, head_dim 128, block 16, lengths U{256..2048},
                       pool 1.1x the blocks needed; q/k/v ~ 0.5 N(0,1); fp16 out
  gqa_bf16             256 seqs, 32 query / 8 kv heads, head_dim 128, block 16,
                       lengths log-normal (median 1024, sigma 0.5) clipped to
                       [128, 4096]; q/k/v ~ N(0,1); fp32 out
  long_splitk_bf16     8 seqs, 32 query / 8 kv heads, head_dim 128, block 32,
                       lengths U{32768..131072}, pool exactly the blocks needed;
                       q,k ~ N(0,1), v ~ U(-1,1); fp32 out
  parallel_sampling_fp16  16 prompts x 5 branches, 32 heads, head_dim 128, block 16,
                       1000-token shared prefix, each branch adds U{1..256} tokens;
                       q/k/v ~ N(0,1); fp16 out
  prefill_llama7b_mha_bf16   8 prompts of 2048 tokens prefilled from empty, 32 heads,
                       head_dim 128, block 16; q/k/v ~ N(0,1); fp32 out
  chunked_prefill_gqa_bf16   16 sequences of 4096 tokens whose last 512 are new,
                       32 query / 8 kv heads, head_dim 128, block 16; fp32 out
  llama7b_mha_int8     llama7b_mha_fp16's shapes and values with an int8 cache (the fp16
                       values quantized at the slot write); fp16 query and out
  gqa_int8             gqa_bf16's shapes and values with an int8 cache; bf16 query, fp32 out
  prefix_cache_fp16    96 requests, each a system prompt (one of 4, lengths U{500..2000},
                       chosen uniformly) followed by U{1..256} user tokens; 32 heads,
                       head_dim 128, block 16; the prompts' blocks come from the prefix
                       cache (written once, shared by every request that uses them);
                       q/k/v ~ N(0,1); fp16 out
  beam_search_fp16     32 prompts of U{256..1024} tokens x beam width 4 (128 beams),
                       32 heads, head_dim 128, block 16; every step each beam picks a
                       parent among its prompt's 4 beams (uniform) and writes one token;
                       q/k/v ~ N(0,1); fp16 out
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Dict, Optional

import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16, "i8": torch.int8}


@dataclass(frozen=True)
class Spec:
    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    kv_dtype: str
    out_dtype: str
    seed: int
    # context-length law: ("fixed", [..]) | ("uniform", lo, hi) | ("lognormal", median, sigma, lo, hi)
    lengths: tuple
    pool_factor: Optional[float]  # pool = ceil(factor * needed); None = fixed pool_blocks
    pool_blocks: int = 0
    q_scale: float = 1.0
    kv_scale: float = 1.0
    v_uniform: bool = False
    partition_size: int = 0  # split-K partition (tokens) the workload is run with; 0 = unsplit
    q_len: int = 0  # prefill workloads: new query tokens per sequence (0 = decode)
    q_dtype: str = ""  # query (and source K/V) type when it differs from the cache's (int8 caches)
    # parallel sampling (copy-on-write) workload
    num_prompts: int = 0
    branches: int = 0
    prefix_len: int = 0
    max_divergent: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def torch_kv_dtype(self) -> torch.dtype:
        return DTYPES[self.kv_dtype]

    @property
    def torch_out_dtype(self) -> torch.dtype:
        return DTYPES[self.out_dtype]

    @property
    def torch_q_dtype(self) -> torch.dtype:
        """The query's type; also the type of the K/V values before an int8
        cache quantizes them."""
        return DTYPES[self.q_dtype or self.kv_dtype]


SPECS: Dict[str, Spec] = {
    "tiny_fp32_mha": Spec("tiny_fp32_mha", 4, 4, 4, 64, 16, "f32", "f32", 3400,
                          ("fixed", (1, 17, 45, 100)), None, pool_blocks=64),
    "llama7b_mha_fp16": Spec("llama7b_mha_fp16", 64, 32, 32, 128, 16, "f16", "f16", 3401,
                             ("uniform", 256, 2048), 1.1, q_scale=0.5, kv_scale=0.5),
    "gqa_bf16": Spec("gqa_bf16", 256, 32, 8, 128, 16, "bf16", "f32", 3402,
                     ("lognormal", 1024, 0.5, 128, 4096), 1.1),
    "long_splitk_bf16": Spec("long_splitk_bf16", 8, 32, 8, 128, 32, "bf16", "f32", 3403,
                             ("uniform", 32768, 131072), 1.0, v_uniform=True, partition_size=1024),
    "parallel_sampling_fp16": Spec("parallel_sampling_fp16", 80, 32, 32, 128, 16, "f16", "f16", 3404,
                                   ("parallel",), None, num_prompts=16, branches=5, prefix_len=1000,
                                   max_divergent=256),
    # prefill: a prompt's tokens attend causally over the paged cache
    "prefill_llama7b_mha_bf16": Spec("prefill_llama7b_mha_bf16", 8, 32, 32, 128, 16, "bf16", "f32", 3405,
                                     ("fixed", (2048,) * 8), 1.0, q_len=2048),
    "chunked_prefill_gqa_bf16": Spec("chunked_prefill_gqa_bf16", 16, 32, 8, 128, 16, "bf16", "f32", 3406,
                                     ("fixed", (4096,) * 16), 1.0, q_len=512),
    # int8 caches: the K/V values (fp16 / bf16) are quantized by the slot write
    "llama7b_mha_int8": Spec("llama7b_mha_int8", 64, 32, 32, 128, 16, "i8", "f16", 3408,
                             ("uniform", 256, 2048), 1.1, q_scale=0.5, kv_scale=0.5, q_dtype="f16"),
    "gqa_int8": Spec("gqa_int8", 256, 32, 8, 128, 16, "i8", "f32", 3409,
                     ("lognormal", 1024, 0.5, 128, 4096), 1.1, q_dtype="bf16"),
    # prefix cache: requests share a few system prompts' blocks through the prefix cache
    "prefix_cache_fp16": Spec("prefix_cache_fp16", 96, 32, 32, 128, 16, "f16", "f16", 3410,
                              ("prefix", 500, 2000), None, num_prompts=4, prefix_len=2000, max_divergent=256),
    # beam search: the beam step (fork, release, copy-on-write) on the device, then decode
    "beam_search_fp16": Spec("beam_search_fp16", 128, 32, 32, 128, 16, "f16", "f16", 3407,
                             ("uniform", 256, 1024), None, num_prompts=32, branches=4, max_divergent=512),
}


def scaled(spec: Spec, **changes) -> Spec:
    """A copy of spec with some fields changed (smaller parity cases)."""
    return replace(spec, **changes)


def _normal(gen: torch.Generator, shape, scale: float, dtype: torch.dtype) -> torch.Tensor:
    out = torch.empty(shape, dtype=dtype)
    flat = out.view(-1)
    chunk = 1 << 24
    for i in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - i)
        x = torch.randn(n, generator=gen, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        flat[i:i + n] = x.to(dtype)
    return out


def _uniform(gen: torch.Generator, shape, dtype: torch.dtype) -> torch.Tensor:
    out = torch.empty(shape, dtype=dtype)
    flat = out.view(-1)
    chunk = 1 << 24
    for i in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - i)
        x = torch.rand(n, generator=gen, dtype=torch.float32).mul_(2.0).sub_(1.0)
        flat[i:i + n] = x.to(dtype)
    return out


def context_lengths(spec: Spec, gen: torch.Generator) -> torch.Tensor:
    law = spec.lengths
    if law[0] == "fixed":
        return torch.tensor(law[1], dtype=torch.int32)
    if law[0] == "uniform":
        return torch.randint(law[1], law[2] + 1, (spec.num_seqs,), generator=gen, dtype=torch.int64).to(torch.int32)
    if law[0] == "lognormal":
        median, sigma, lo, hi = law[1:]
        z = torch.randn(spec.num_seqs, generator=gen, dtype=torch.float64)
        x = torch.round(median * torch.exp(sigma * z)).clamp_(lo, hi)
        return x.to(torch.int32)
    raise ValueError(law)


def make_decode_inputs(spec: Spec) -> dict:
    """Inputs for one decode step of a non-sampling workload.

    Returns CPU tensors: context_lens [S] int32 (the newest token included);
    free_order [NB] int32, the order in which the pool hands out physical
    blocks (a seeded permutation); k_pool/v_pool [NB, Hkv, bs, D] (every slot
    random; the newest token's slot is overwritten by the slot write);
    new_key/new_value [S, Hkv, D], the newest token of each sequence;
    query [S, Hq, D].
    """
    assert spec.lengths[0] != "parallel"
    gen = torch.Generator().manual_seed(spec.seed)
    dt = spec.torch_q_dtype  # int8 caches: the values before quantization
    ctx = context_lengths(spec, gen)
    needed = int(sum((int(c) + spec.block_size - 1) // spec.block_size for c in ctx.tolist()))
    nb = spec.pool_blocks if spec.pool_factor is None else int(math.ceil(spec.pool_factor * needed))
    nb = max(nb, needed)
    free_order = torch.randperm(nb, generator=gen).to(torch.int32)
    shape = (nb, spec.num_kv_heads, spec.block_size, spec.head_dim)
    k_pool = _normal(gen, shape, spec.kv_scale, dt)
    v_pool = _uniform(gen, shape, dt) if spec.v_uniform else _normal(gen, shape, spec.kv_scale, dt)
    kv_shape = (spec.num_seqs, spec.num_kv_heads, spec.head_dim)
    new_key = _normal(gen, kv_shape, spec.kv_scale, dt)
    new_value = _uniform(gen, kv_shape, dt) if spec.v_uniform else _normal(gen, kv_shape, spec.kv_scale, dt)
    query = _normal(gen, (spec.num_seqs, spec.num_heads, spec.head_dim), spec.q_scale, dt)
    return dict(context_lens=ctx, free_order=free_order, k_pool=k_pool, v_pool=v_pool,
                new_key=new_key, new_value=new_value, query=query, num_blocks=nb)


def make_parallel_sampling_inputs(spec: Spec) -> dict:
    """Inputs for the parallel-sampling workload: num_prompts prompts of
    prefix_len tokens, each forked into `branches` branches that append
    U{1..max_divergent} tokens each, then one decode over every branch.

    Returns CPU tensors: prefix_key/prefix_value [P, prefix_len, Hkv, D];
    divergent_lens [P, branches] int32; divergent_key/divergent_value
    [sum(divergent_lens), Hkv, D] in (prompt, branch, token) order;
    query [P * branches, Hq, D]; free_order [NB] int32; num_blocks.
    """
    assert spec.lengths[0] == "parallel"
    gen = torch.Generator().manual_seed(spec.seed)
    dt = spec.torch_kv_dtype
    P, B = spec.num_prompts, spec.branches
    div = torch.randint(1, spec.max_divergent + 1, (P, B), generator=gen, dtype=torch.int64).to(torch.int32)
    prefix_blocks = (spec.prefix_len + spec.block_size - 1) // spec.block_size
    per_branch = (spec.prefix_len + spec.max_divergent + spec.block_size - 1) // spec.block_size + 1
    nb = P * (prefix_blocks + B * per_branch)
    free_order = torch.randperm(nb, generator=gen).to(torch.int32)
    kv = (spec.num_kv_heads, spec.head_dim)
    prefix_key = _normal(gen, (P, spec.prefix_len) + kv, 1.0, dt)
    prefix_value = _normal(gen, (P, spec.prefix_len) + kv, 1.0, dt)
    total = int(div.sum())
    divergent_key = _normal(gen, (total,) + kv, 1.0, dt)
    divergent_value = _normal(gen, (total,) + kv, 1.0, dt)
    query = _normal(gen, (P * B, spec.num_heads, spec.head_dim), 1.0, dt)
    return dict(prefix_key=prefix_key, prefix_value=prefix_value, divergent_lens=div,
                divergent_key=divergent_key, divergent_value=divergent_value, query=query,
                free_order=free_order, num_blocks=nb)


def make_prefix_cache_inputs(spec: Spec) -> dict:
    """Inputs for the prefix-cache workload: num_prompts system prompts
    (lengths U{lo..hi} of the spec's law, random token ids), and num_seqs
    requests, each one system prompt (chosen uniformly) followed by
    U{1..max_divergent} user tokens.

    Returns CPU tensors: system_lens [P] int32; system_tokens [P, prefix_len]
    int32 (the first system_lens[p] are prompt p's tokens); choice [R] int32;
    user_lens [R] int32; prefix_key/prefix_value [P, prefix_len, Hkv, D];
    user_key/user_value [sum(user_lens), Hkv, D] in request order; query
    [R, Hq, D]; free_order [NB] int32; num_blocks (room for every prompt and
    request, with no block ever freed)."""
    assert spec.lengths[0] == "prefix"
    lo, hi = spec.lengths[1], spec.lengths[2]
    gen = torch.Generator().manual_seed(spec.seed)
    dt = spec.torch_kv_dtype
    P, R, bs = spec.num_prompts, spec.num_seqs, spec.block_size
    system_lens = torch.randint(lo, hi + 1, (P,), generator=gen, dtype=torch.int64).to(torch.int32)
    system_tokens = torch.randint(0, 1 << 30, (P, spec.prefix_len), generator=gen, dtype=torch.int64).to(torch.int32)
    choice = torch.randint(0, P, (R,), generator=gen, dtype=torch.int64).to(torch.int32)
    user_lens = torch.randint(1, spec.max_divergent + 1, (R,), generator=gen, dtype=torch.int64).to(torch.int32)
    nb = P * ((spec.prefix_len + bs - 1) // bs) + R * ((spec.max_divergent + bs - 1) // bs + 2)
    free_order = torch.randperm(nb, generator=gen).to(torch.int32)
    kv = (spec.num_kv_heads, spec.head_dim)
    prefix_key = _normal(gen, (P, spec.prefix_len) + kv, spec.kv_scale, dt)
    prefix_value = _normal(gen, (P, spec.prefix_len) + kv, spec.kv_scale, dt)
    total = int(user_lens.sum())
    user_key = _normal(gen, (total,) + kv, spec.kv_scale, dt)
    user_value = _normal(gen, (total,) + kv, spec.kv_scale, dt)
    query = _normal(gen, (R, spec.num_heads, spec.head_dim), spec.q_scale, dt)
    return dict(system_lens=system_lens, system_tokens=system_tokens, choice=choice, user_lens=user_lens,
                prefix_key=prefix_key, prefix_value=prefix_value, user_key=user_key, user_value=user_value,
                query=query, free_order=free_order, num_blocks=nb)


def make_prefill_inputs(spec: Spec) -> dict:
    """Inputs for one prefill step: every sequence holds context_lens - q_len
    cached tokens and appends q_len new ones (their K/V in new_key/new_value,
    their queries in query, sequence-major).

    Returns CPU tensors: context_lens [S]; free_order [NB]; k_pool/v_pool
    [NB, Hkv, bs, D]; new_key/new_value [S * q_len, Hkv, D]; query
    [S * q_len, Hq, D]; num_blocks."""
    assert spec.q_len > 0
    gen = torch.Generator().manual_seed(spec.seed)
    dt = spec.torch_kv_dtype
    ctx = context_lengths(spec, gen)
    needed = int(sum((int(c) + spec.block_size - 1) // spec.block_size for c in ctx.tolist()))
    nb = max(needed, int(math.ceil((spec.pool_factor or 1.0) * needed)))
    free_order = torch.randperm(nb, generator=gen).to(torch.int32)
    shape = (nb, spec.num_kv_heads, spec.block_size, spec.head_dim)
    k_pool = _normal(gen, shape, spec.kv_scale, dt)
    v_pool = _normal(gen, shape, spec.kv_scale, dt)
    T = spec.num_seqs * spec.q_len
    new_key = _normal(gen, (T, spec.num_kv_heads, spec.head_dim), spec.kv_scale, dt)
    new_value = _normal(gen, (T, spec.num_kv_heads, spec.head_dim), spec.kv_scale, dt)
    query = _normal(gen, (T, spec.num_heads, spec.head_dim), spec.q_scale, dt)
    return dict(context_lens=ctx, free_order=free_order, k_pool=k_pool, v_pool=v_pool, new_key=new_key,
                new_value=new_value, query=query, num_blocks=nb)


def make_beam_inputs(spec: Spec, distinct_steps: int = 16) -> dict:
    """Inputs for the beam-search workload: num_prompts prompts (lengths by the
    spec's law), each the root of `branches` beams; for `distinct_steps`
    steps (cycled by longer runs) each beam's parent among its prompt's beams
    and the new token's query, key and value. The pool has room for the
    prompts plus max_divergent new tokens on every beam.

    Returns CPU tensors: prompt_lens [P] int32; parents [steps, W] int32
    (global beam indices); query [steps, W, Hq, D]; new_key/new_value
    [steps, W, Hkv, D]; free_order [NB]; k_pool/v_pool [NB, Hkv, bs, D] (the
    prompts' cached K/V are whatever their blocks hold); num_blocks."""
    gen = torch.Generator().manual_seed(spec.seed)
    dt = spec.torch_kv_dtype
    P, B = spec.num_prompts, spec.branches
    W = P * B
    lens = context_lengths(replace(spec, num_seqs=P), gen)
    bs = spec.block_size
    needed = int(sum((int(c) + bs - 1) // bs for c in lens.tolist()))
    nb = needed + W * ((spec.max_divergent + bs - 1) // bs + 2)
    free_order = torch.randperm(nb, generator=gen).to(torch.int32)
    choice = torch.randint(0, B, (distinct_steps, W), generator=gen, dtype=torch.int64)
    parents = (choice + (torch.arange(W) // B * B)).to(torch.int32)
    shape = (nb, spec.num_kv_heads, bs, spec.head_dim)
    k_pool = _normal(gen, shape, 1.0, dt)
    v_pool = _normal(gen, shape, 1.0, dt)
    query = _normal(gen, (distinct_steps, W, spec.num_heads, spec.head_dim), 1.0, dt)
    new_key = _normal(gen, (distinct_steps, W, spec.num_kv_heads, spec.head_dim), 1.0, dt)
    new_value = _normal(gen, (distinct_steps, W, spec.num_kv_heads, spec.head_dim), 1.0, dt)
    return dict(prompt_lens=lens, parents=parents, query=query, new_key=new_key, new_value=new_value,
                free_order=free_order, k_pool=k_pool, v_pool=v_pool, num_blocks=nb)
