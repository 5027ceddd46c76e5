"""Prefix cache over the block pool (oracle side).

TEST INFRASTRUCTURE, like the rest of ``oracle/``. Plain Python written from
[P4 "PagedAttention 实现细节", §3.2 (Prefix Caching: CachedPrefix,
PrefixCacheManager.get_or_create / release)]; shares no code with the
library's C++ prefix cache, which it is compared against.

Rules, in the pages' order:
  * get_or_create(prompt tokens): if the prompt is cached, its use count goes
    up by one and its block ids are returned (a hit); otherwise
    ceil(len / block_size) blocks are allocated from the pool (all of them or,
    if the pool has too few free blocks, none and an error), recorded under
    the prompt with use count 1, and returned (a miss).
  * release(prompt tokens): an unknown prompt is ignored; otherwise its use
    count drops by one and at zero its blocks are freed and the entry removed.

Reading: the pages key the cache by a 12-hex-digit md5 of the token list and
never compare contents, so two prompts with one digest would share KV. Here
the key is the token list itself (equality of contents), which is what the
digest stands for.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Sequence as Sequence_, Tuple

import numpy as np

from .block_pool import BlockPool, PoolExhausted, Sequence, append_tokens, fork, release


@dataclass
class CachedPrefix:
    block_ids: List[int]
    ref_count: int
    content_length: int


class PrefixCacheManager:
    def __init__(self, pool: BlockPool):
        self.pool = pool
        self.cache: Dict[Tuple[int, ...], CachedPrefix] = {}

    def get_or_create(self, tokens: Sequence_[int]) -> Tuple[List[int], bool]:
        """Returns (block ids, hit)."""
        key = tuple(int(t) for t in tokens)
        if key in self.cache:
            entry = self.cache[key]
            entry.ref_count += 1
            return list(entry.block_ids), True
        bs = self.pool.block_size
        n = (len(key) + bs - 1) // bs
        if self.pool.num_free() < n:
            raise PoolExhausted("not enough free blocks for the prefix")
        ids = [self.pool.allocate() for _ in range(n)]
        self.cache[key] = CachedPrefix(block_ids=ids, ref_count=1, content_length=len(key))
        return list(ids), False

    def release(self, tokens: Sequence_[int]) -> None:
        key = tuple(int(t) for t in tokens)
        entry = self.cache.get(key)
        if entry is None:
            return
        entry.ref_count -= 1
        if entry.ref_count <= 0:
            for b in entry.block_ids:
                self.pool.free(b)
            del self.cache[key]

    def ref_count(self, tokens: Sequence_[int]) -> int:
        entry = self.cache.get(tuple(int(t) for t in tokens))
        return 0 if entry is None else entry.ref_count

    def num_entries(self) -> int:
        return len(self.cache)


def request_flow(system_lens, system_tokens, choice, user_lens, num_blocks: int, free_order, block_size: int,
                 max_blocks: int, finish_after=None):
    """Requests that share system prompts through the cache, on a FIFO pool
    handing out free_order: for request r in order, get_or_create its system
    prompt's blocks (a miss is followed by the write of the prompt's K/V, token
    t at slot block * block_size + t % block_size of the block holding t,
    [P3 "Ascend C ... PagedAttention融合算子" §3.1]); fork them into the
    request's own sequence; append its user tokens by the copy-on-write rule
    ([P4] §3.3); then every request in finish_after[r] releases its prompt and
    its blocks. Returns (ops as (kind, index, slots or pairs) in order, tables
    int32 [R, max_blocks] (-1 where unused or finished), context lengths [R],
    live [R])."""
    R = len(choice)
    pool = BlockPool(num_blocks, block_size, policy="fifo", free_order=[int(b) for b in free_order])
    mgr = PrefixCacheManager(pool)
    seqs = [None] * R
    ops = []

    def prompt_of(r):
        p = int(choice[r])
        return p, [int(t) for t in system_tokens[p][:int(system_lens[p])]]

    for r in range(R):
        p, prompt = prompt_of(r)
        ids, hit = mgr.get_or_create(prompt)
        if not hit:
            ops.append(("prefix", p, [ids[t // block_size] * block_size + t % block_size
                                      for t in range(len(prompt))]))
        seqs[r] = fork(pool, Sequence(block_table=list(ids), num_tokens=len(prompt)))
        slots, cow = append_tokens(pool, seqs[r], int(user_lens[r]))
        if cow:
            ops.append(("copy", r, [list(c) for c in cow]))
        ops.append(("user", r, slots))
        for j in (finish_after or {}).get(r, ()):
            mgr.release(prompt_of(j)[1])
            release(pool, seqs[j])
            seqs[j] = None
            ops.append(("finish", j, []))
    tables = np.full((R, max_blocks), -1, np.int32)
    ctx = np.zeros(R, np.int32)
    live = np.array([sq is not None for sq in seqs])
    for r, sq in enumerate(seqs):
        if sq is not None:
            tables[r, :len(sq.block_table)] = sq.block_table
            ctx[r] = sq.num_tokens
    return ops, tables, ctx, live
