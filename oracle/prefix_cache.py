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

from .block_pool import BlockPool, PoolExhausted


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
