"""Host block pool with reference counts and copy-on-write (oracle side).

TEST INFRASTRUCTURE, like the rest of ``oracle/``. Plain Python, written from
the pages' description of the allocator; shares no code with the library's C++
pool, which it is compared against.

Rules, by source:
  * A pool of physical blocks with a free list; allocation takes a free block
    and sets its reference count to 1; freeing drops the count and returns the
    block to the free list at 0. [P2 "PagedAttention原理与KV Cache显存优化", §3.3
    and §4.2 (PhysicalBlockPool: free list, ref_counts, pop on allocate, append
    on free at 0)]; [P1 "PagedAttention 源码解析", §2–§3 (free_blocks pool,
    raise when empty)].
  * Which free block is taken: ``"lifo"`` takes the free list's last entry
    (``pop()`` in [P2] §4.2); ``"fifo"`` takes its first entry (``pop(0)`` in
    [P1] §3). Freed blocks go to the end of the list in both. The pages use
    both; callers pick one.
  * A sequence appends tokens one at a time; when its cached token count is a
    multiple of the block size it takes a new block first; token t goes to
    table[t // bs] at offset t % bs. [P2] §4.2 (append_token_kv).
  * Sharing (parallel sampling, prefix reuse) raises the count of every shared
    block. [P2] §3.4; [P4 "PagedAttention 实现细节", §3.2].
  * Copy-on-write: before writing into a block whose count is above 1, take a
    new block, copy the whole old block into it, drop the old block's count,
    give the new one count 1, point this sequence's table at it, then write.
    A block with count 1 is written in place. [P4] §3.3 (the Seq-A/Seq-B
    timeline); [P2] §3.4 (check before the write).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence as Sequence_, Tuple


class PoolExhausted(RuntimeError):
    pass


class BlockPool:
    def __init__(self, num_blocks: int, block_size: int, policy: str = "lifo",
                 free_order: Optional[Sequence_[int]] = None):
        """free_order: the initial free list (default 0 .. num_blocks-1);
        "fifo" hands its entries out from the front, "lifo" from the back."""
        if policy not in ("lifo", "fifo"):
            raise ValueError(policy)
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.policy = policy
        self.free_blocks: List[int] = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        if sorted(self.free_blocks) != list(range(num_blocks)):
            raise ValueError("free_order must be a permutation of the pool's block ids")
        self.ref_counts: List[int] = [0] * num_blocks

    def allocate(self) -> int:
        if not self.free_blocks:
            raise PoolExhausted("no free blocks")
        bid = self.free_blocks.pop() if self.policy == "lifo" else self.free_blocks.pop(0)
        self.ref_counts[bid] = 1
        return bid

    def share(self, bid: int) -> None:
        if self.ref_counts[bid] <= 0:
            raise ValueError(f"block {bid} is free")
        self.ref_counts[bid] += 1

    def free(self, bid: int) -> None:
        if self.ref_counts[bid] <= 0:
            raise ValueError(f"block {bid} is already free")
        self.ref_counts[bid] -= 1
        if self.ref_counts[bid] == 0:
            self.free_blocks.append(bid)

    def num_free(self) -> int:
        return len(self.free_blocks)


@dataclass
class Sequence:
    block_table: List[int] = field(default_factory=list)
    num_tokens: int = 0


def append_tokens(pool: BlockPool, seq: Sequence, n: int) -> Tuple[List[int], List[Tuple[int, int]]]:
    """Appends n tokens; returns (slot of each new token, copy-on-write
    (src, dst) pairs in the order they were taken)."""
    slots: List[int] = []
    cow: List[Tuple[int, int]] = []
    bs = pool.block_size
    for _ in range(n):
        t = seq.num_tokens
        if t % bs == 0:
            seq.block_table.append(pool.allocate())
        else:
            old = seq.block_table[t // bs]
            if pool.ref_counts[old] > 1:
                new = pool.allocate()
                cow.append((old, new))
                pool.free(old)
                seq.block_table[t // bs] = new
        slots.append(seq.block_table[t // bs] * bs + t % bs)
        seq.num_tokens += 1
    return slots, cow


def fork(pool: BlockPool, seq: Sequence) -> Sequence:
    """A new sequence sharing every block of seq (counts go up by one)."""
    for bid in seq.block_table:
        pool.share(bid)
    return Sequence(block_table=list(seq.block_table), num_tokens=seq.num_tokens)


def release(pool: BlockPool, seq: Sequence) -> None:
    """Drops the sequence's reference to each of its blocks."""
    for bid in seq.block_table:
        pool.free(bid)
    seq.block_table.clear()
    seq.num_tokens = 0


def beam_step(pool: BlockPool, beams: List[Sequence], parents: Sequence_[int]) -> Tuple[
        List[Sequence], List[int], List[Tuple[int, int]]]:
    """One beam-search step over the pool: new beam i continues old beam
    parents[i] and writes one new token. In this order: every new beam forks
    its parent (counts up), every old beam is released in beam order (blocks
    reaching count 0 return to the free list), then the new beams write their
    token in beam order, each by the copy-on-write rule. Returns (new beams,
    slot of each new beam's token, copy-on-write pairs in the order taken).
    [P2 "PagedAttention原理与KV Cache显存优化", §3.4 (beam search shares blocks
    between beams, copy on write when one diverges)]; [P4 "PagedAttention
    实现细节", §3.3 (the copy-on-write rule)]. The order of the three phases is
    a reading: the pages give the rule, not a schedule; forking before
    releasing keeps a parent's blocks alive for its children."""
    children = [fork(pool, beams[p]) for p in parents]
    for b in beams:
        release(pool, b)
    slots: List[int] = []
    cow: List[Tuple[int, int]] = []
    for c in children:
        s, pairs = append_tokens(pool, c, 1)
        slots += s
        cow += pairs
    return children, slots, cow
