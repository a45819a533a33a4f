"""Host-side block manager: the bookkeeping that produces the library's inputs.

It keeps a free list of physical KV blocks, a reference count per block and,
for every sequence, the list of physical blocks its logical blocks map to.
From that it emits the three integer arrays the device calls consume:
``block_tables`` (int32 ``[S, MB]``), ``slot_mapping`` (int64, one slot per
new token) and ``block_mapping`` (int64 ``[P, 2]`` copy-on-write pairs).

Behaviour follows the pages:

* "vLLM PagedAttention 大模型推理架构深度实战", section 2.2: fixed 16-token
  blocks, a per-sequence block table like an OS page table, blocks allocated
  only when needed and returned as soon as a sequence ends.
* same page, section 2.3: sequences forked from one prompt share its blocks;
  a block's reference count is the number of sequences that map it, and a
  sequence about to modify a block whose count is above one first copies it
  (copy-on-write) so the other sharers keep their data.
* same page, section 六 (decode loop): after writing a token into its block,
  check whether the next token needs a new block.

No attention arithmetic lives here.
"""
from __future__ import annotations

from collections import deque
from dataclasses import dataclass, field
from typing import Iterable, List, Optional, Tuple

import numpy as np


class OutOfBlocks(RuntimeError):
    """The free list is empty."""


@dataclass
class SeqBlocks:
    """One sequence: its physical blocks in logical order and its token count."""

    blocks: List[int] = field(default_factory=list)
    length: int = 0


class BlockManager:
    """Free list + reference counts over ``num_blocks`` physical blocks.

    The free list starts in the order given by ``rng.permutation`` (a seeded
    shuffle), so consecutive logical blocks land far apart in the pool.
    Block ids in ``reserved`` are never handed out.
    """

    def __init__(self, num_blocks: int, block_size: int = 16,
                 rng: Optional[np.random.Generator] = None, reserved: Iterable[int] = ()):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        reserved = set(int(b) for b in reserved)
        order = rng.permutation(self.num_blocks) if rng is not None else np.arange(self.num_blocks)
        self.free: deque = deque(int(b) for b in order if int(b) not in reserved)
        self.refcount = np.zeros(self.num_blocks, dtype=np.int32)
        self.copy_pairs: List[Tuple[int, int]] = []
        self.released: List[int] = []

    # -- raw block operations ------------------------------------------------
    def allocate(self) -> int:
        if not self.free:
            raise OutOfBlocks("no free KV block left")
        b = self.free.popleft()
        self.refcount[b] = 1
        return b

    def release(self, b: int) -> None:
        if self.refcount[b] <= 0:
            raise ValueError(f"block {b} released more often than referenced")
        self.refcount[b] -= 1
        if self.refcount[b] == 0:
            self.free.append(int(b))
            self.released.append(int(b))

    @property
    def num_free(self) -> int:
        return len(self.free)

    # -- sequence operations -------------------------------------------------
    def new_sequence(self) -> SeqBlocks:
        return SeqBlocks()

    def fork(self, parent: SeqBlocks) -> SeqBlocks:
        """A new sequence sharing every block of ``parent`` (refcounts + 1)."""
        for b in parent.blocks:
            self.refcount[b] += 1
        return SeqBlocks(blocks=list(parent.blocks), length=parent.length)

    def append_slot(self, seq: SeqBlocks) -> int:
        """Reserve the slot of the next token of ``seq`` and return it.

        A token at a block boundary gets a freshly allocated block.  A token
        going into a block with refcount > 1 triggers copy-on-write: a new
        block is allocated, the pair (shared, new) is queued on
        ``copy_pairs`` and the sequence's table now names the new block.
        """
        pos = seq.length
        if pos % self.block_size == 0:
            seq.blocks.append(self.allocate())
        elif self.refcount[seq.blocks[-1]] > 1:
            self.copy_last_block(seq)
        seq.length = pos + 1
        return seq.blocks[pos // self.block_size] * self.block_size + pos % self.block_size

    def copy_last_block(self, seq: SeqBlocks) -> int:
        """Give ``seq`` a private copy of its last block, whatever its refcount.

        Queues the (old, new) pair on ``copy_pairs`` and drops one reference
        to the old block; returns the new block id.
        """
        last = seq.blocks[-1]
        new = self.allocate()
        self.copy_pairs.append((last, new))
        self.release(last)
        seq.blocks[-1] = new
        return new

    def free_sequence(self, seq: SeqBlocks) -> None:
        for b in seq.blocks:
            self.release(b)
        seq.blocks = []
        seq.length = 0

    def take_copy_pairs(self) -> np.ndarray:
        pairs = np.asarray(self.copy_pairs, dtype=np.int64).reshape(-1, 2)
        self.copy_pairs = []
        return pairs

    def take_released(self) -> np.ndarray:
        r = np.asarray(self.released, dtype=np.int64)
        self.released = []
        return r


def block_tables(seqs: List[SeqBlocks], max_blocks_per_seq: int, pad_block: int) -> np.ndarray:
    """int32 ``[len(seqs), max_blocks_per_seq]``; unused entries name ``pad_block``."""
    bt = np.full((len(seqs), max_blocks_per_seq), pad_block, dtype=np.int32)
    for i, s in enumerate(seqs):
        if len(s.blocks) > max_blocks_per_seq:
            raise ValueError("sequence has more blocks than max_blocks_per_seq")
        bt[i, :len(s.blocks)] = s.blocks
    return bt


def validate_block_mapping(block_mapping: np.ndarray, num_blocks: int) -> None:
    """Host check for ``pa_copy_blocks`` pairs: ids in range, destinations
    distinct and never also a source (pairs are copied concurrently)."""
    bm = np.asarray(block_mapping, dtype=np.int64).reshape(-1, 2)
    if bm.size == 0:
        return
    if bm.min() < 0 or bm.max() >= num_blocks:
        raise ValueError("block id out of range")
    dst = bm[:, 1]
    if len(np.unique(dst)) != len(dst):
        raise ValueError("duplicate destination block")
    if np.intersect1d(dst, bm[:, 0]).size:
        raise ValueError("a destination block is also a source")


def validate_slot_mapping(slot_mapping: np.ndarray, num_blocks: int, block_size: int) -> None:
    """Host check for ``pa_reshape_and_cache`` slots: in range and distinct."""
    sm = np.asarray(slot_mapping, dtype=np.int64)
    live = sm[sm >= 0]
    if live.size and live.max() >= num_blocks * block_size:
        raise ValueError("slot out of range")
    if len(np.unique(live)) != len(live):
        raise ValueError("duplicate slot")
