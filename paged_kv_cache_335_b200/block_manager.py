"""Host-side block manager: free pool, per-sequence block tables, reference
counts and copy-on-write decisions.

This is the allocator side of PagedAttention that the device kernels assume
(pages, by title and section):

* "PagedAttention：大模型推理性能优化的核心技术解析", § 核心工作机制与创新:
  fixed-size blocks mapped through a page table (1 页表式管理); a shared block
  is copied only when a sharer writes to it (2 写入时拷贝); blocks are taken on
  demand and returned to the global pool when a sequence ends (3 动态内存分配).
* "AI 推理系列（十六）：PagedAttention——…", § PagedAttention 如何把连续序列映射到
  离散显存块: the block table maps logical block j to a physical block; the
  per-step flowchart appends K/V into the current block and asks for a new
  physical block when the current one is full.
* "PagedAttention原理详解：GPU显存优化与模型路由技术", § PagedAttention的三大核心
  优势: beams / samples share prefix blocks through reference counts and copy
  on divergence.

The manager produces plain integer arrays (block tables, slot indices,
(src, dst) copy pairs) for the device calls ``pa_kv_append`` and
``pa_block_copy``; it does no attention arithmetic.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


class PoolExhausted(RuntimeError):
    """Raised when an allocation finds the free pool empty."""


@dataclass
class Sequence:
    """One logical sequence: its block table and how many token slots it holds."""
    table: list = field(default_factory=list)
    length: int = 0


class BlockManager:
    """Fixed pool of ``num_blocks`` blocks of ``block_size`` slots.

    ``order`` is the order in which free blocks are handed out; a random
    permutation scatters a sequence's blocks over the pool, which is what the
    paged layout must tolerate. ``reserved`` ids are never handed out.
    """

    def __init__(self, num_blocks: int, block_size: int, order=None, reserved=()):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        ids = list(range(num_blocks)) if order is None else [int(i) for i in order]
        if sorted(ids) != list(range(num_blocks)):
            raise ValueError("order must be a permutation of range(num_blocks)")
        reserved = {int(r) for r in reserved}
        # pop() takes from the end: reverse so that order[0] is handed out first.
        self._free = [i for i in reversed(ids) if i not in reserved]
        self.refcount = np.zeros(num_blocks, dtype=np.int64)
        self.copies: list = []  # (src, dst) pairs recorded by copy-on-write

    # -- pool ---------------------------------------------------------------
    @property
    def num_free(self) -> int:
        return len(self._free)

    def allocate(self) -> int:
        if not self._free:
            raise PoolExhausted(f"no free block left in a pool of {self.num_blocks}")
        b = self._free.pop()
        assert self.refcount[b] == 0
        self.refcount[b] = 1
        return b

    def _release(self, b: int) -> None:
        if self.refcount[b] <= 0:
            raise AssertionError(f"block {b} released with refcount {self.refcount[b]}")
        self.refcount[b] -= 1
        if self.refcount[b] == 0:
            self._free.append(b)

    # -- sequences ----------------------------------------------------------
    def new_sequence(self, length: int = 0) -> Sequence:
        """A sequence whose first ``length`` positions are already filled (prefill)."""
        seq = Sequence()
        for _ in range(length):
            self.append_slot(seq)
        return seq

    def fork(self, parent: Sequence) -> Sequence:
        """A child that shares every block of ``parent`` (refcount + 1 each)."""
        for b in parent.table:
            self.refcount[b] += 1
        return Sequence(table=list(parent.table), length=parent.length)

    def free(self, seq: Sequence) -> None:
        """Sequence finished: drop its references; unreferenced blocks return to the pool."""
        for b in seq.table:
            self._release(b)
        seq.table = []
        seq.length = 0

    def append_slot(self, seq: Sequence) -> int:
        """Reserve the slot of position ``seq.length`` and return its slot index.

        If the position opens a new block, a block is allocated. If it falls in
        a block that other sequences still reference, the block is first
        replaced by a private copy and the (src, dst) pair is recorded in
        ``self.copies`` for ``pa_block_copy``.
        """
        pos = seq.length
        j, off = divmod(pos, self.block_size)
        if j == len(seq.table):
            seq.table.append(self.allocate())
        else:
            b = seq.table[j]
            if self.refcount[b] > 1:
                nb = self.allocate()
                self.copies.append((b, nb))
                self.refcount[b] -= 1
                seq.table[j] = nb
        seq.length = pos + 1
        return seq.table[j] * self.block_size + off

    def take_copies(self) -> np.ndarray:
        """Copy pairs recorded since the last call, as int64 [P][2]."""
        pairs = np.asarray(self.copies, dtype=np.int64).reshape(-1, 2)
        self.copies = []
        return pairs

    # -- views --------------------------------------------------------------
    def tables_array(self, seqs, width: int, pad: int) -> np.ndarray:
        """Block tables as int32 [len(seqs)][width]; entries past a table's end = ``pad``."""
        out = np.full((len(seqs), width), pad, dtype=np.int32)
        for i, s in enumerate(seqs):
            if len(s.table) > width:
                raise ValueError("block table wider than the requested width")
            out[i, :len(s.table)] = s.table
        return out
