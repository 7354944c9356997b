"""Host-side block allocator: physical KV blocks, block tables, slot mapping.

The KV cache is a pool of fixed-size physical blocks (16 or 32 tokens).  A
sequence owns a block table -- the list of physical block IDs that hold its
logical positions 0..n-1 in order -- and receives a new block only when its
last one is full; a finished sequence returns its blocks to the pool
("vLLM serving internals", AI Engineering from Scratch, Phase 17 / 04,
"PagedAttention as a virtual memory system"; "Inference optimization",
Phase 10 / 12, "Paged attention").

Blocks can be shared: ``fork`` gives a child every block of its parent and
bumps the reference counts, which is how rollouts of one prompt (GRPO) or
requests with one system prompt reference a prefix stored once.  Writing into a
block whose count is above one first moves the writer onto a fresh private
block and records the (source, destination) pair in ``pending_copies``; the
caller copies those rows before the append ("How vLLM gets real throughput on
H100s", deniz.in, "PagedAttention borrows from operating systems": the copy
happens only where the completions start to diverge).

The allocator only produces integer metadata (``block_table``,
``context_lens``, ``append_slots``); it never touches KV data.
"""
from __future__ import annotations

from collections import deque

import numpy as np


class OutOfBlocks(RuntimeError):
    """The pool has no free block left."""


class BlockAllocator:
    def __init__(self, num_blocks: int, block_size: int, seed: int | None = None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        order = np.arange(self.num_blocks, dtype=np.int64)
        if seed is not None:
            order = np.random.Generator(np.random.PCG64(seed)).permutation(self.num_blocks)
        self._free: deque[int] = deque(int(b) for b in order)
        self._ref = np.zeros(self.num_blocks, dtype=np.int64)
        self._tables: dict[int, list[int]] = {}
        self._lens: dict[int, int] = {}
        self.pending_copies: list[tuple[int, int]] = []

    # ---- pool -------------------------------------------------------------
    @property
    def num_free(self) -> int:
        return len(self._free)

    def refcount(self, block: int) -> int:
        return int(self._ref[block])

    def _take(self) -> int:
        if not self._free:
            raise OutOfBlocks(f"all {self.num_blocks} blocks are in use")
        b = self._free.popleft()
        self._ref[b] = 1
        return b

    def _release(self, b: int) -> None:
        self._ref[b] -= 1
        if self._ref[b] == 0:
            self._free.append(b)
        elif self._ref[b] < 0:  # pragma: no cover - internal invariant
            raise AssertionError(f"block {b} released twice")

    def blocks_needed(self, num_tokens: int) -> int:
        """ceil(num_tokens / block_size): blocks that hold num_tokens positions."""
        return -(-int(num_tokens) // self.block_size)

    # ---- sequences --------------------------------------------------------
    def add_sequence(self, seq_id: int, num_tokens: int = 0) -> None:
        """Register a sequence whose first ``num_tokens`` positions are stored."""
        if seq_id in self._tables:
            raise KeyError(f"sequence {seq_id} already exists")
        self._tables[seq_id] = []
        self._lens[seq_id] = 0
        if num_tokens:
            self.append_slots(seq_id, num_tokens)

    def fork(self, parent: int, child: int) -> None:
        """``child`` starts as a copy of ``parent`` that shares all its blocks."""
        if child in self._tables:
            raise KeyError(f"sequence {child} already exists")
        table = list(self._tables[parent])
        for b in table:
            self._ref[b] += 1
        self._tables[child] = table
        self._lens[child] = self._lens[parent]

    def free(self, seq_id: int) -> None:
        """Return the sequence's blocks to the pool (shared ones when unreferenced)."""
        for b in self._tables.pop(seq_id):
            self._release(b)
        del self._lens[seq_id]

    def length(self, seq_id: int) -> int:
        return self._lens[seq_id]

    def table(self, seq_id: int) -> list[int]:
        return list(self._tables[seq_id])

    def slot(self, seq_id: int, pos: int) -> int:
        """Slot of logical position ``pos``: block_id * block_size + pos % block_size."""
        table = self._tables[seq_id]
        return table[pos // self.block_size] * self.block_size + pos % self.block_size

    def append_slots(self, seq_id: int, n: int) -> np.ndarray:
        """Reserve the next ``n`` positions of ``seq_id`` and return their slots.

        A new block is taken whenever a position starts one.  If the block that
        receives a write is shared, the sequence first switches to a private
        copy of it (copy-on-write) and the copy is queued in ``pending_copies``.
        """
        table = self._tables[seq_id]
        start = self._lens[seq_id]
        out = np.empty(int(n), dtype=np.int32)
        bs = self.block_size
        for i in range(int(n)):
            pos = start + i
            lb = pos // bs
            if lb == len(table):
                table.append(self._take())
            elif self._ref[table[lb]] > 1:
                fresh = self._take()
                self.pending_copies.append((table[lb], fresh))
                self._release(table[lb])
                table[lb] = fresh
            out[i] = table[lb] * bs + pos % bs
        self._lens[seq_id] = start + int(n)
        return out

    # ---- batch metadata -----------------------------------------------------
    def block_table(self, seq_ids, max_blocks: int | None = None) -> np.ndarray:
        """int32 [len(seq_ids), max_blocks], unused entries -1."""
        rows = [self._tables[s] for s in seq_ids]
        width = max([len(r) for r in rows] + [1]) if max_blocks is None else int(max_blocks)
        bt = np.full((len(rows), width), -1, dtype=np.int32)
        for i, r in enumerate(rows):
            if len(r) > width:
                raise ValueError(f"sequence {seq_ids[i]} needs {len(r)} blocks > {width}")
            bt[i, :len(r)] = r
        return bt

    def context_lens(self, seq_ids) -> np.ndarray:
        return np.array([self._lens[s] for s in seq_ids], dtype=np.int32)

    # ---- statistics -------------------------------------------------------
    def used_blocks(self) -> int:
        return self.num_blocks - len(self._free)

    def internal_waste(self) -> float:
        """Fraction of the slots in allocated blocks that hold no token.

        Shared blocks count once, with the tokens of their longest user.
        """
        filled = np.zeros(self.num_blocks, dtype=np.int64)
        bs = self.block_size
        for sid, table in self._tables.items():
            n = self._lens[sid]
            for lb, b in enumerate(table):
                filled[b] = max(filled[b], min(bs, n - lb * bs))
        used = self.used_blocks()
        if used == 0:
            return 0.0
        return 1.0 - filled.sum() / (used * bs)


def static_reservation_waste(lengths, max_len: int) -> float:
    """Waste when every request reserves ``max_len`` contiguous slots up front."""
    lengths = np.asarray(lengths, dtype=np.float64)
    return 1.0 - lengths.sum() / (len(lengths) * float(max_len))
