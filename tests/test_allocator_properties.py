"""Property test of the host block allocator: random programs of add, fork,
append and free against a model of what each sequence holds.

A store maps slots to the token written there. Every append writes its token
to the slot the allocator returned, after doing the block copies the
allocator queued (copy-on-write). The invariants are the paging of "vLLM
serving internals" ("PagedAttention as a virtual memory system"): every live
position reads back its own token through the block table; a block's
reference count is the number of tables holding it; free blocks are the
unreferenced ones; a table has ceil(len / block_size) entries; and an
appended position always lands in a block that no other sequence holds.
"""
from __future__ import annotations

import numpy as np
from hypothesis import settings
from hypothesis import strategies as st
from hypothesis.stateful import RuleBasedStateMachine, invariant, precondition, rule

from paged_kv_cache_445_b200.allocator import BlockAllocator, OutOfBlocks

NUM_BLOCKS = 24


class PagedCache(RuleBasedStateMachine):
    def __init__(self):
        super().__init__()
        self.bs = 4
        self.a = BlockAllocator(NUM_BLOCKS, self.bs, seed=7)
        self.store: dict[int, int] = {}      # slot -> token
        self.content: dict[int, list[int]] = {}  # sequence -> its tokens
        self.next_id = 0
        self.next_token = 1

    def _apply_copies(self):
        for src, dst in self.a.pending_copies:
            for off in range(self.bs):
                if src * self.bs + off in self.store:
                    self.store[dst * self.bs + off] = self.store[src * self.bs + off]
        self.a.pending_copies.clear()

    def _append(self, s: int, n: int) -> None:
        try:
            slots = self.a.append_slots(s, n)
        except OutOfBlocks:
            # the pool ran dry part-way through: drop the sequence (every block in its
            # table, the ones just taken included, goes back to the pool)
            self._apply_copies()
            self.a.free(s)
            del self.content[s]
            return
        self._apply_copies()
        for slot in slots:
            owner = int(slot) // self.bs
            assert self.a.refcount(owner) == 1, "a write must land in a private block"
            self.store[int(slot)] = self.next_token
            self.content[s].append(self.next_token)
            self.next_token += 1

    @rule(n=st.integers(0, 9))
    def add(self, n):
        s = self.next_id
        self.next_id += 1
        self.a.add_sequence(s)
        self.content[s] = []
        self._append(s, n)

    @precondition(lambda self: self.content)
    @rule(data=st.data(), n=st.integers(1, 6))
    def append(self, data, n):
        s = data.draw(st.sampled_from(sorted(self.content)))
        self._append(s, n)

    @precondition(lambda self: self.content)
    @rule(data=st.data())
    def fork(self, data):
        parent = data.draw(st.sampled_from(sorted(self.content)))
        child = self.next_id
        self.next_id += 1
        self.a.fork(parent, child)
        self.content[child] = list(self.content[parent])

    @precondition(lambda self: self.content)
    @rule(data=st.data())
    def free(self, data):
        s = data.draw(st.sampled_from(sorted(self.content)))
        self.a.free(s)
        del self.content[s]

    @invariant()
    def every_position_reads_back_its_token(self):
        for s, toks in self.content.items():
            assert self.a.length(s) == len(toks)
            for pos, tok in enumerate(toks):
                assert self.store.get(self.a.slot(s, pos)) == tok

    @invariant()
    def refcounts_and_free_list_agree_with_the_tables(self):
        held = np.zeros(NUM_BLOCKS, dtype=np.int64)
        for s in self.content:
            table = self.a.table(s)
            assert len(table) == -(-self.a.length(s) // self.bs)
            for b in table:
                held[b] += 1
        for b in range(NUM_BLOCKS):
            assert self.a.refcount(b) == held[b]
        assert self.a.num_free == int(np.sum(held == 0))


PagedCache.TestCase.settings = settings(max_examples=60, stateful_step_count=40, deadline=None)
TestPagedCache = PagedCache.TestCase
