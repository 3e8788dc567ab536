"""Host-side free-list allocator of fixed 16-token KV pages.

"KV Cache:推理慢的真正原因", section "工程优化手段 / PagedAttention": the cache
is cut into fixed blocks, a block table maps each sequence's logical blocks to
physical ones, and a finished request's blocks go straight back to the pool.
"KV缓存与Flash注意力", section "练习" (hard exercise): fixed 16-token blocks
with a free list.

The allocator only builds block tables (input structure for the decode step);
it does no attention arithmetic.
"""
from __future__ import annotations

from collections import deque

PAGE_TOKENS = 16


class OutOfPages(RuntimeError):
    pass


class BlockAllocator:
    """LIFO free list over physical pages 0..num_pages-1.

    Sequences own a list of physical pages (their block-table row).  Growing
    a sequence by tokens allocates pages only when it crosses a page edge.
    """

    def __init__(self, num_pages: int, order=None):
        if num_pages <= 0:
            raise ValueError("num_pages must be positive")
        self.num_pages = num_pages
        ids = list(range(num_pages)) if order is None else [int(i) for i in order]
        if sorted(ids) != list(range(num_pages)):
            raise ValueError("order must be a permutation of the pool")
        # pop() hands out ids[0] first
        self._free = deque(reversed(ids))
        self.tables: dict[int, list[int]] = {}
        self.lengths: dict[int, int] = {}
        self._refs: dict[int, int] = {}

    @property
    def free_pages(self) -> int:
        return len(self._free)

    @property
    def used_pages(self) -> int:
        return self.num_pages - len(self._free)

    def _take(self) -> int:
        if not self._free:
            raise OutOfPages("KV page pool exhausted")
        p = self._free.pop()
        self._refs[p] = 1
        return p

    def _drop(self, p: int) -> bool:
        self._refs[p] -= 1
        if self._refs[p] == 0:
            del self._refs[p]
            self._free.append(p)
            return True
        return False

    def add(self, seq_id: int, tokens: int = 0) -> list[int]:
        if seq_id in self.tables:
            raise KeyError(f"sequence {seq_id} already present")
        self.tables[seq_id] = []
        self.lengths[seq_id] = 0
        try:
            self.grow(seq_id, tokens)
        except OutOfPages:
            del self.tables[seq_id]
            del self.lengths[seq_id]
            raise
        return self.tables[seq_id]

    def grow(self, seq_id: int, tokens: int) -> list[int]:
        """Extend seq_id by `tokens`; returns the pages newly allocated."""
        if tokens < 0:
            raise ValueError("tokens must be >= 0")
        new_len = self.lengths[seq_id] + tokens
        need = (new_len + PAGE_TOKENS - 1) // PAGE_TOKENS
        table = self.tables[seq_id]
        fresh = []
        try:
            while len(table) < need:
                p = self._take()
                table.append(p)
                fresh.append(p)
        except OutOfPages:
            for p in reversed(fresh):
                table.pop()
                self._drop(p)
            raise
        self.lengths[seq_id] = new_len
        return fresh

    def fork(self, parent: int, child: int, shared_tokens: int) -> list[int]:
        """New sequence `child` sharing the parent's first shared_tokens tokens.

        shared_tokens must be a whole number of pages, so later appends of
        either sequence never write into a shared page.
        """
        if shared_tokens % PAGE_TOKENS:
            raise ValueError("shared prefix must be page aligned")
        n = shared_tokens // PAGE_TOKENS
        if n > len(self.tables[parent]):
            raise ValueError("parent is shorter than the shared prefix")
        if child in self.tables:
            raise KeyError(f"sequence {child} already present")
        self.tables[child] = list(self.tables[parent][:n])
        self.lengths[child] = shared_tokens
        for p in self.tables[child]:
            self._refs[p] += 1
        return self.tables[child]

    def release(self, seq_id: int) -> int:
        """Finish seq_id; returns how many pages went back to the free list.

        A page shared with another live sequence stays allocated until its
        last holder is released."""
        table = self.tables.pop(seq_id)
        self.lengths.pop(seq_id)
        return sum(1 for p in reversed(table) if self._drop(p))

    def block_table_row(self, seq_id: int, width: int, fill: int = -1) -> list[int]:
        row = list(self.tables[seq_id])
        if len(row) > width:
            raise ValueError("block table row wider than width")
        return row + [fill] * (width - len(row))
