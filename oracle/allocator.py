"""Oracle block manager (test infrastructure; see the package header).

What the pages fix (vLLM launch blog, "PagedAttention" section, summarised on
the CSDN discovery note, item 2; agientry.com overview, opening section):

* the KV cache is cut into blocks of a fixed number of tokens;
* a per-sequence block table maps logical blocks to physical blocks that need
  not be contiguous;
* physical blocks are allocated on demand as tokens arrive, so only a
  sequence's last block can hold unused slots;
* parallel samples share the prompt's physical blocks through reference
  counts, and a write into a shared block first copies it (copy-on-write).

What the pages leave open, and the reading taken here:

* allocation order: a LIFO free stack.  The caller gives the initial order
  (``free_order[0]`` is handed out first); a freed block goes on top and is
  the next one handed out.  ``free`` releases a sequence's blocks in table
  order, so its last block ends on top.
* copy-on-write trigger: a token is written into the last block when that
  block is partly filled; if its reference count is above one, a fresh block
  is taken, the pair (old, new) is emitted for a whole-block copy, the old
  block's count drops by one, and the table points at the new block.  A full
  shared last block is never copied: the next token opens a fresh block.
* ``append`` is all-or-nothing: if the free stack cannot cover every block the
  call needs, it raises ``OutOfBlocks`` and changes nothing.
* slot of logical position t of a sequence: ``table[t // bs] * bs + t % bs``.
"""

from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple


class AllocatorError(ValueError):
    """Invalid request (unknown or duplicate sequence id, bad block id)."""


class OutOfBlocks(RuntimeError):
    """Not enough free blocks; the allocator state is unchanged."""


class BlockAllocator:
    def __init__(self, num_blocks: int, block_size: int, free_order: Optional[Sequence[int]] = None):
        if num_blocks <= 0 or block_size <= 0:
            raise AllocatorError("num_blocks and block_size must be positive")
        if free_order is None:
            free_order = list(range(num_blocks))
        free_order = [int(b) for b in free_order]
        if sorted(free_order) != list(range(num_blocks)):
            raise AllocatorError("free_order must be a permutation of 0..num_blocks-1")
        self.num_blocks = num_blocks
        self.block_size = block_size
        # top of the stack = end of the list
        self._free: List[int] = list(reversed(free_order))
        self._ref: List[int] = [0] * num_blocks
        self._table: Dict[int, List[int]] = {}
        self._len: Dict[int, int] = {}

    # -- queries ---------------------------------------------------------
    def num_free(self) -> int:
        return len(self._free)

    def refcount(self, block: int) -> int:
        return self._ref[block]

    def block_table(self, seq: int) -> List[int]:
        return list(self._table[seq])

    def length(self, seq: int) -> int:
        return self._len[seq]

    def sequences(self) -> List[int]:
        return list(self._table.keys())

    def slot(self, seq: int, pos: int) -> int:
        bs = self.block_size
        return self._table[seq][pos // bs] * bs + pos % bs

    # -- requests --------------------------------------------------------
    def add(self, seq: int) -> None:
        if seq in self._table:
            raise AllocatorError(f"sequence {seq} exists")
        self._table[seq] = []
        self._len[seq] = 0

    def _blocks_needed(self, seq: int, n: int) -> int:
        bs = self.block_size
        pos = self._len[seq]
        need = 0
        if n > 0 and pos % bs != 0 and self._ref[self._table[seq][-1]] > 1:
            need += 1  # copy-on-write of the shared, partly filled last block
        # a fresh block opens at every position that is a multiple of bs
        first = -(-pos // bs) * bs
        if first < pos + n:
            need += (pos + n - 1 - first) // bs + 1
        return need

    def append(self, seq: int, n: int) -> Tuple[List[int], List[Tuple[int, int]]]:
        """Append n tokens; return (slots of the new tokens, copy-on-write pairs)."""
        if seq not in self._table:
            raise AllocatorError(f"unknown sequence {seq}")
        if n < 0:
            raise AllocatorError("negative token count")
        if self._blocks_needed(seq, n) > len(self._free):
            raise OutOfBlocks(f"sequence {seq}: {n} tokens need more than {len(self._free)} free blocks")
        bs = self.block_size
        table = self._table[seq]
        slots: List[int] = []
        cow: List[Tuple[int, int]] = []
        for _ in range(n):
            pos = self._len[seq]
            if pos % bs == 0:
                b = self._free.pop()
                self._ref[b] = 1
                table.append(b)
            else:
                last = table[-1]
                if self._ref[last] > 1:
                    b = self._free.pop()
                    self._ref[b] = 1
                    self._ref[last] -= 1
                    table[-1] = b
                    cow.append((last, b))
            slots.append(table[pos // bs] * bs + pos % bs)
            self._len[seq] = pos + 1
        return slots, cow

    def fork(self, parent: int, child: int) -> None:
        """The child starts as a copy of the parent's table; every block it
        names gains one reference."""
        if parent not in self._table:
            raise AllocatorError(f"unknown sequence {parent}")
        if child in self._table:
            raise AllocatorError(f"sequence {child} exists")
        self._table[child] = list(self._table[parent])
        self._len[child] = self._len[parent]
        for b in self._table[child]:
            self._ref[b] += 1

    def free(self, seq: int) -> None:
        if seq not in self._table:
            raise AllocatorError(f"unknown sequence {seq}")
        for b in self._table.pop(seq):
            self._ref[b] -= 1
            if self._ref[b] == 0:
                self._free.append(b)
        del self._len[seq]

    # -- statistics and invariants ----------------------------------------
    def waste_slots(self) -> int:
        """Unused slots in blocks that are in use: for each used block, bs minus
        the largest number of its slots any sequence holding it has filled."""
        bs = self.block_size
        filled: Dict[int, int] = {}
        for seq, table in self._table.items():
            length = self._len[seq]
            for k, b in enumerate(table):
                f = min(bs, length - k * bs)
                filled[b] = max(filled.get(b, 0), f)
        return sum(bs - f for f in filled.values())

    def check_invariants(self) -> None:
        bs = self.block_size
        count = [0] * self.num_blocks
        for seq, table in self._table.items():
            if len(table) != -(-self._len[seq] // bs):
                raise AssertionError(f"sequence {seq}: table length does not match its token count")
            for b in table:
                count[b] += 1
        if count != self._ref:
            raise AssertionError("reference counts differ from the number of tables naming each block")
        free = set(self._free)
        if len(free) != len(self._free):
            raise AssertionError("a block is on the free stack twice")
        used = {b for b in range(self.num_blocks) if self._ref[b] > 0}
        if free & used or (free | used) != set(range(self.num_blocks)):
            raise AssertionError("free and used blocks do not partition the pool")
