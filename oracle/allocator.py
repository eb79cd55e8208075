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

Prefix caching (gitcode repo walkthrough, section 2.2: requests reuse the
already computed KV of an identical prefix such as a system prompt;
agientry.com overview, opening section: blocks can be shared across requests)
— the pages give the effect, not the mechanism; the reading taken here:

* sequences created with ``add_prefix`` and extended with ``append_tokens``
  carry their token ids; when such a block becomes full it is registered
  under the key (parent block, its token ids), the parent being the
  sequence's previous block (-1 for the first).  A block is registered only
  if its parent is registered (or it is a first block) and no block holds the
  key yet, so a key match implies the whole prefix matches, exactly.
* ``add_prefix`` follows the longest chain of registered keys along the
  prompt, over at most (n - 1) // bs full blocks so that one token is left to
  compute, and starts the sequence on those blocks (one more reference each).
* a registered block whose count drops to 0 is not freed but becomes
  evictable, kept in least-recently-freed order; blocks are taken from the
  free stack first, then by evicting the least recently freed evictable
  block.  Evicting (or otherwise unregistering) a block unregisters its
  registered children in increasing block order, depth first; an evictable
  child that loses its key goes onto the free stack.

Swapping (agientry.com overview, opening section: blocks can be swapped out)
— the reading taken here: a second pool of host blocks with its own LIFO free
stack.  ``swap_out`` gives each of a sequence's blocks, in table order, a
host block (all or nothing), reports (device, host) pairs for the copy, then
releases the device blocks as ``free`` would (a shared block is copied and
keeps its other holders).  ``swap_in`` takes device blocks for the host blocks
in order (all or nothing), reports (host, device) pairs, returns the host
blocks to their free stack in order, and re-registers the sequence's full
blocks for prefix reuse when its token ids are known.  A swapped-out sequence
can only be swapped in or freed.
"""

from __future__ import annotations

from collections import OrderedDict
from typing import Dict, List, Optional, Sequence, Set, Tuple


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
        # prefix caching
        self._tokens: Dict[int, Optional[List[int]]] = {}  # None: token ids unknown
        self._cache: Dict[Tuple[int, Tuple[int, ...]], int] = {}
        self._key_of: Dict[int, Tuple[int, Tuple[int, ...]]] = {}
        self._children: Dict[int, Set[int]] = {}
        self._evictable: "OrderedDict[int, None]" = OrderedDict()
        # swapping
        self.num_host_blocks = 0
        self._host_free: List[int] = []
        self._swapped: Dict[int, List[int]] = {}

    # -- queries ---------------------------------------------------------
    def num_free(self) -> int:
        """Blocks available to allocation: free plus evictable."""
        return len(self._free) + len(self._evictable)

    def num_cached(self) -> int:
        return len(self._cache)

    def num_evictable(self) -> int:
        return len(self._evictable)

    def is_cached(self, block: int) -> bool:
        return block in self._key_of

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

    def num_host_free(self) -> int:
        return len(self._host_free)

    def is_swapped(self, seq: int) -> bool:
        return seq in self._swapped

    def host_table(self, seq: int) -> List[int]:
        return list(self._swapped[seq])

    # -- requests --------------------------------------------------------
    def set_host_pool(self, num_host_blocks: int, host_free_order: Optional[Sequence[int]] = None) -> None:
        if self._swapped:
            raise AllocatorError("sequences are swapped out")
        order = list(range(num_host_blocks)) if host_free_order is None else [int(b) for b in host_free_order]
        if sorted(order) != list(range(num_host_blocks)):
            raise AllocatorError("host_free_order must be a permutation")
        self.num_host_blocks = num_host_blocks
        self._host_free = list(reversed(order))

    def _check_resident(self, seq: int) -> None:
        if seq not in self._table:
            raise AllocatorError(f"unknown sequence {seq}")
        if seq in self._swapped:
            raise AllocatorError(f"sequence {seq} is swapped out")

    def swap_out(self, seq: int) -> List[Tuple[int, int]]:
        self._check_resident(seq)
        table = self._table[seq]
        if len(table) > len(self._host_free):
            raise OutOfBlocks(f"sequence {seq}: {len(table)} blocks, {len(self._host_free)} host blocks free")
        pairs = []
        host = []
        for b in table:
            h = self._host_free.pop()
            pairs.append((b, h))
            host.append(h)
        for b in table:
            self._release(b)
        self._table[seq] = []
        self._swapped[seq] = host
        return pairs

    def swap_in(self, seq: int) -> List[Tuple[int, int]]:
        if seq not in self._swapped:
            raise AllocatorError(f"sequence {seq} is not swapped out")
        host = self._swapped[seq]
        if len(host) > self.num_free():
            raise OutOfBlocks(f"sequence {seq}: {len(host)} blocks, {self.num_free()} free")
        pairs = []
        table = []
        for h in host:
            b = self._take_block()
            self._ref[b] = 1
            table.append(b)
            pairs.append((h, b))
        for h in host:
            self._host_free.append(h)
        del self._swapped[seq]
        self._table[seq] = table
        toks = self._tokens.get(seq)
        if toks is not None:
            bs = self.block_size
            for j in range(self._len[seq] // bs):
                self._register(table[j], table[j - 1] if j else -1, tuple(toks[j * bs:(j + 1) * bs]))
        return pairs

    def add(self, seq: int) -> None:
        if seq in self._table:
            raise AllocatorError(f"sequence {seq} exists")
        self._table[seq] = []
        self._len[seq] = 0
        self._tokens[seq] = []

    # -- prefix-cache primitives ------------------------------------------
    def _take_block(self) -> int:
        if self._free:
            return self._free.pop()
        b, _ = self._evictable.popitem(last=False)
        self._unregister(b)
        return b

    def _unregister(self, b: int) -> None:
        key = self._key_of.pop(b)
        del self._cache[key]
        parent = key[0]
        if parent >= 0 and parent in self._children:
            self._children[parent].discard(b)
        for c in sorted(self._children.pop(b, set())):
            self._unregister_subtree(c)

    def _unregister_subtree(self, c: int) -> None:
        self._unregister(c)
        if c in self._evictable:
            del self._evictable[c]
            self._free.append(c)

    def _register(self, b: int, parent: int, toks: Tuple[int, ...]) -> None:
        if parent >= 0 and parent not in self._key_of:
            return
        key = (parent, toks)
        if key in self._cache or b in self._key_of:
            return
        self._cache[key] = b
        self._key_of[b] = key
        if parent >= 0:
            self._children.setdefault(parent, set()).add(b)

    def _release(self, b: int) -> None:
        self._ref[b] -= 1
        if self._ref[b] == 0:
            if b in self._key_of:
                self._evictable[b] = None
            else:
                self._free.append(b)

    def add_prefix(self, seq: int, tokens: Sequence[int]) -> int:
        """Add a sequence whose prompt is ``tokens``; reuse the longest chain
        of registered full blocks (leaving at least one token).  Returns the
        number of prompt tokens already in the cache (a multiple of bs)."""
        if seq in self._table:
            raise AllocatorError(f"sequence {seq} exists")
        bs = self.block_size
        tokens = [int(t) for t in tokens]
        hits: List[int] = []
        parent = -1
        for k in range(max(0, (len(tokens) - 1) // bs)):
            b = self._cache.get((parent, tuple(tokens[k * bs:(k + 1) * bs])))
            if b is None:
                break
            hits.append(b)
            parent = b
        for b in hits:
            if self._ref[b] == 0:
                del self._evictable[b]
            self._ref[b] += 1
        self._table[seq] = list(hits)
        self._len[seq] = len(hits) * bs
        self._tokens[seq] = tokens[:len(hits) * bs]
        return len(hits) * bs

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
        self._check_resident(seq)
        if n < 0:
            raise AllocatorError("negative token count")
        return self._append(seq, n, None)

    def append_tokens(self, seq: int, tokens: Sequence[int]) -> Tuple[List[int], List[Tuple[int, int]]]:
        """Append tokens with known ids (the sequence's ids so far must be
        known); blocks that become full are registered for prefix reuse."""
        self._check_resident(seq)
        if self._tokens.get(seq) is None:
            raise AllocatorError(f"sequence {seq} has tokens of unknown id")
        return self._append(seq, len(tokens), [int(t) for t in tokens])

    def _append(self, seq: int, n: int, ids: Optional[List[int]]):
        if self._blocks_needed(seq, n) > self.num_free():
            raise OutOfBlocks(f"sequence {seq}: {n} tokens need more than {self.num_free()} free blocks")
        bs = self.block_size
        table = self._table[seq]
        if ids is None:
            self._tokens[seq] = None
        toks = self._tokens[seq]
        slots: List[int] = []
        cow: List[Tuple[int, int]] = []
        for k in range(n):
            pos = self._len[seq]
            if pos % bs == 0:
                b = self._take_block()
                self._ref[b] = 1
                table.append(b)
            else:
                last = table[-1]
                if self._ref[last] > 1:
                    b = self._take_block()
                    self._ref[b] = 1
                    self._ref[last] -= 1
                    table[-1] = b
                    cow.append((last, b))
            slots.append(table[pos // bs] * bs + pos % bs)
            self._len[seq] = pos + 1
            if toks is not None:
                toks.append(ids[k])
                if (pos + 1) % bs == 0:
                    j = pos // bs
                    self._register(table[j], table[j - 1] if j else -1, tuple(toks[j * bs:(j + 1) * bs]))
        return slots, cow

    def fork(self, parent: int, child: int) -> None:
        """The child starts as a copy of the parent's table; every block it
        names gains one reference."""
        self._check_resident(parent)
        if child in self._table:
            raise AllocatorError(f"sequence {child} exists")
        self._table[child] = list(self._table[parent])
        self._len[child] = self._len[parent]
        t = self._tokens.get(parent)
        self._tokens[child] = None if t is None else list(t)
        for b in self._table[child]:
            self._ref[b] += 1

    def free(self, seq: int) -> None:
        if seq not in self._table:
            raise AllocatorError(f"unknown sequence {seq}")
        for b in self._table.pop(seq):
            self._release(b)
        for h in self._swapped.pop(seq, []):
            self._host_free.append(h)
        del self._len[seq]
        del self._tokens[seq]

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
            if seq in self._swapped:
                if table or len(self._swapped[seq]) != -(-self._len[seq] // bs):
                    raise AssertionError(f"swapped sequence {seq}: table and host blocks disagree")
                continue
            if len(table) != -(-self._len[seq] // bs):
                raise AssertionError(f"sequence {seq}: table length does not match its token count")
            for b in table:
                count[b] += 1
        if count != self._ref:
            raise AssertionError("reference counts differ from the number of tables naming each block")
        free = set(self._free)
        if len(free) != len(self._free):
            raise AssertionError("a block is on the free stack twice")
        evict = set(self._evictable)
        used = {b for b in range(self.num_blocks) if self._ref[b] > 0}
        if (free & used) or (free & evict) or (evict & used) or (free | used | evict) != set(range(self.num_blocks)):
            raise AssertionError("free, evictable and used blocks do not partition the pool")
        for key, b in self._cache.items():
            if self._key_of.get(b) != key:
                raise AssertionError("cache key and block disagree")
            if key[0] >= 0 and key[0] not in self._key_of:
                raise AssertionError("a registered block's parent is not registered")
        if not evict <= set(self._key_of):
            raise AssertionError("an evictable block is not registered")
        host_used = [h for hs in self._swapped.values() for h in hs]
        if len(set(host_used)) != len(host_used) or set(host_used) & set(self._host_free) or \
                len(host_used) + len(self._host_free) != self.num_host_blocks:
            raise AssertionError("host blocks are not partitioned")
