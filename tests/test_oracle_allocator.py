"""Pins for the oracle block manager.

The pages fix the mechanism (fixed-size blocks, block table, on-demand
allocation, refcounts + copy-on-write; vLLM launch blog, "PagedAttention"
section, CSDN discovery note item 2) but print no worked example, so the
oracle is pinned by:
  * a hand-worked fork / copy-on-write example (tests/golden/fork_cow_example.json);
  * invariants checked after every request on random request sequences;
  * an isolation model: each sequence reads back exactly its own logical
    tokens through its slots, whatever the sharing, which a wrong
    copy-on-write rule breaks;
  * brute force over every short request sequence on a 4-block pool;
  * the "only the last block wastes" property (agientry.com overview and
    the launch blog: waste is confined to a sequence's last block).
"""

import itertools
import json
import os
import random

import pytest

from oracle.allocator import AllocatorError, BlockAllocator, OutOfBlocks

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_hand_worked_fork_example():
    g = _load("fork_cow_example.json")
    a = BlockAllocator(g["num_blocks"], g["block_size"], g["free_order"])
    for st in g["steps"]:
        op = st["op"]
        if op == "add":
            a.add(st["seq"])
        elif op == "fork":
            a.fork(st["parent"], st["child"])
        elif op == "free":
            a.free(st["seq"])
        elif op == "append":
            if st.get("error") == "out_of_blocks":
                before = (a.num_free(), [a.refcount(b) for b in range(g["num_blocks"])],
                          {s: a.block_table(s) for s in a.sequences()})
                with pytest.raises(OutOfBlocks):
                    a.append(st["seq"], st["n"])
                after = (a.num_free(), [a.refcount(b) for b in range(g["num_blocks"])],
                         {s: a.block_table(s) for s in a.sequences()})
                assert before == after
            else:
                slots, cow = a.append(st["seq"], st["n"])
                assert slots == st["slots"]
                assert [list(p) for p in cow] == st["cow"]
        a.check_invariants()
    fin = g["final"]
    assert {str(s): a.block_table(s) for s in a.sequences()} == fin["tables"]
    assert {str(s): a.length(s) for s in a.sequences()} == fin["lengths"]
    assert [a.refcount(b) for b in range(g["num_blocks"])] == fin["refcounts"]
    assert a.num_free() == fin["num_free"]
    assert a.waste_slots() == fin["waste_slots"]
    # the next blocks handed out follow the free stack
    a.add(99)
    slots, _ = a.append(99, 2 * g["block_size"])
    assert [s // g["block_size"] for s in slots[:: g["block_size"]]] == fin["next_free"]


class IsolationModel:
    """Logical model: every appended token gets a unique id; a fork copies the
    parent's list.  A physical array of token ids is written through the
    allocator's slots (after applying its copy-on-write copies); each live
    sequence must read back its own list."""

    def __init__(self, alloc: BlockAllocator):
        self.a = alloc
        self.logical = {}
        self.phys = [None] * (alloc.num_blocks * alloc.block_size)
        self.next_id = 0

    def add(self, s):
        self.a.add(s)
        self.logical[s] = []

    def fork(self, p, c):
        self.a.fork(p, c)
        self.logical[c] = list(self.logical[p])

    def free(self, s):
        self.a.free(s)
        del self.logical[s]

    def append(self, s, n):
        slots, cow = self.a.append(s, n)
        bs = self.a.block_size
        for src, dst in cow:
            self.phys[dst * bs:(dst + 1) * bs] = self.phys[src * bs:(src + 1) * bs]
        for sl in slots:
            self.phys[sl] = self.next_id
            self.logical[s].append(self.next_id)
            self.next_id += 1
        return slots, cow

    def check(self):
        self.a.check_invariants()
        for s, toks in self.logical.items():
            got = [self.phys[self.a.slot(s, t)] for t in range(self.a.length(s))]
            assert got == toks, f"sequence {s} does not read back its own tokens"


def _random_session(seed, num_blocks=24, bs=4, steps=300):
    rnd = random.Random(seed)
    order = list(range(num_blocks))
    rnd.shuffle(order)
    m = IsolationModel(BlockAllocator(num_blocks, bs, order))
    next_seq = 0
    for _ in range(steps):
        live = list(m.logical)
        r = rnd.random()
        try:
            if r < 0.15 or not live:
                m.add(next_seq)
                next_seq += 1
            elif r < 0.30:
                m.fork(rnd.choice(live), next_seq)
                next_seq += 1
            elif r < 0.42:
                m.free(rnd.choice(live))
            else:
                m.append(rnd.choice(live), rnd.choice([1, 1, 2, 3, bs - 1, bs, bs + 1, 2 * bs + 3]))
        except OutOfBlocks:
            pass
        m.check()
    return m


@pytest.mark.parametrize("seed", range(12))
def test_random_sessions_keep_invariants_and_isolation(seed):
    _random_session(seed)


def test_out_of_blocks_leaves_state_unchanged():
    a = BlockAllocator(3, 4, [2, 0, 1])
    a.add(1)
    a.append(1, 6)  # blocks 2, 0
    a.fork(1, 2)
    snap = (a.num_free(), [a.refcount(b) for b in range(3)], a.block_table(1), a.block_table(2))
    with pytest.raises(OutOfBlocks):
        a.append(2, 7)  # copy-on-write (1) + fresh blocks at positions 8 and 12 (2) = 3 > 1 free
    assert snap == (a.num_free(), [a.refcount(b) for b in range(3)], a.block_table(1), a.block_table(2))
    a.append(2, 2)  # copy-on-write of block 0 into block 1 only
    assert a.block_table(2) == [2, 1] and a.refcount(0) == 1 and a.num_free() == 0


def test_bad_requests():
    a = BlockAllocator(4, 4)
    a.add(0)
    with pytest.raises(AllocatorError):
        a.add(0)
    with pytest.raises(AllocatorError):
        a.append(7, 1)
    with pytest.raises(AllocatorError):
        a.fork(7, 8)
    with pytest.raises(AllocatorError):
        a.fork(0, 0)
    with pytest.raises(AllocatorError):
        a.free(5)
    with pytest.raises(AllocatorError):
        BlockAllocator(3, 4, [0, 1, 1])


def test_only_last_block_wastes():
    """Unshared sequences waste at most bs-1 slots each, all in the last block."""
    rnd = random.Random(5)
    bs = 16
    a = BlockAllocator(4096, bs, list(range(4096)))
    lens = [rnd.randint(1, 700) for _ in range(40)]
    for s, n in enumerate(lens):
        a.add(s)
        a.append(s, n)
    assert a.waste_slots() == sum((-n) % bs for n in lens)
    assert all((-n) % bs <= bs - 1 for n in lens)
    # every block but the last is full
    for s, n in enumerate(lens):
        assert len(a.block_table(s)) == -(-n // bs)


def _brute_force_ops(num_seqs_max=3):
    """All request sequences of length <= 4 over a small alphabet."""
    alphabet = []
    for s in range(num_seqs_max):
        alphabet += [("append", s, 1), ("append", s, 3), ("append", s, 5), ("free", s)]
        for c in range(num_seqs_max):
            if c != s:
                alphabet.append(("fork", s, c))
    return alphabet


def test_brute_force_small_pool():
    bs, nb = 4, 4
    alphabet = _brute_force_ops()
    n_checked = 0
    for length in range(1, 5):
        for seq in itertools.product(alphabet, repeat=length):
            m = IsolationModel(BlockAllocator(nb, bs, [3, 1, 0, 2]))
            m.add(0)
            for op in seq:
                try:
                    if op[0] == "append" and op[1] in m.logical:
                        before = (m.a.num_free(), [m.a.refcount(b) for b in range(nb)])
                        try:
                            m.append(op[1], op[2])
                        except OutOfBlocks:
                            assert before == (m.a.num_free(), [m.a.refcount(b) for b in range(nb)])
                    elif op[0] == "free" and op[1] in m.logical:
                        m.free(op[1])
                    elif op[0] == "fork" and op[1] in m.logical and op[2] not in m.logical:
                        m.fork(op[1], op[2])
                except AllocatorError:
                    raise
                m.check()
                n_checked += 1
    assert n_checked > 10000


class _MutantNoCow(BlockAllocator):
    """Planted mistake: writes into a shared partly filled block in place."""

    def append(self, seq, n):
        bs = self.block_size
        table = self._table[seq]
        slots = []
        for _ in range(n):
            pos = self._len[seq]
            if pos % bs == 0:
                b = self._free.pop()
                self._ref[b] = 1
                table.append(b)
            slots.append(table[pos // bs] * bs + pos % bs)
            self._len[seq] = pos + 1
        return slots, []


class _MutantForkNoRef(BlockAllocator):
    """Planted mistake: fork forgets to take references."""

    def fork(self, parent, child):
        self._table[child] = list(self._table[parent])
        self._len[child] = self._len[parent]


@pytest.mark.parametrize("mutant", [_MutantNoCow, _MutantForkNoRef])
def test_pins_catch_planted_mistakes(mutant):
    a = mutant(24, 4, list(range(24)))
    m = IsolationModel(a)
    failed = False
    try:
        m.add(0)
        m.append(0, 5)
        m.fork(0, 1)
        m.append(1, 2)
        m.append(0, 2)
        m.check()
        m.free(0)
        m.check()
    except AssertionError:
        failed = True
    assert failed
