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


# ---------------------------------------------------------------------------
# prefix caching
# ---------------------------------------------------------------------------

def run_prefix_example(alloc_factory, appendf, append_tokensf, add_prefixf, evictable_of, cached_of):
    g = _load("prefix_cache_example.json")
    a = alloc_factory(g["num_blocks"], g["block_size"], g["free_order"])
    for st in g["steps"]:
        op = st["op"]
        if op == "add":
            a.add(st["seq"])
        elif op == "free":
            a.free(st["seq"])
        elif op == "add_prefix":
            assert add_prefixf(a, st["seq"], st["tokens"]) == st["hit"], st
        elif op == "append_tokens":
            slots, cow = append_tokensf(a, st["seq"], st["tokens"])
            assert list(slots) == st["slots"] and [list(p) for p in cow] == st["cow"], st
        elif op == "append":
            slots, cow = appendf(a, st["seq"], st["n"])
            assert list(slots) == st["slots"] and [list(p) for p in cow] == st["cow"], st
        elif op == "check":
            assert a.num_free() == st["num_free"], st
            assert evictable_of(a) == st["evictable"], st
            assert cached_of(a) == st["cached"], st
    assert [a.refcount(b) for b in range(g["num_blocks"])] == g["final_refcounts"]
    return a


def test_prefix_cache_hand_worked_example():
    a = run_prefix_example(BlockAllocator, lambda a, s, n: a.append(s, n), lambda a, s, t: a.append_tokens(s, t),
                           lambda a, s, t: a.add_prefix(s, t), lambda a: list(a._evictable), lambda a: a.num_cached())
    a.check_invariants()


class PrefixIsolationModel(IsolationModel):
    """Context model with prefix reuse.  A token's K/V depends on every token
    before it, so the content of a slot is the whole token prefix of the
    sequence that wrote it, up to that token.  A sequence must read back its
    own prefixes at every position; a reused block must therefore have been
    written under exactly the same prefix, and a false prefix hit is caught."""

    def add_prefix(self, s, toks):
        hit = self.a.add_prefix(s, toks)
        self.logical[s] = list(toks[:hit])
        return hit

    def _write(self, s, slots, cow, ids):
        bs = self.a.block_size
        for src, dst in cow:
            self.phys[dst * bs:(dst + 1) * bs] = self.phys[src * bs:(src + 1) * bs]
        for sl, t in zip(slots, ids):
            self.logical[s].append(t)
            self.phys[sl] = tuple(self.logical[s])

    def append_tokens(self, s, toks):
        slots, cow = self.a.append_tokens(s, toks)
        self._write(s, slots, cow, list(toks))
        return slots, cow

    def append(self, s, n):
        slots, cow = self.a.append(s, n)
        ids = [-1 - self.next_id - k for k in range(n)]  # unknown tokens: ids no prompt uses
        self.next_id += n
        self._write(s, slots, cow, ids)
        return slots, cow

    def check(self):
        self.a.check_invariants()
        for s, toks in self.logical.items():
            got = [self.phys[self.a.slot(s, t)] for t in range(self.a.length(s))]
            assert got == [tuple(toks[:t + 1]) for t in range(len(toks))], f"sequence {s} reads a foreign prefix"


def _prefix_session(seed, num_blocks=30, bs=4, steps=400):
    rnd = random.Random(seed)
    order = list(range(num_blocks))
    rnd.shuffle(order)
    m = PrefixIsolationModel(BlockAllocator(num_blocks, bs, order))
    systems = [[rnd.randrange(3) for _ in range(rnd.choice([4, 8, 9, 12]))] for _ in range(3)]
    nxt = 0
    hits = 0
    for _ in range(steps):
        live = list(m.logical)
        r = rnd.random()
        try:
            if r < 0.25 or not live:
                prompt = rnd.choice(systems) + [rnd.randrange(3) for _ in range(rnd.randrange(0, 7))]
                if not prompt:
                    prompt = [0]
                hit = m.add_prefix(nxt, prompt)
                hits += hit > 0
                nxt += 1
                m.append_tokens(nxt - 1, prompt[hit:])
            elif r < 0.35:
                m.fork(rnd.choice(live), nxt)
                nxt += 1
            elif r < 0.55:
                m.free(rnd.choice(live))
            elif r < 0.85:
                s = rnd.choice(live)
                if m.a._tokens.get(s) is not None:
                    m.append_tokens(s, [rnd.randrange(3) for _ in range(rnd.choice([1, 2, 3, 5]))])
                else:
                    m.append(s, rnd.choice([1, 2, 5]))
            else:
                m.append(rnd.choice(live), rnd.choice([1, 3]))
        except OutOfBlocks:
            pass
        m.check()
    return hits


@pytest.mark.parametrize("seed", range(10))
def test_prefix_sessions_keep_invariants_and_isolation(seed):
    assert _prefix_session(seed) > 0


class _MutantPrefixIgnoresParent(BlockAllocator):
    """Planted mistake: matches a block by its own tokens only."""

    def add_prefix(self, seq, tokens):
        bs = self.block_size
        saved = dict(self._cache)
        self._cache = {(-1, k[1]): b for k, b in saved.items()} | saved
        try:
            hits = []
            for k in range(max(0, (len(tokens) - 1) // bs)):
                b = self._cache.get((-1, tuple(tokens[k * bs:(k + 1) * bs])))
                if b is None:
                    break
                hits.append(b)
        finally:
            self._cache = saved
        if seq in self._table:
            raise AllocatorError("exists")
        for b in hits:
            if self._ref[b] == 0:
                del self._evictable[b]
            self._ref[b] += 1
        self._table[seq] = hits
        self._len[seq] = len(hits) * bs
        self._tokens[seq] = list(tokens[:len(hits) * bs])
        return len(hits) * bs


def test_prefix_pins_catch_planted_mistake():
    m = PrefixIsolationModel(_MutantPrefixIgnoresParent(20, 4, list(range(20))))
    m.add_prefix(0, [1, 1, 1, 1, 2, 2, 2, 2, 3])
    m.append_tokens(0, [1, 1, 1, 1, 2, 2, 2, 2, 3])
    m.check()
    # the same four tokens as seq 0's second block, but at the start of a prompt
    hit = m.add_prefix(1, [2, 2, 2, 2, 9])
    assert hit == 4  # the mutant reuses a block written under another prefix
    with pytest.raises(AssertionError):
        m.check()


def test_forks_of_forks_share_and_copy():
    """Beam-search style: forks of forks share every full block and copy the
    shared partial one on their first write."""
    m = IsolationModel(BlockAllocator(40, 4, list(range(40))))
    m.add(0)
    m.append(0, 6)
    m.fork(0, 1)
    m.fork(1, 2)
    m.fork(2, 3)
    assert m.a.refcount(m.a.block_table(0)[1]) == 4
    for s in (3, 2, 1, 0):
        m.append(s, 1)
        m.check()
    assert len({m.a.block_table(s)[1] for s in range(4)}) == 4
    assert len({m.a.block_table(s)[0] for s in range(4)}) == 1


# ---------------------------------------------------------------------------
# swapping
# ---------------------------------------------------------------------------

class SwapModel(PrefixIsolationModel):
    """Adds a host pool: swap_out copies device blocks to host blocks by the
    reported pairs, swap_in copies them back; a swapped sequence must still
    read back its own prefixes through its host blocks."""

    def __init__(self, alloc, num_host):
        super().__init__(alloc)
        alloc.set_host_pool(num_host, list(range(num_host)))
        self.host = [None] * (num_host * alloc.block_size)

    def swap_out(self, s):
        bs = self.a.block_size
        pairs = self.a.swap_out(s)
        for b, h in pairs:
            self.host[h * bs:(h + 1) * bs] = self.phys[b * bs:(b + 1) * bs]
        return pairs

    def swap_in(self, s):
        bs = self.a.block_size
        pairs = self.a.swap_in(s)
        for h, b in pairs:
            self.phys[b * bs:(b + 1) * bs] = self.host[h * bs:(h + 1) * bs]
        return pairs

    def check(self):
        self.a.check_invariants()
        bs = self.a.block_size
        for s, toks in self.logical.items():
            want = [tuple(toks[:t + 1]) for t in range(len(toks))]
            if self.a.is_swapped(s):
                ht = self.a.host_table(s)
                got = [self.host[ht[t // bs] * bs + t % bs] for t in range(self.a.length(s))]
            else:
                got = [self.phys[self.a.slot(s, t)] for t in range(self.a.length(s))]
            assert got == want, f"sequence {s} reads a foreign prefix"


def _swap_session(seed, alloc_cls=BlockAllocator, num_blocks=24, num_host=20, bs=4, steps=500):
    rnd = random.Random(seed)
    order = list(range(num_blocks))
    rnd.shuffle(order)
    m = SwapModel(alloc_cls(num_blocks, bs, order), num_host)
    systems = [[rnd.randrange(3) for _ in range(rnd.choice([4, 8, 9]))] for _ in range(2)]
    nxt, swaps = 0, 0
    for _ in range(steps):
        live = list(m.logical)
        resident = [s for s in live if not m.a.is_swapped(s)]
        swapped = [s for s in live if m.a.is_swapped(s)]
        r = rnd.random()
        try:
            if r < 0.2 or not live:
                prompt = rnd.choice(systems) + [rnd.randrange(3) for _ in range(rnd.randrange(0, 6))]
                hit = m.add_prefix(nxt, prompt)
                nxt += 1
                m.append_tokens(nxt - 1, prompt[hit:])
            elif r < 0.3 and resident:
                m.fork(rnd.choice(resident), nxt)
                nxt += 1
            elif r < 0.45:
                m.free(rnd.choice(live))
            elif r < 0.6 and resident:
                m.swap_out(rnd.choice(resident))
                swaps += 1
            elif r < 0.75 and swapped:
                m.swap_in(rnd.choice(swapped))
            elif resident:
                s = rnd.choice(resident)
                if m.a._tokens.get(s) is not None:
                    m.append_tokens(s, [rnd.randrange(3) for _ in range(rnd.choice([1, 3, 5]))])
                else:
                    m.append(s, rnd.choice([1, 4]))
        except OutOfBlocks:
            pass
        m.check()
    return swaps


@pytest.mark.parametrize("seed", range(10))
def test_swap_sessions_keep_contents(seed):
    assert _swap_session(seed) > 0


def test_swapped_sequence_accepts_only_swap_in_or_free():
    a = BlockAllocator(8, 4, list(range(8)))
    a.set_host_pool(4)
    a.add(0)
    a.append(0, 6)
    a.swap_out(0)
    for fn, args in ((a.append, (0, 1)), (a.fork, (0, 1)), (a.swap_out, (0,)), (a.append_tokens, (0, [1]))):
        with pytest.raises(AllocatorError):
            fn(*args)
    a.free(0)
    assert a.num_host_free() == 4 and a.num_free() == 8
    a.check_invariants()


class _MutantSwapInReversed(BlockAllocator):
    """Planted mistake: pairs host blocks with device blocks in reverse order."""

    def swap_in(self, seq):
        pairs = super().swap_in(seq)
        hs = [h for h, _ in pairs]
        return list(zip(reversed(hs), [b for _, b in pairs]))


def test_swap_pins_catch_planted_mistake():
    with pytest.raises(AssertionError):
        for seed in range(10):
            _swap_session(seed, alloc_cls=_MutantSwapInReversed)
