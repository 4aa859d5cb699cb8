"""The library's host-side block manager (pkv_bm_*), on CPU.

Pinned to the glossary's worked example, the allocation and copy-on-write
rules of the pages, conservation of blocks, and equivalence with the test
harness's independent Python allocator on random operation sequences.
"""
import json
import os

import numpy as np
import pytest

from paged_kv_cache_324_b200 import workload as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def BM():
    from paged_kv_cache_324_b200 import binding, build
    build.build()
    return binding.BlockManager


def test_worked_example(BM):
    g = json.load(open(os.path.join(GOLDEN, "ul_worked_example.json")))
    B, n = g["block_size"], g["num_tokens"]
    order = g["free_blocks"] + [b for b in range(g["pool_blocks"]) if b not in g["free_blocks"]]
    m = BM(g["pool_blocks"], B, order)
    m.add_sequence(0)
    slots = [int(m.append_slots([0])[0][0]) for _ in range(n)]
    table, lens = m.block_tables([0], 4)
    assert table[0, :3].tolist() == g["expected"]["block_table"] and table[0, 3] == -1
    assert lens[0] == n
    assert slots == [table[0, p // B] * B + p % B for p in range(n)]
    assert 3 * B - n == g["expected"]["unused_slots_paged"]


def test_copy_on_write_rule(BM):
    m = BM(100, 16)
    m.add_sequence(0)
    for _ in range(20):                      # one full block + 4 tokens
        m.append_slots([0])
    for c in (1, 2, 3):
        m.fork(0, c)
    t0, _ = m.block_tables([0], 4)
    full, partial = int(t0[0, 0]), int(t0[0, 1])
    assert m.ref_count(full) == 4 and m.ref_count(partial) == 4
    slots, pairs = m.append_slots([1, 2, 3, 0])
    assert pairs.shape == (3, 2) and (pairs[:, 0] == partial).all() and len(set(pairs[:, 1])) == 3
    t, lens = m.block_tables([1, 2, 3, 0], 4)
    assert (t[:, 0] == full).all()                     # full block stays shared
    assert t[3, 1] == partial                          # last holder writes in place
    assert set(t[:3, 1]) == set(pairs[:, 1])
    assert m.ref_count(partial) == 1 and m.ref_count(full) == 4
    assert (lens == 21).all()
    assert all(slots[i] == t[i, 1] * 16 + 4 for i in range(4))


def test_free_returns_blocks_and_conserves_the_pool(BM):
    rng = np.random.default_rng(3)
    NB, B = 300, 16
    m = BM(NB, B, rng.permutation(NB))
    live = []
    nxt = 0
    for step in range(400):
        op = rng.integers(0, 4)
        if op == 0 or not live:
            m.add_sequence(nxt)
            live.append(nxt)
            nxt += 1
        elif op == 1:
            m.fork(int(rng.choice(live)), nxt)
            live.append(nxt)
            nxt += 1
        elif op == 2 and len(live) > 1:
            victim = int(rng.choice(live))
            m.free_sequence(victim)
            live.remove(victim)
        else:
            ids = rng.choice(live, size=min(len(live), 5), replace=False)
            try:
                m.append_slots(ids)
            except Exception:
                pass
        # conservation: free blocks + distinct referenced blocks == pool size, refs match tables
        tabs, lens = m.block_tables(live, 64)
        used = {}
        for row, L in zip(tabs, lens):
            nb = -(-int(L) // B)
            assert (row[:nb] >= 0).all() and (row[nb:] == -1).all()
            assert nb * B - L <= B - 1                 # waste below one block
            for b in row[:nb]:
                used[int(b)] = used.get(int(b), 0) + 1
        assert m.num_free + len(used) == NB
        assert all(m.ref_count(b) == c for b, c in used.items())


def test_out_of_blocks_changes_nothing(BM):
    m = BM(3, 4)
    for s in range(3):
        m.add_sequence(s)
    m.append_slots([0, 1, 2])
    assert m.num_free == 0
    for _ in range(3):
        m.append_slots([0, 1, 2])                      # fill the three blocks
    from paged_kv_cache_324_b200.binding import PagedKVError
    with pytest.raises(PagedKVError) as e:
        m.append_slots([0, 1])
    assert e.value.status == 6
    assert m.sequence_length(0) == 4 and m.sequence_length(1) == 4
    m.free_sequence(2)
    assert m.num_free == 1
    slots, pairs = m.append_slots([0])
    assert len(pairs) == 0 and m.sequence_length(0) == 5


def test_matches_the_harness_allocator(BM):
    """Same tables, slots and copy pairs as the Python allocator the workloads use."""
    rng = np.random.default_rng(9)
    NB, B = 2000, 16
    order = rng.permutation(NB)
    m = BM(NB, B, order)
    py = wl.BlockAllocator(order)
    py_tables = {}
    seqs = []
    for s in range(6):
        m.add_sequence(s)
        py_tables[s] = []
        seqs.append(s)
    lens = {s: 0 for s in seqs}
    for step in range(300):
        if step % 37 == 5:                              # fork a random sequence
            parent = int(rng.choice(seqs))
            child = max(seqs) + 1
            m.fork(parent, child)
            py_tables[child] = py.fork(py_tables[parent])
            lens[child] = lens[parent]
            seqs.append(child)
        ids = [int(x) for x in rng.choice(seqs, size=min(3, len(seqs)), replace=False)]
        slots, pairs = m.append_slots(ids)
        py_pairs, py_slots = [], []
        for s in ids:
            py_slots.append(py.slot_for_append(py_tables[s], lens[s], B, py_pairs))
            lens[s] += 1
        assert slots.tolist() == py_slots
        assert [tuple(p) for p in pairs.tolist()] == py_pairs
    tabs, L = m.block_tables(seqs, 64)
    for i, s in enumerate(seqs):
        assert tabs[i, :len(py_tables[s])].tolist() == py_tables[s] and L[i] == lens[s]


def test_free_order_must_cover_the_pool(BM):
    with pytest.raises(ValueError):
        BM(8, 4, [0, 1, 2])                              # shorter than the pool: refused before the library
    with pytest.raises(ValueError):
        BM(4, 4, [0, 1, 1, 2])                           # not a permutation: refused by the library
    assert BM(4, 4, [3, 1, 0, 2]).num_free == 4


def test_bad_arguments(BM):
    with pytest.raises(ValueError):
        BM(4, 16, [0, 1, 1, 2])                         # not a permutation
    m = BM(4, 16)
    m.add_sequence(1)
    from paged_kv_cache_324_b200.binding import PagedKVError
    with pytest.raises(PagedKVError):
        m.add_sequence(1)
    with pytest.raises(PagedKVError):
        m.fork(7, 8)
    with pytest.raises(PagedKVError):
        m.append_slots([1, 1])                          # one token per sequence per call
    with pytest.raises(PagedKVError):
        m.free_sequence(5)


# --------------------------------------------------------------------------
# prefix caching by block content, and swapping between two managers
# --------------------------------------------------------------------------

def _fill(m, seq, n):
    """Append n tokens to seq one at a time; returns the slots."""
    return [int(m.append_slots([seq])[0][0]) for _ in range(n)]


def test_prefix_cache_shares_whole_matching_blocks(BM):
    m = BM(64, 4, np.random.default_rng(1).permutation(64))
    a = np.arange(100, 122)                                  # 22 tokens: 5 full blocks + 2
    m.add_sequence(0)
    _fill(m, 0, len(a))
    m.cache_sequence(0, a)
    assert m.num_cached == 5
    b = np.concatenate([a[:13], [999], a[14:]])               # differs inside block 3
    got = m.add_sequence_cached(1, b)
    assert got == 12                                          # blocks 0-2 match, block 3 does not
    ta, _ = m.block_tables([0], 8)
    tb, lb = m.block_tables([1], 8)
    assert tb[0, :3].tolist() == ta[0, :3].tolist() and tb[0, 3] == -1 and lb[0] == 12
    assert all(m.ref_count(int(x)) == 2 for x in ta[0, :3]) and m.ref_count(int(ta[0, 3])) == 1
    # the rest of the prompt is appended into fresh blocks
    _fill(m, 1, len(b) - got)
    tb, lb = m.block_tables([1], 8)
    assert lb[0] == len(b) and tb[0, 3] not in ta[0].tolist()


def test_prefix_cache_leaves_one_token_to_compute(BM):
    m = BM(32, 4)
    a = np.arange(12)                                         # exactly 3 blocks
    m.add_sequence(0)
    _fill(m, 0, 12)
    m.cache_sequence(0, a)
    assert m.add_sequence_cached(1, a) == 8                   # not all 12: the last token is computed
    assert m.add_sequence_cached(2, a[:1]) == 0
    assert m.add_sequence_cached(3, np.arange(13)) == 12


def test_idle_cached_blocks_are_reused_then_evicted_oldest_first(BM):
    m = BM(6, 2, np.arange(6))
    m.add_sequence(0)
    _fill(m, 0, 4)                                            # blocks 0, 1
    m.cache_sequence(0, [5, 6, 7, 8])
    m.add_sequence(1)
    _fill(m, 1, 4)                                            # blocks 2, 3
    m.cache_sequence(1, [1, 2, 3, 4])
    m.free_sequence(0)                                        # blocks 0, 1 idle first
    m.free_sequence(1)                                        # then 2, 3
    assert m.num_free == 6 and m.num_cached == 4
    assert m.add_sequence_cached(2, [5, 6, 7, 8, 9]) == 4     # hit on idle blocks
    t, _ = m.block_tables([2], 4)
    assert t[0, :2].tolist() == [0, 1] and m.ref_count(0) == 1
    m.add_sequence(3)
    _fill(m, 3, 6)                                            # free 4, 5, then evicts idle 2 (oldest idle)
    t, _ = m.block_tables([3], 4)
    assert t[0, :3].tolist() == [4, 5, 2]
    assert m.num_cached == 3                                  # block 2's entry is gone
    assert m.add_sequence_cached(4, [1, 2, 3, 4, 0]) == 0     # its first block was evicted: no hit


def test_blocks_after_a_duplicate_prefix_block_stay_reachable(BM):
    """Two sequences prefilled with the same first block in different physical blocks: the second
    one's later blocks are chained on the block already cached for that content, so a request
    with the second sequence's prompt hits all of its full blocks."""
    m = BM(16, 2)
    x, y = [1, 2, 3, 4], [1, 2, 7, 8]
    m.add_sequence(0)
    _fill(m, 0, 4)
    m.cache_sequence(0, x)
    m.add_sequence(1)
    _fill(m, 1, 4)                                            # its own copy of tokens 1, 2
    m.cache_sequence(1, y)
    assert m.num_cached == 3                                  # [1,2] once, [3,4] and [7,8]
    assert m.add_sequence_cached(2, y + [9]) == 4
    t, _ = m.block_tables([0, 1, 2], 3)
    assert t[2, 0] == t[0, 0] and t[2, 1] == t[1, 1]


def test_stale_child_of_a_recycled_block_does_not_match(BM):
    m = BM(4, 2, np.arange(4))
    m.add_sequence(0)
    _fill(m, 0, 4)                                            # blocks 0 (tokens 1,2), 1 (tokens 3,4)
    m.cache_sequence(0, [1, 2, 3, 4])
    m.free_sequence(0)
    m.add_sequence(1)
    _fill(m, 1, 6)                                            # 2, 3, then evicts 0 and reuses it
    m.cache_sequence(1, [1, 2, 9, 9, 7, 7])                   # block 2 now holds tokens 1,2 again
    # block 1 (tokens 3,4) still names block 0 of the old generation as its predecessor
    m.free_sequence(1)
    got = m.add_sequence_cached(2, [1, 2, 3, 4, 5])
    t, _ = m.block_tables([2], 4)
    assert got == 2 and t[0, 0] == 2                          # only the first block matches


def test_swap_moves_a_group_and_its_shared_blocks(BM):
    gpu = BM(40, 4, np.random.default_rng(2).permutation(40))
    host = BM(20, 4, np.arange(20))
    gpu.add_sequence(0)
    _fill(gpu, 0, 9)                                          # 3 blocks, the last partial
    gpu.fork(0, 1)
    gpu.fork(0, 2)
    _fill(gpu, 1, 1)                                          # copy-on-write of the partial block
    gpu.add_sequence(3)
    _fill(gpu, 3, 5)
    before, lens0 = gpu.block_tables([0, 1, 2, 3], 4)
    free0 = gpu.num_free
    pairs = gpu.swap_to(host, [1, 2])                         # the group of samples 1 and 2
    distinct = set(before[1, :3].tolist()) | set(before[2, :3].tolist())
    assert len(pairs) == len(distinct) == 4                   # 2 shared full + 1 shared partial + 1 copy
    assert set(pairs[:, 0].tolist()) == distinct
    assert gpu.sequence_length(1) == -1 and host.sequence_length(1) == 10 and host.sequence_length(2) == 9
    ht, _ = host.block_tables([1, 2], 4)
    m = dict(pairs.tolist())
    assert ht[0, :3].tolist() == [m[b] for b in before[1, :3]]
    assert ht[1, :3].tolist() == [m[b] for b in before[2, :3]]
    assert host.ref_count(m[int(before[1, 0])]) == 2          # shared by both swapped samples
    assert gpu.num_free == free0 + 1                          # only the private copy left the GPU pool
    # and back, into whatever blocks the GPU manager has free now
    back = host.swap_to(gpu, [1, 2])
    assert len(back) == 4 and host.num_free == 20
    t2, lens2 = gpu.block_tables([1, 2], 4)
    assert lens2.tolist() == lens0[1:3].tolist()


def test_swap_is_all_or_nothing(BM):
    from paged_kv_cache_324_b200.binding import PagedKVError
    gpu = BM(10, 4)
    host = BM(1, 4)
    gpu.add_sequence(0)
    _fill(gpu, 0, 8)                                          # 2 blocks, host has 1
    with pytest.raises(PagedKVError) as e:
        gpu.swap_to(host, [0])
    assert e.value.status == 6 and gpu.sequence_length(0) == 8 and host.num_free == 1
    with pytest.raises(PagedKVError):
        gpu.swap_to(host, [5])                                # unknown sequence


class _ModelManager:
    """An independent Python statement of the manager's rules, for randomized comparison:
    FIFO free list; a new block only when the last is full; fork shares; copy on write for a
    shared partial last block (the last holder writes in place); full blocks registered under
    their token content chained on their predecessor, hits confirmed exactly (tokens, the
    predecessor block and its generation); registered blocks without holders stay cached and are
    reused oldest-released first when the free list is empty."""

    def __init__(self, n, bs, order):
        self.bs = bs
        self.free = list(order)
        self.ref = [0] * n
        self.seqs = {}
        self.key_of = {}          # block -> (content key)
        self.cache = {}           # content key -> block
        self.gen = [0] * n
        self.idle = []            # cached blocks with no holder, oldest first

    def _take(self):
        if self.free:
            b = self.free.pop(0)
        else:
            b = self.idle.pop(0)
            self._uncache(b)
        self.ref[b] = 1
        return b

    def _uncache(self, b):
        k = self.key_of.pop(b)
        if self.cache.get(k) == b:
            del self.cache[k]
        self.gen[b] += 1

    def _release(self, b):
        self.ref[b] -= 1
        if self.ref[b] == 0:
            (self.idle if b in self.key_of else self.free).append(b)

    def _acquire(self, b):
        if b in self.idle:
            self.idle.remove(b)
        self.ref[b] += 1

    def available(self):
        return len(self.free) + len(self.idle)

    def append(self, ids):
        need, copied = 0, {}
        for s in ids:
            blocks, L = self.seqs[s]
            if L % self.bs == 0:
                need += 1
            else:
                last = blocks[-1]
                if self.ref[last] - copied.get(last, 0) > 1:
                    copied[last] = copied.get(last, 0) + 1
                    need += 1
        if need > self.available():
            return None
        slots, pairs = [], []
        for s in ids:
            blocks, L = self.seqs[s]
            off = L % self.bs
            if off == 0:
                blocks.append(self._take())
            elif self.ref[blocks[-1]] > 1:
                fresh = self._take()
                pairs.append((blocks[-1], fresh))
                self.ref[blocks[-1]] -= 1
                blocks[-1] = fresh
            slots.append(blocks[-1] * self.bs + off)
            self.seqs[s] = (blocks, L + 1)
        return slots, pairs

    def fork(self, p, c):
        blocks, L = self.seqs[p]
        for b in blocks:
            self._acquire(b)
        self.seqs[c] = (list(blocks), L)

    def free_seq(self, s):
        for b in self.seqs.pop(s)[0]:
            self._release(b)

    def cache_seq(self, s, toks):
        blocks, _ = self.seqs[s]
        prev, prev_gen = -1, 0
        for j in range(len(toks) // self.bs):
            b = blocks[j]
            key = (tuple(toks[j * self.bs:(j + 1) * self.bs]), prev, prev_gen)
            if b not in self.key_of and key in self.cache:
                b = self.cache[key]               # the same prefix is cached in another block
            elif b not in self.key_of:
                self.key_of[b] = key
                self.cache[key] = b
            prev, prev_gen = b, self.gen[b]

    def add_cached(self, s, toks):
        got, prev, prev_gen = [], -1, 0
        for j in range((len(toks) - 1) // self.bs if len(toks) else 0):
            key = (tuple(toks[j * self.bs:(j + 1) * self.bs]), prev, prev_gen)
            b = self.cache.get(key)
            if b is None:
                break
            got.append(b)
            prev, prev_gen = b, self.gen[b]
        for b in got:
            self._acquire(b)
        self.seqs[s] = (got, len(got) * self.bs)
        return len(got) * self.bs


def test_randomized_against_a_python_model(BM):
    """Random add / cached add / append / fork / register / free sequences: the library and the
    model give the same slots, copy pairs, cached-token counts, tables and free counts."""
    from paged_kv_cache_324_b200.binding import PagedKVError
    rng = np.random.default_rng(31)
    NB, B = 48, 4
    order = rng.permutation(NB)
    m = BM(NB, B, order)
    py = _ModelManager(NB, B, order.tolist())
    toks = {}                                    # tokens written per sequence
    vocab = 3                                    # small, so prompts repeat and the cache hits
    nxt = 0
    for step in range(1500):
        live = sorted(py.seqs)
        op = rng.integers(0, 6)
        if op == 0 or not live:
            prompt = rng.integers(0, vocab, size=int(rng.integers(1, 14))).tolist()
            got = m.add_sequence_cached(nxt, prompt)
            assert got == py.add_cached(nxt, prompt)
            toks[nxt] = prompt[:got]
            nxt += 1
        elif op == 1:
            p = int(rng.choice(live))
            m.fork(p, nxt)
            py.fork(p, nxt)
            toks[nxt] = list(toks[p])
            nxt += 1
        elif op == 2 and len(live) > 2:
            s = int(rng.choice(live))
            m.free_sequence(s)
            py.free_seq(s)
            del toks[s]
        elif op == 3:
            s = int(rng.choice(live))
            m.cache_sequence(s, toks[s])
            py.cache_seq(s, toks[s])
        else:
            ids = [int(x) for x in rng.choice(live, size=min(len(live), int(rng.integers(1, 4))), replace=False)]
            want = py.append(ids)
            if want is None:
                with pytest.raises(PagedKVError):
                    m.append_slots(ids)
                continue
            slots, pairs = m.append_slots(ids)
            assert slots.tolist() == want[0] and [tuple(p) for p in pairs.tolist()] == want[1]
            for s in ids:
                toks[s].append(int(rng.integers(0, vocab)))
        assert m.num_free == py.available()
    live = sorted(py.seqs)
    tabs, lens = m.block_tables(live, 16)
    for i, s in enumerate(live):
        blocks, L = py.seqs[s]
        assert tabs[i, :len(blocks)].tolist() == blocks and lens[i] == L


def test_append_tokens_equals_repeated_single_appends(BM):
    """A chunk append gives the same slots, copy pairs, tables and free counts as one
    single-token append per token, on twin managers driven through random forks and chunks."""
    rng = np.random.default_rng(23)
    for B in (1, 4, 16):
        NB = 400
        order = rng.permutation(NB).tolist()
        a, b = BM(NB, B, order), BM(NB, B, order)
        live = []
        for step in range(150):
            r = rng.random()
            if r < 0.15 or not live:
                sid = 1000 * B + step
                a.add_sequence(sid)
                b.add_sequence(sid)
                live.append(sid)
            elif r < 0.35:
                sid, child = int(rng.choice(live)), 1000 * B + step
                a.fork(sid, child)
                b.fork(sid, child)
                live.append(child)
            else:
                sid, n = int(rng.choice(live)), int(rng.integers(0, 3 * B + 2))
                try:
                    got_slots, got_pairs = a.append_tokens(sid, n)
                except Exception:
                    assert a.num_free < n // B + 2      # only for want of blocks
                    continue
                want_slots, want_pairs = [], []
                for _ in range(n):
                    s1, p1 = b.append_slots([sid])
                    want_slots.append(int(s1[0]))
                    want_pairs += [tuple(x) for x in p1.tolist()]
                assert got_slots.tolist() == want_slots
                assert [tuple(x) for x in got_pairs.tolist()] == want_pairs and len(want_pairs) <= 1
            assert a.num_free == b.num_free
        ta, la = a.block_tables(live, 64)
        tb, lb = b.block_tables(live, 64)
        assert np.array_equal(ta, tb) and np.array_equal(la, lb)


def test_append_tokens_is_all_or_nothing(BM):
    from paged_kv_cache_324_b200.binding import PagedKVError
    m = BM(4, 4)
    m.add_sequence(0)
    m.append_tokens(0, 6)                              # blocks 0, 1 (two slots left)
    m.fork(0, 1)
    with pytest.raises(PagedKVError):
        m.append_tokens(1, 11)                         # a copy + 2 new blocks > 2 free
    assert m.num_free == 2 and m.sequence_length(1) == 6
    slots, pairs = m.append_tokens(1, 2)               # the copy of the shared partial block
    assert len(pairs) == 1 and m.num_free == 1 and m.sequence_length(1) == 8
    assert m.append_tokens(0, 0)[0].size == 0 and m.sequence_length(0) == 6
