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
