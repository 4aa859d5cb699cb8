"""The native block manager under concurrent callers, on CPU.

ctypes releases the GIL for the duration of each foreign call, so several Python
threads drive one manager at the same time: each thread adds, forks, appends
(single tokens and chunks) and frees its own sequences, and two more threads swap
sequences between two managers in opposite directions (a lock-order mistake
would deadlock them).  Afterwards every block is accounted for: the free count
plus the blocks in use equals the pool, and each block's reference count equals
the number of sequences whose table holds it.
"""
import threading

import numpy as np

from paged_kv_cache_324_b200.binding import BlockManager, PagedKVError

NB, BS = 512, 4


def conserve(m, seqs):
    holders = {}
    if seqs:
        t, lens = m.block_tables(seqs, 128)
        for row, L in zip(t, lens):
            for b in row[: -(-int(L) // BS)]:
                holders[int(b)] = holders.get(int(b), 0) + 1
    assert m.num_free + len(holders) == NB
    for b in range(NB):
        assert m.ref_count(b) == holders.get(b, 0), b


def test_concurrent_callers_keep_every_block_accounted_for():
    from paged_kv_cache_324_b200 import build
    build.build()
    a, b = BlockManager(NB, BS), BlockManager(NB, BS)
    owned = {a: set(), b: set()}
    lock = threading.Lock()                          # guards the test's own bookkeeping only
    errors = []

    def worker(tid):
        rng = np.random.default_rng(100 + tid)
        mine = []
        try:
            for step in range(400):
                r = rng.random()
                sid = tid * 100000 + step
                if r < 0.15 or not mine:
                    a.add_sequence(sid)
                    mine.append(sid)
                elif r < 0.25:
                    a.fork(int(rng.choice(mine)), sid)
                    mine.append(sid)
                elif r < 0.6:
                    ids = list(rng.choice(mine, size=min(len(mine), 3), replace=False))
                    try:
                        a.append_slots(ids)
                    except PagedKVError:
                        pass
                elif r < 0.8:
                    try:
                        a.append_tokens(int(rng.choice(mine)), int(rng.integers(1, 9)))
                    except PagedKVError:
                        pass
                else:
                    s = mine.pop(int(rng.integers(0, len(mine))))
                    a.free_sequence(s)
            with lock:
                owned[a].update(mine)
        except Exception as e:                       # reported on the main thread
            errors.append(e)

    def swapper(src, dst, base):
        rng = np.random.default_rng(base)
        try:
            for i in range(150):
                sid = base + i
                src.add_sequence(sid)
                try:
                    src.append_tokens(sid, int(rng.integers(1, 12)))
                    src.swap_to(dst, [sid])
                    dst.free_sequence(sid)
                except PagedKVError:
                    src.free_sequence(sid)
        except Exception as e:
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(t,)) for t in range(4)]
    threads += [threading.Thread(target=swapper, args=(a, b, 10_000_000)),
                threading.Thread(target=swapper, args=(b, a, 20_000_000))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
        assert not t.is_alive(), "a thread did not finish (deadlock?)"
    assert not errors, errors
    conserve(a, sorted(owned[a]))
    conserve(b, [])
