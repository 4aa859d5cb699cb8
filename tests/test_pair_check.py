"""Host check of block-pair lists (pkv_check_block_pairs), on CPU.

The copy-on-write and swap kernels copy every pair independently, so their
pair lists must name blocks inside the pools, never write one destination
twice and, within one pool, never write a block another pair reads.  The
kernels cannot check this without a synchronisation; the host check does, and
the native block manager's own pair lists must always pass it.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_324_b200 import binding as B


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_324_b200 import build
    build.build()


def ok(pairs, src_nb=10, dst_nb=10, same=True):
    try:
        B.check_block_pairs(np.asarray(pairs, np.int64).reshape(-1, 2), src_nb, dst_nb, same)
        return True
    except ValueError:
        return False


def test_valid_lists_pass():
    assert ok([])
    assert ok([[0, 1], [2, 3], [4, 5]])
    assert ok([[0, 1], [0, 2], [0, 3]])            # one source copied to several blocks
    assert ok([[9, 0]], src_nb=10, dst_nb=1, same=False)


def test_ids_out_of_range_fail():
    assert not ok([[10, 1]])
    assert not ok([[-1, 1]])
    assert not ok([[1, 10]])
    assert not ok([[1, -3]])
    assert not ok([[0, 5]], src_nb=10, dst_nb=5, same=False)
    assert not ok([[7, 0]], src_nb=5, dst_nb=10, same=False)


def test_repeated_destination_fails():
    assert not ok([[0, 4], [1, 4]])
    assert not ok([[0, 4], [1, 2], [3, 4]], same=False)


def test_destination_that_is_a_source_fails_only_within_one_pool():
    assert not ok([[0, 1], [1, 2]])                # block 1 written by one pair, read by another
    assert not ok([[3, 3]])                        # a block onto itself
    assert ok([[0, 1], [1, 2]], same=False)        # two pools: source 1 and destination 1 differ
    assert ok([[3, 3]], same=False)


def test_bad_sizes_fail():
    with pytest.raises(ValueError):
        B.check_block_pairs(np.zeros((1, 2), np.int64), 0, 10, True)
    with pytest.raises(ValueError):
        B.check_block_pairs(np.zeros((1, 2), np.int64), 10, 0, False)


def test_brute_force_agreement():
    """Random small lists against a direct statement of the three conditions."""
    rng = np.random.default_rng(5)
    for _ in range(2000):
        n = int(rng.integers(0, 6))
        src_nb, dst_nb = int(rng.integers(1, 8)), int(rng.integers(1, 8))
        same = bool(rng.integers(0, 2))
        if same:
            dst_nb = src_nb
        p = rng.integers(-1, 9, size=(n, 2))
        want = (all(0 <= s < src_nb and 0 <= d < dst_nb for s, d in p)
                and len({int(d) for _, d in p}) == n
                and (not same or not ({int(d) for _, d in p} & {int(s) for s, _ in p})))
        assert ok(p, src_nb, dst_nb, same) == want, (p.tolist(), src_nb, dst_nb, same)


def test_copy_blocks_checks_before_touching_the_pools(monkeypatch):
    """check=True (or PKV_DEBUG) rejects a bad list before any pointer is taken; without either,
    the call goes straight to the library (here it then rejects the CPU tensors)."""
    k = torch.zeros((8, 2, 16, 64), dtype=torch.float16)
    v = torch.zeros_like(k)
    bad = torch.tensor([[0, 3], [1, 3]], dtype=torch.int64)
    with pytest.raises(ValueError, match="block pairs"):
        B.copy_blocks(k, v, bad, check=True)
    monkeypatch.setenv("PKV_DEBUG", "1")
    with pytest.raises(ValueError, match="block pairs"):
        B.copy_blocks(k, v, bad)
    with pytest.raises(ValueError, match="block pairs"):
        B.swap_blocks(k, v, k, v, torch.tensor([[0, 1], [1, 2]], dtype=torch.int64))
    with pytest.raises(ValueError, match="CUDA tensor"):
        B.copy_blocks(k, v, bad, check=False)
    monkeypatch.delenv("PKV_DEBUG")
    with pytest.raises(ValueError, match="CUDA tensor"):
        B.copy_blocks(k, v, bad)
    good = torch.tensor([[0, 3], [1, 4]], dtype=torch.int64)
    with pytest.raises(ValueError, match="CUDA tensor"):  # passes the check, then needs the GPU
        B.copy_blocks(k, v, good, check=True)


def test_block_manager_pairs_always_pass():
    """Random forks, appends, frees and swaps on the native manager: every copy-on-write list
    (one pool) and every swap list (two pools) satisfies the copy kernels' preconditions."""
    rng = np.random.default_rng(17)
    NB, NH, Bs = 96, 64, 4
    gpu, host = B.BlockManager(NB, Bs), B.BlockManager(NH, Bs)
    live, swapped, nxt = [], [], 0
    n_cow = n_swap = 0
    for _ in range(600):
        r = rng.random()
        if r < 0.1 or not live:
            gpu.add_sequence(nxt)
            live.append(nxt)
            nxt += 1
        elif r < 0.25:
            gpu.fork(int(rng.choice(live)), nxt)
            live.append(nxt)
            nxt += 1
        elif r < 0.75:
            ids = rng.choice(live, size=int(rng.integers(1, len(live) + 1)), replace=False)
            try:
                _, pairs = gpu.append_slots(ids)
            except B.PagedKVError:                  # out of blocks: nothing was changed
                continue
            B.check_block_pairs(pairs, NB, NB, True)
            n_cow += len(pairs)
        elif r < 0.85:
            s = int(rng.choice(live))
            gpu.free_sequence(s)
            live.remove(s)
        elif r < 0.93 and live:
            s = int(rng.choice(live))
            try:
                pairs = gpu.swap_to(host, [s])
            except B.PagedKVError:
                continue
            B.check_block_pairs(pairs, NB, NH, False)
            n_swap += len(pairs)
            live.remove(s)
            swapped.append(s)
        elif swapped:
            s = swapped.pop(int(rng.integers(0, len(swapped))))
            try:
                pairs = host.swap_to(gpu, [s])
            except B.PagedKVError:
                swapped.append(s)
                continue
            B.check_block_pairs(pairs, NH, NB, False)
            n_swap += len(pairs)
            live.append(s)
    assert n_cow > 0 and n_swap > 0
