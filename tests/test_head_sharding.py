"""Sharding a decode workload by KV head (one share per GPU, identical block tables), on CPU:
every shard's pools are the full pools' slice, and the oracle's outputs of the shards placed
side by side along the head axis equal the whole workload's, bit for bit."""
import numpy as np
import pytest

from paged_kv_cache_324_b200 import workload as wl
from tests import harness as H


@pytest.mark.parametrize("name,world", [("gqa", 2), ("gqa", 8), ("fp8", 4), ("prefix", 2), ("tiny", 4)])
def test_shards_side_by_side_equal_the_whole(name, world):
    w = wl.make(name, small=True)
    full = H.oracle_step(w)
    outs = []
    n = w.num_kv_heads // world
    for r in range(world):
        sh = wl.shard_heads(w, r, world)
        assert sh.num_kv_heads == n and sh.num_heads == w.num_heads // world
        assert np.array_equal(sh.block_tables, w.block_tables) and np.array_equal(sh.context_lens, w.context_lens)
        assert np.array_equal(sh.initial_pool("k"), w.initial_pool("k")[:, r * n:(r + 1) * n])
        o = H.oracle_step(sh)
        assert np.array_equal(o["k_pool"], full["k_pool"][:, r * n:(r + 1) * n])
        assert np.array_equal(o["v_pool"], full["v_pool"][:, r * n:(r + 1) * n])
        outs.append(o["out"])
    assert np.array_equal(np.concatenate(outs, axis=1), full["out"])


def test_uneven_or_repeated_splits_are_refused():
    w = wl.make("tiny", small=True)                    # 8 KV heads
    with pytest.raises(ValueError):
        wl.shard_heads(w, 0, 3)
    with pytest.raises(ValueError):
        wl.shard_heads(w, 2, 2)
    with pytest.raises(ValueError):
        wl.shard_heads(wl.shard_heads(w, 0, 2), 0, 2)


def test_shard_bytes_add_up_to_the_whole():
    """KV, q and out bytes split exactly; every rank reads the block tables and lengths itself."""
    w = wl.make("gqa", small=True)
    world = 4
    shards = [wl.shard_heads(w, r, world) for r in range(world)]
    nblk = int(((w.context_lens.astype(np.int64) + w.block_size - 1) // w.block_size).sum())
    per_rank_tables = 4 * nblk + 4 * w.num_seqs
    assert sum(wl.decode_algorithmic_bytes(s) for s in shards) == \
        wl.decode_algorithmic_bytes(w) + (world - 1) * per_rank_tables
