"""The benchmark's multi-rank host logic on CPU: two gloo ranks, no GPU.

Each rank reports its own bytes and time; the job's throughput is all ranks'
bytes over the slowest rank's time (weak scaling, no collective on the data
path), and rank 0 alone runs the oracle reference arm."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        # rank r moved (r + 1) GB in (r + 1) * 100 ms over 10 steps
        gbps, ms_step = bench.job_throughput((rank + 1) * 1e9, (rank + 1) * 100.0, 10, True, torch, "cpu")
        mx = bench.max_over_ranks(torch, float(rank), True, "cpu")
        sm = bench.sum_over_ranks(torch, 1.0, True, "cpu")
        q.put((rank, gbps, ms_step, mx, sm))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_like_the_driver():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, gbps, ms_step, mx, sm in res:
        # slowest rank: 200 ms / 10 steps; all bytes: 1 + 2 GB per step
        assert ms_step == pytest.approx(20.0)
        assert gbps == pytest.approx(3e9 / 20e-3 / 1e9)
        assert mx == 1.0 and sm == 2.0


def test_single_rank_needs_no_process_group():
    import bench
    gbps, ms = bench.job_throughput(2e9, 50.0, 5, False, torch)
    assert ms == pytest.approx(10.0) and gbps == pytest.approx(200.0)


def test_reference_arm_byte_accounting_on_cpu():
    """The CPU reference arm's per-step sample bytes equal the workload's step bytes
    when the sample is the whole batch (tiny workload)."""
    import bench
    from paged_kv_cache_324_b200 import workload as wl
    w = wl.make("tiny")
    r = bench.OracleRunner(w)
    assert r.step() == wl.step_algorithmic_bytes(w)
    assert 0 < r.step(1) < wl.step_algorithmic_bytes(w)


def test_cpu_baseline_sample_reports_a_one_core_figure():
    """The bench's oracle sample: whole steps on all cores, then a one-thread step over a prefix
    of the sequences, both with positive byte counts and times."""
    import bench
    from paged_kv_cache_324_b200 import workload as wl
    w = wl.make("tiny")
    n, nbytes, el, cores, (n1, b1, el1) = bench.cpu_oracle_sample(w, 0.05, one_core_s=0.05)
    assert n >= 1 and nbytes == n * wl.step_algorithmic_bytes(w) and el > 0 and cores >= 1
    assert 1 <= n1 <= w.num_seqs and b1 > 0 and el1 > 0


def _sharded_worker(rank, world, port, q):
    """One rank of a head-sharded decode: its share of the KV heads (identical block tables), its
    outputs computed alone, then gathered over gloo the way the ranks' outputs would be."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from paged_kv_cache_324_b200 import workload as wl
        from tests import harness as H
        w = wl.make("gqa", small=True)
        sh = wl.shard_heads(w, rank, world)
        out = torch.from_numpy(H.oracle_step(sh)["out"])
        parts = [torch.empty_like(out) for _ in range(world)]
        dist.all_gather(parts, out)
        if rank == 0:
            q.put(torch.cat(parts, dim=1).numpy())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_with_head_shards_reassemble_the_whole_batch():
    """Two processes, each holding half of the KV heads: their outputs side by side equal the
    single-process result bit for bit (the path shards with no exchange inside attention)."""
    import numpy as np
    from paged_kv_cache_324_b200 import workload as wl
    from tests import harness as H
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_sharded_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = q.get(timeout=300)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert np.array_equal(got, H.oracle_step(wl.make("gqa", small=True))["out"])
