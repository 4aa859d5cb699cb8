"""GPU parity: the CUDA library against the float64 oracle on the same seeded inputs.

Pools after reshape_and_cache / copy_blocks must be bit-identical to the
oracle's; attention outputs must meet the comparison rule in tests/parity.py.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_324_b200 import binding as B_
from paged_kv_cache_324_b200 import workload as wl
from tests import harness as H
from tests.parity import attention_close

pytestmark = pytest.mark.gpu


def check_step(w, partition_size=None, pools=True):
    g = H.gpu_step(w, partition_size=partition_size, keep_pools=pools)
    o = H.oracle_step(w)
    assert g["err"] == 0, f"device error word {g['err']:#x}"
    if pools:
        assert np.array_equal(g["k_pool"], o["k_pool"]), "K pool differs from the oracle's"
        assert np.array_equal(g["v_pool"], o["v_pool"]), "V pool differs from the oracle's"
    ok, rep = attention_close(g["out"], o["out"], w.kv_dtype, w.q_dtype)
    assert ok, rep
    return g, o, rep


@pytest.mark.parametrize("name", wl.NAMES)
def test_small_workload(name):
    check_step(wl.make(name, small=True))


@pytest.mark.parametrize("ps", [64, 128, 512, 1 << 20])
def test_partition_size_does_not_change_result(ps):
    w = wl.make("gqa", small=True)
    g = H.gpu_step(w, partition_size=ps, keep_pools=False)
    o = H.oracle_step(w)
    assert g["err"] == 0
    ok, rep = attention_close(g["out"], o["out"], w.kv_dtype, w.q_dtype)
    assert ok, (ps, rep)


@pytest.mark.parametrize("q_dtype,kv_dtype,B", [("f16", "f16", 16), ("bf16", "bf16", 32), ("f16", "e4m3", 16),
                                                ("bf16", "e4m3", 32)])
def test_stated_partitions_streamed_several_per_cta(q_dtype, kv_dtype, B):
    """Enough sequences that the automatic partition (1,024 tokens of 16-bit K/V, 2,048 of E4M3)
    holds several stated 128-token ones: CTAs stream runs of them, each run's partitions ending in
    partials of their own, with lengths below, at and around partition and run boundaries."""
    lens = [1, 127, 128, 129, 700, 1023, 1024, 1025, 1500, 255, 256, 2047] * 4
    Hkv, G, D = 8, 4, 128
    w = wl.independent_sequences(f"runs-{q_dtype}-{kv_dtype}-{B}", 300 + B, len(lens), Hkv * G, Hkv, D, B,
                                 4096, q_dtype, kv_dtype, lens)
    auto = B_.decode_partition_size(w.num_seqs, Hkv, D, kv_dtype, B, w.max_context_len, 0)
    assert auto >= 8 * 128                        # a CTA takes several stated partitions
    g = H.gpu_step(w, partition_size=128, keep_pools=False)
    o = H.oracle_step(w)
    assert g["err"] == 0
    ok, rep = attention_close(g["out"], o["out"], w.kv_dtype, w.q_dtype)
    assert ok, rep


EDGE_LENS = [1, 15, 16, 17, 31, 32, 33, 63, 64, 65, 511, 512, 513, 1025]


@pytest.mark.parametrize("q_dtype,kv_dtype", [("f16", "f16"), ("bf16", "bf16"), ("f16", "e4m3"),
                                              ("bf16", "e4m3")])
@pytest.mark.parametrize("B", [16, 32])
@pytest.mark.parametrize("G", [1, 4, 8, 12, 16])
def test_edge_lengths_and_groups(q_dtype, kv_dtype, B, G):
    Hkv = 2
    D = 128
    w = wl.independent_sequences(f"edge-{q_dtype}-{kv_dtype}-{B}-{G}", 100 + B + G, len(EDGE_LENS), Hkv * G,
                                 Hkv, D, B, 600, q_dtype, kv_dtype, EDGE_LENS)
    for ps in (0, 64 if B == 16 else 128, 512):
        g = H.gpu_step(w, partition_size=ps, keep_pools=False)
        o = H.oracle_step(w)
        assert g["err"] == 0
        ok, rep = attention_close(g["out"], o["out"], w.kv_dtype, w.q_dtype)
        assert ok, (ps, rep)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("B", [16, 32])
def test_head_dim_64(dtype, B):
    w = wl.independent_sequences("d64", 7, 6, 8, 4, 64, B, 200, dtype, dtype, [1, 40, B, 300, 700, 1000])
    check_step(w)


def test_zero_length_sequences_give_zero():
    w = wl.independent_sequences("zero", 8, 4, 8, 2, 128, 16, 100, "f16", "f16", [5, 30, 7, 70])
    lens = w.context_lens.copy()
    lens[[1, 3]] = 0
    g = H.gpu_step(w, context_lens=lens, keep_pools=False)
    o = H.oracle_step(w, context_lens=lens)
    assert g["err"] == 0
    assert not g["out"][[1, 3]].any()
    ok, rep = attention_close(g["out"], o["out"], "f16", "f16")
    assert ok, rep


def test_bad_block_id_flags_and_poisons_only_that_sequence():
    from paged_kv_cache_324_b200.binding import DEVERR_BLOCK_ID
    w = wl.independent_sequences("badid", 9, 4, 8, 2, 128, 16, 300, "f16", "f16", [100, 900, 40, 600])
    tab = w.block_tables.copy()
    tab[1, 20] = w.num_blocks + 7
    g = H.gpu_step(w, block_tables=tab, keep_pools=False)
    o = H.oracle_step(w)
    assert g["err"] & DEVERR_BLOCK_ID
    assert np.isnan(g["out"][1]).all()
    keep = [0, 2, 3]
    ok, rep = attention_close(g["out"][keep], o["out"][keep], "f16", "f16")
    assert ok, rep


def test_bad_context_len_flags_and_poisons():
    from paged_kv_cache_324_b200.binding import DEVERR_CONTEXT_LEN
    w = wl.independent_sequences("badlen", 10, 3, 4, 4, 128, 16, 200, "bf16", "bf16", [50, 60, 70])
    lens = w.context_lens.copy()
    lens[2] = w.max_blocks * 16 + 5          # beyond the table's capacity
    g = H.gpu_step(w, context_lens=lens, max_context_len=int(lens.max()), keep_pools=False)
    assert g["err"] & DEVERR_CONTEXT_LEN
    assert np.isnan(g["out"][2]).all() and np.isfinite(g["out"][:2]).all()


def test_reshape_bad_slot_is_skipped_and_flagged():
    from paged_kv_cache_324_b200 import binding as B
    from paged_kv_cache_324_b200.binding import DEVERR_SLOT
    import oracle
    rng = np.random.default_rng(12)
    NB, Hkv, Bs, D, T = 20, 2, 16, 128, 12
    kp0 = wl.garbage_bytes(rng, NB * Hkv * Bs * D * 2).view(np.uint16).reshape(NB, Hkv, Bs, D)
    k = wl.normal_bits(rng, (T, Hkv, D), "f16")
    v = wl.normal_bits(rng, (T, Hkv, D), "f16")
    slots = rng.choice(NB * Bs, size=T, replace=False).astype(np.int64)
    slots[3] = NB * Bs + 4
    slots[5] = -1
    dev = torch.device("cuda:0")
    kp = H.to_dev_bits(kp0, "f16", dev)
    vp = H.to_dev_bits(kp0, "f16", dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    B.reshape_and_cache(H.to_dev_bits(k, "f16", dev), H.to_dev_bits(v, "f16", dev), kp, vp,
                        torch.from_numpy(slots).to(dev), device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & DEVERR_SLOT
    ok_slots = slots.copy()
    ok_slots[3] = -1
    ko, vo = kp0.copy(), kp0.copy()
    oracle.reshape_and_cache(k, v, "f16", ko, vo, "f16", ok_slots)
    assert np.array_equal(H.to_host_bits(kp), ko) and np.array_equal(H.to_host_bits(vp), vo)


def test_copy_blocks_bad_pair_is_skipped_and_flagged():
    from paged_kv_cache_324_b200 import binding as B
    from paged_kv_cache_324_b200.binding import DEVERR_PAIR
    import oracle
    rng = np.random.default_rng(13)
    kp0 = wl.garbage_bytes(rng, 30 * 4 * 16 * 128).view(np.uint8).reshape(30, 4, 16, 128)
    vp0 = wl.garbage_bytes(rng, 30 * 4 * 16 * 128).view(np.uint8).reshape(30, 4, 16, 128)
    pairs = np.array([[1, 2], [3, 40], [5, 6], [-1, 7], [8, 9]], np.int64)
    dev = torch.device("cuda:0")
    kp, vp = torch.from_numpy(kp0).to(dev), torch.from_numpy(vp0).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    B.copy_blocks(kp, vp, torch.from_numpy(pairs).to(dev), device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & DEVERR_PAIR
    ko, vo = kp0.copy(), vp0.copy()
    oracle.copy_blocks(ko, vo, pairs[[0, 2, 4]])
    assert np.array_equal(kp.cpu().numpy(), ko) and np.array_equal(vp.cpu().numpy(), vo)


def test_gpu_output_fails_against_mutated_oracle():
    """Negative controls: the comparison catches a dropped block, an off-by-one mask and a
    foreign block (mistakes planted in the oracle's inputs, on the CPU)."""
    w = wl.make("opt13b", small=True)
    g = H.gpu_step(w, keep_pools=False)
    lens = w.context_lens
    s = int(np.argmax(lens))
    off = lens.copy()
    off[s] -= 1
    drop = lens.copy()
    drop[s] -= (lens[s] - 1) % w.block_size + 1
    other = w.block_tables.copy()
    other[s, 0] = other[(s + 1) % w.num_seqs, 0]
    for what, kw in {"off_by_one": dict(context_lens=off), "drop_last_block": dict(context_lens=drop),
                     "foreign_block": dict(block_tables=other)}.items():
        bad = H.oracle_step(w, **kw)["out"]
        assert not attention_close(g["out"], bad, w.kv_dtype, w.q_dtype)[0], what


@pytest.mark.parametrize("name", ["tiny", "opt13b", "gqa", "prefix", "fp8", "fp8_b32"])
def test_full_size_workload(name):
    """The five workloads at full size, in the launch configuration the benchmark times
    (the workload's stated partition size, else the automatic one)."""
    w = wl.make(name)
    g, o, rep = check_step(w)
    print(name, rep)


def test_full_size_fp8_automatic_partitions():
    """The long-context FP8 workload with the automatic (2,048-token) partitions as well."""
    w = wl.make("fp8")
    g, o, rep = check_step(w, partition_size=0, pools=False)
    print("fp8 auto", rep)
