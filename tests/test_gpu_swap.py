"""Block swap between the GPU pools and pinned host memory, and prefix caching, on the GPU.

- pkv_swap_blocks moves blocks GPU -> pinned host -> GPU bit for bit (against the
  oracle's block swap), leaves every other block alone, and refuses pageable host
  memory before launching anything.
- Preemption by swapping inside a decode loop driven by the library's block
  managers (one for the GPU pool, one for the host pool): a group of sequences is
  swapped out, the freed GPU blocks are reused by the sequences still running,
  the group is swapped back into other blocks, and its attention output is bit
  for bit what it was before (the kernel does not depend on physical block ids).
- A request whose prompt shares leading blocks with a cached one starts from the
  cached blocks, prefills only the rest, and gets the output of a from-scratch
  prefill of its whole prompt (oracle on private blocks).
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_324_b200 import binding as B
from paged_kv_cache_324_b200 import workload as wl
from tests import harness as H
from tests.parity import attention_close, prefill_close

pytestmark = pytest.mark.gpu


def test_swap_blocks_round_trip_through_pinned_host_memory():
    rng = np.random.default_rng(80)
    dev = torch.device("cuda:0")
    NB, NH, Hkv, Bs, D = 64, 24, 8, 16, 128
    gk = wl.garbage_bytes(rng, NB * Hkv * Bs * D * 2).view(np.uint16).reshape(NB, Hkv, Bs, D)
    gv = wl.garbage_bytes(rng, gk.nbytes).view(np.uint16).reshape(gk.shape)
    hk = wl.garbage_bytes(rng, NH * gk[0].nbytes).view(np.uint16).reshape(NH, Hkv, Bs, D)
    hv = wl.garbage_bytes(rng, hk.nbytes).view(np.uint16).reshape(hk.shape)
    dgk, dgv = H.to_dev_bits(gk, "f16", dev), H.to_dev_bits(gv, "f16", dev)
    phk = torch.from_numpy(hk.view(np.int16).copy()).view(torch.float16).pin_memory()
    phv = torch.from_numpy(hv.view(np.int16).copy()).view(torch.float16).pin_memory()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    out = np.stack([rng.choice(NB, 20, replace=False), rng.choice(NH, 20, replace=False)], axis=1)
    B.swap_blocks(dgk, dgv, phk, phv, torch.from_numpy(out).to(dev), device_error=err)
    torch.cuda.synchronize()
    oracle.swap_blocks(gk, gv, hk, hv, out)
    assert np.array_equal(phk.view(torch.int16).numpy().view(np.uint16), hk)
    assert np.array_equal(phv.view(torch.int16).numpy().view(np.uint16), hv)
    # back into other GPU blocks (the old ones are considered reused)
    back = np.stack([out[:, 1], rng.permutation(NB)[:20]], axis=1)
    B.swap_blocks(phk, phv, dgk, dgv, torch.from_numpy(back).to(dev), device_error=err)
    torch.cuda.synchronize()
    oracle.swap_blocks(hk, hv, gk, gv, back)
    assert np.array_equal(H.to_host_bits(dgk), gk) and np.array_equal(H.to_host_bits(dgv), gv)
    assert int(err.item()) == 0
    # a pair outside the destination pool is skipped and flagged
    bad = torch.tensor([[0, NH + 3]], dtype=torch.int64, device=dev)
    B.swap_blocks(dgk, dgv, phk, phv, bad, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & 0x4
    assert np.array_equal(phk.view(torch.int16).numpy().view(np.uint16), hk)


def test_swap_refuses_pageable_host_memory():
    dev = torch.device("cuda:0")
    g = torch.zeros((4, 1, 16, 8), dtype=torch.float16, device=dev)
    pageable = torch.zeros((4, 1, 16, 8), dtype=torch.float16)          # not pinned
    pairs = torch.tensor([[0, 1]], dtype=torch.int64, device=dev)
    P = ctypes.c_void_p
    st = B.lib().pkv_swap_blocks(P(g.data_ptr()), P(g.data_ptr()), 4, P(pageable.data_ptr()),
                                 P(pageable.data_ptr()), 4, g[0].numel() * 2, P(pairs.data_ptr()), 1, None, None)
    assert st == 1
    with pytest.raises(ValueError):
        B.swap_blocks(g, g, pageable, pageable, pairs)


def test_preemption_by_swap_gives_identical_attention():
    rng = np.random.default_rng(81)
    dev = torch.device("cuda:0")
    NB, NH, Bs, H_, Hkv, D = 160, 96, 16, 8, 2, 128
    gpu = B.BlockManager(NB, Bs, rng.permutation(NB))
    host = B.BlockManager(NH, Bs)
    kp = H.to_dev_bits(wl.garbage_bytes(rng, NB * Hkv * Bs * D * 2).view(np.uint16).reshape(NB, Hkv, Bs, D), "bf16", dev)
    vp = H.to_dev_bits(wl.garbage_bytes(rng, NB * Hkv * Bs * D * 2).view(np.uint16).reshape(NB, Hkv, Bs, D), "bf16", dev)
    hk = torch.empty((NH, Hkv, Bs, D), dtype=torch.bfloat16).pin_memory()
    hv = torch.empty((NH, Hkv, Bs, D), dtype=torch.bfloat16).pin_memory()
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(ids):
        slots, pairs = gpu.append_slots(ids)
        if len(pairs):
            B.copy_blocks(kp, vp, torch.from_numpy(pairs).to(dev), device_error=err)
        k = H.to_dev_bits(wl.normal_bits(rng, (len(ids), Hkv, D), "bf16"), "bf16", dev)
        v = H.to_dev_bits(wl.normal_bits(rng, (len(ids), Hkv, D), "bf16"), "bf16", dev)
        B.reshape_and_cache(k, v, kp, vp, torch.from_numpy(slots).to(dev), device_error=err)

    def decode(ids, q):
        tables, lens = gpu.block_tables(ids, 32, pad=int(wl.TABLE_POISON))
        out = torch.empty_like(q)
        B.paged_attn_decode(out, q, kp, vp, torch.from_numpy(tables).to(dev), torch.from_numpy(lens).to(dev),
                            1 / np.sqrt(D), max_context_len=int(lens.max()), device_error=err)
        torch.cuda.synchronize()
        return out.clone()

    for s in range(4):
        gpu.add_sequence(s)
    for t in range(150):
        step([s for s in range(4) if t < 60 + 30 * s])
    for s in range(4):                                    # two samples per prompt share its blocks
        gpu.fork(s, 10 + s)
    for _ in range(20):
        step(list(range(4)) + [10 + s for s in range(4)])
    group = [1, 11, 3, 13]
    q = H.to_dev_bits(wl.normal_bits(rng, (4, H_, D), "bf16"), "bf16", dev)
    before = decode(group, q)
    pairs = gpu.swap_to(host, group)
    B.swap_blocks(kp, vp, hk, hv, torch.from_numpy(pairs).to(dev), device_error=err)
    for _ in range(60):                                   # the others run on, reusing the freed blocks
        step([0, 10, 2, 12])
    back = host.swap_to(gpu, group)
    B.swap_blocks(hk, hv, kp, vp, torch.from_numpy(back).to(dev), device_error=err)
    after = decode(group, q)
    assert int(err.item()) == 0
    assert torch.equal(before.view(torch.int16), after.view(torch.int16))
    tables, lens = gpu.block_tables(group, 32, pad=int(wl.TABLE_POISON))
    assert host.num_free == NH


def test_prefix_cache_hit_then_partial_prefill_equals_full_prefill():
    rng = np.random.default_rng(82)
    dev = torch.device("cuda:0")
    NB, Bs, H_, Hkv, D, V = 64, 16, 8, 2, 128, 50
    # K/V of a token are a fixed function of (token id, position), as a model's would be
    ktab = wl.normal_bits(rng, (V, 128, Hkv, D), "bf16")
    vtab = wl.normal_bits(rng, (V, 128, Hkv, D), "bf16")
    a = rng.integers(0, V, size=100)
    b = np.concatenate([a[:70], rng.integers(0, V, size=20)])
    m = B.BlockManager(NB, Bs, rng.permutation(NB))
    kp_h = wl.garbage_bytes(rng, NB * Hkv * Bs * D * 2).view(np.uint16).reshape(NB, Hkv, Bs, D)
    vp_h = wl.garbage_bytes(rng, kp_h.nbytes).view(np.uint16).reshape(kp_h.shape)
    kp, vp = H.to_dev_bits(kp_h, "bf16", dev), H.to_dev_bits(vp_h, "bf16", dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def write(seq, toks, start):
        slots = np.array([int(m.append_slots([seq])[0][0]) for _ in range(start, len(toks))], np.int64)
        pos = np.arange(start, len(toks))
        B.reshape_and_cache(H.to_dev_bits(np.ascontiguousarray(ktab[toks[start:], pos]), "bf16", dev),
                            H.to_dev_bits(np.ascontiguousarray(vtab[toks[start:], pos]), "bf16", dev), kp, vp,
                            torch.from_numpy(slots).to(dev), device_error=err)

    assert m.add_sequence_cached(0, a) == 0
    write(0, a, 0)
    m.cache_sequence(0, a)
    got = m.add_sequence_cached(1, b)
    assert got == 64                                              # four full blocks of the 70 shared tokens
    write(1, b, got)
    ta, _ = m.block_tables([0], 8)
    tb, lb = m.block_tables([1], 8)
    assert tb[0, :4].tolist() == ta[0, :4].tolist() and lb[0] == len(b)
    C = len(b) - got
    q = wl.normal_bits(rng, (C, H_, D), "bf16")
    out = torch.empty((C, H_, D), dtype=torch.bfloat16, device=dev)
    B.paged_attn_prefill(out, H.to_dev_bits(q, "bf16", dev), kp, vp, torch.from_numpy(tb).to(dev),
                         torch.from_numpy(lb).to(dev), torch.tensor([0, C], dtype=torch.int32, device=dev),
                         1 / np.sqrt(D), max_query_len=C, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    # reference: the whole prompt b written to private blocks of a fresh pool, prefilled by the oracle
    nblk = -(-len(b) // Bs)
    fk = np.zeros((nblk, Hkv, Bs, D), np.uint16)
    fv = np.zeros_like(fk)
    pos = np.arange(len(b))
    oracle.reshape_and_cache(np.ascontiguousarray(ktab[b, pos]), np.ascontiguousarray(vtab[b, pos]), "bf16", fk, fv,
                             "bf16", pos.astype(np.int64))
    ref = oracle.paged_attn_prefill(q, "bf16", fk, fv, "bf16", np.arange(nblk, dtype=np.int32)[None],
                                    np.array([len(b)], np.int32), np.array([0, C], np.int32), np.float32(1 / np.sqrt(D)))
    ok, rep = prefill_close(H.out_f64(out), ref, "bf16")
    assert ok, rep
