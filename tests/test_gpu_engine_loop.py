"""A decode loop driven by the library's block manager, on the GPU, against the oracle.

Prompts are written token by token, then forked into parallel samples (shared
blocks, reference counts); every step appends one token per live sequence,
applies the copy-on-write pairs the manager returns (copy_blocks), scatters the
new K/V (reshape_and_cache) and runs paged attention.  Sequences finish midway
so their blocks return to the free list and are reused.  The oracle replays the
same operations on the host; pools and outputs are compared.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_324_b200 import binding as B
from paged_kv_cache_324_b200 import workload as wl
from tests import harness as H
from tests.parity import attention_close

pytestmark = pytest.mark.gpu


def test_block_manager_driven_decode_loop():
    rng = np.random.default_rng(21)
    NB, BS, H_, Hkv, D = 600, 16, 8, 2, 128
    dev = torch.device("cuda:0")
    bm = B.BlockManager(NB, BS, rng.permutation(NB))
    kp_h = wl.garbage_bytes(rng, NB * Hkv * BS * D * 2).view(np.uint16).reshape(NB, Hkv, BS, D)
    vp_h = wl.garbage_bytes(rng, NB * Hkv * BS * D * 2).view(np.uint16).reshape(NB, Hkv, BS, D)
    kp, vp = H.to_dev_bits(kp_h, "f16", dev), H.to_dev_bits(vp_h, "f16", dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(ids):
        slots, pairs = bm.append_slots(ids)
        k = wl.normal_bits(rng, (len(ids), Hkv, D), "f16")
        v = wl.normal_bits(rng, (len(ids), Hkv, D), "f16")
        if len(pairs):
            B.copy_blocks(kp, vp, torch.from_numpy(pairs).to(dev), device_error=err)
            oracle.copy_blocks(kp_h, vp_h, pairs)
        B.reshape_and_cache(H.to_dev_bits(k, "f16", dev), H.to_dev_bits(v, "f16", dev), kp, vp,
                            torch.from_numpy(slots).to(dev), device_error=err)
        oracle.reshape_and_cache(k, v, "f16", kp_h, vp_h, "f16", slots)
        return len(pairs)

    prompts = [0, 1, 2, 3]
    plens = rng.integers(20, 100, size=4)
    for s in prompts:
        bm.add_sequence(s)
    for t in range(int(plens.max())):
        live = [s for s in prompts if t < plens[s]]
        step(live)
    live = list(prompts)
    nxt = 4
    for s in prompts:                                   # three more samples per prompt
        for _ in range(3):
            bm.fork(s, nxt)
            live.append(nxt)
            nxt += 1
    copies = 0
    for it in range(30):
        if it == 12:                                    # two samples finish; their blocks return
            for s in (5, 9):
                bm.free_sequence(s)
                live.remove(s)
        copies += step(live)
        if it % 10 == 9 or it == 29:
            tables, lens = bm.block_tables(live, 16, pad=int(wl.TABLE_POISON))
            q = wl.normal_bits(rng, (len(live), H_, D), "f16")
            out = torch.empty((len(live), H_, D), dtype=torch.float16, device=dev)
            B.paged_attn_decode(out, H.to_dev_bits(q, "f16", dev), kp, vp, torch.from_numpy(tables).to(dev),
                                torch.from_numpy(lens).to(dev), 1 / np.sqrt(D), max_context_len=int(lens.max()),
                                device_error=err)
            torch.cuda.synchronize()
            ref = oracle.paged_attn_decode(q, "f16", kp_h, vp_h, "f16", tables, lens, np.float32(1 / np.sqrt(D)))
            ok, rep = attention_close(H.out_f64(out), ref, "f16", "f16")
            assert ok, (it, rep)
    assert int(err.item()) == 0
    # each prompt with a partially filled last block: 3 of its 4 holders copied it
    assert copies == 3 * int((plens % BS != 0).sum())
    assert np.array_equal(H.to_host_bits(kp), kp_h) and np.array_equal(H.to_host_bits(vp), vp_h)
