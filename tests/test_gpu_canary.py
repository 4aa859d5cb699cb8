"""Canary-guarded buffers: every buffer a kernel writes (pools, outputs, workspaces,
the error word) sits between guard bytes, and after the calls the guards must be
unchanged.  This stands in for a memory checker: it catches writes just outside
a buffer, which the bit-for-bit pool comparisons (inside the buffers) cannot see.
Decode steps on four small workloads, both prefills, and the memory kernels at
the first and last block and slot of a pool are covered; results are also checked
against the oracle.
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

TORCH = {"f16": torch.float16, "bf16": torch.bfloat16, "e4m3": torch.uint8}


def guarded_bits(bits, dtype, dev):
    return H.Guarded(bits.shape, TORCH[dtype], dev, init=H.to_dev_bits(bits, dtype, dev))


def error_word(dev):
    return H.Guarded((1,), torch.int32, dev, init=torch.zeros(1, dtype=torch.int32, device=dev))


@pytest.mark.parametrize("name", ["tiny", "gqa", "prefix", "fp8"])
def test_decode_step_writes_nothing_outside_its_buffers(name):
    dev = torch.device("cuda:0")
    w = wl.make(name, small=True)
    kp = guarded_bits(w.initial_pool("k"), w.kv_dtype, dev)
    vp = guarded_bits(w.initial_pool("v"), w.kv_dtype, dev)
    err = error_word(dev)
    ops = list(w.setup) + ([w.step_copy] if w.step_copy is not None else []) + [w.step_scatter]
    for op in ops:
        if isinstance(op, wl.Scatter):
            B.reshape_and_cache(H.to_dev_bits(op.k, w.src_dtype, dev), H.to_dev_bits(op.v, w.src_dtype, dev),
                                kp.t, vp.t, torch.from_numpy(op.slots).to(dev), float(w.k_scale), float(w.v_scale),
                                device_error=err.t)
        else:
            B.copy_blocks(kp.t, vp.t, torch.from_numpy(op.pairs).to(dev), device_error=err.t)
    q = H.to_dev_bits(w.q, w.q_dtype, dev)
    out = H.Guarded(q.shape, q.dtype, dev)
    need = B.decode_workspace_bytes(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.kv_dtype, w.block_size,
                                    w.max_context_len, w.partition_size)
    ws = H.Guarded((max(need, 256),), torch.uint8, dev)
    B.paged_attn_decode(out.t, q, kp.t, vp.t, torch.from_numpy(w.block_tables).to(dev),
                        torch.from_numpy(w.context_lens).to(dev), float(w.scale), max_context_len=w.max_context_len,
                        k_scale=float(w.k_scale), v_scale=float(w.v_scale), partition_size=w.partition_size,
                        workspace=ws.t, device_error=err.t)
    torch.cuda.synchronize()
    assert int(err.t.item()) == 0
    for g, what in ((kp, "k_pool"), (vp, "v_pool"), (out, "out"), (ws, "workspace"), (err, "device_error")):
        assert g.intact(), f"a write outside {what}"
    ref = H.oracle_step(w)
    assert np.array_equal(H.to_host_bits(kp.t), ref["k_pool"]) and np.array_equal(H.to_host_bits(vp.t), ref["v_pool"])
    ok, rep = attention_close(H.out_f64(out.t), ref["out"], w.kv_dtype, w.q_dtype)
    assert ok, rep


@pytest.mark.parametrize("fp8", [False, True])
def test_prefill_writes_nothing_outside_its_buffers(fp8):
    dev = torch.device("cuda:0")
    w = wl.make_prefill(small=True)
    ops = [op for op in list(w.setup) + [w.step_scatter] if op.slots.size]
    if fp8:
        ks = float(max(wl.amax_scale(op.k, w.dtype) for op in ops))
        vs = float(max(wl.amax_scale(op.v, w.dtype) for op in ops))
        rng = np.random.default_rng(8)
        n = int(np.prod(w.pool_shape))
        kp = guarded_bits(wl.garbage_bytes(rng, n).reshape(w.pool_shape), "e4m3", dev)
        vp = guarded_bits(wl.garbage_bytes(rng, n).reshape(w.pool_shape), "e4m3", dev)
    else:
        ks = vs = 1.0
        kp = guarded_bits(w.initial_pool("k"), w.dtype, dev)
        vp = guarded_bits(w.initial_pool("v"), w.dtype, dev)
    err = error_word(dev)
    for op in ops:
        B.reshape_and_cache(H.to_dev_bits(op.k, w.dtype, dev), H.to_dev_bits(op.v, w.dtype, dev), kp.t, vp.t,
                            torch.from_numpy(op.slots).to(dev), ks, vs, device_error=err.t)
    q = H.to_dev_bits(w.q, w.dtype, dev)
    out = H.Guarded(q.shape, q.dtype, dev)
    tables = torch.from_numpy(w.block_tables).to(dev)
    lens = torch.from_numpy(w.context_lens).to(dev)
    qs = torch.from_numpy(w.query_start).to(dev)
    guards = [(kp, "k_pool"), (vp, "v_pool"), (out, "out"), (err, "device_error")]
    if fp8:
        need = B.prefill_fp8_workspace_bytes(w.num_seqs, w.max_blocks, w.num_kv_heads, w.head_dim, w.block_size)
        ws = H.Guarded((need,), torch.uint8, dev)
        guards.append((ws, "workspace"))
        B.paged_attn_prefill_fp8(out.t, q, kp.t, vp.t, tables, lens, qs, float(w.scale), ks, vs,
                                 max_query_len=w.max_query_len, workspace=ws.t, device_error=err.t)
    else:   # bf16: V is narrowed to f16 in the workspace first
        need = B.prefill_workspace_bytes(w.dtype, w.num_seqs, w.max_blocks, w.num_kv_heads, w.head_dim, w.block_size)
        assert need > 0
        ws = H.Guarded((need,), torch.uint8, dev)
        guards.append((ws, "workspace"))
        B.paged_attn_prefill(out.t, q, kp.t, vp.t, tables, lens, qs, float(w.scale), max_query_len=w.max_query_len,
                             workspace=ws.t, device_error=err.t)
    torch.cuda.synchronize()
    assert int(err.t.item()) == 0
    for g, what in guards:
        assert g.intact(), f"a write outside {what}"
    assert bool(torch.isfinite(out.t).all())


def test_memory_kernels_write_nothing_outside_their_buffers():
    """Scatter into the first and last slot of a pool (16-bit and E4M3), copy-on-write into the
    first and last block, swap out to pinned host memory and back into the first and last block;
    the pools end bit-identical to the oracle's after the same operations."""
    dev = torch.device("cuda:0")
    NB, Hkv, Bs, D = 32, 2, 16, 128
    shape = (NB, Hkv, Bs, D)
    rng = np.random.default_rng(3)
    k16, v16 = wl.normal_bits(rng, shape, "f16"), wl.normal_bits(rng, shape, "f16")
    kp, vp = guarded_bits(k16, "f16", dev), guarded_bits(v16, "f16", dev)
    kq = guarded_bits(np.zeros(shape, np.uint8), "e4m3", dev)
    vq = guarded_bits(np.zeros(shape, np.uint8), "e4m3", dev)
    err = error_word(dev)
    kn, vn = wl.normal_bits(rng, (3, Hkv, D), "f16"), wl.normal_bits(rng, (3, Hkv, D), "f16")
    slots = np.array([0, NB * Bs - 1, -1], np.int64)
    B.reshape_and_cache(H.to_dev_bits(kn, "f16", dev), H.to_dev_bits(vn, "f16", dev), kp.t, vp.t,
                        torch.from_numpy(slots).to(dev), device_error=err.t)
    B.reshape_and_cache(H.to_dev_bits(kn, "f16", dev), H.to_dev_bits(vn, "f16", dev), kq.t, vq.t,
                        torch.from_numpy(slots).to(dev), 0.05, 0.05, device_error=err.t)
    cow = np.array([[5, 0], [6, NB - 1]], np.int64)
    B.copy_blocks(kp.t, vp.t, torch.from_numpy(cow).to(dev), device_error=err.t)
    hk = torch.zeros(shape, dtype=torch.float16).pin_memory()
    hv = torch.zeros(shape, dtype=torch.float16).pin_memory()
    out_pairs = np.array([[7, 0], [8, 1]], np.int64)
    in_pairs = np.array([[0, NB - 1], [1, 0]], np.int64)
    B.swap_blocks(kp.t, vp.t, hk, hv, torch.from_numpy(out_pairs).to(dev), device_error=err.t)
    B.swap_blocks(hk, hv, kp.t, vp.t, torch.from_numpy(in_pairs).to(dev), device_error=err.t)
    torch.cuda.synchronize()
    assert int(err.t.item()) == 0
    for g, what in ((kp, "k_pool"), (vp, "v_pool"), (kq, "E4M3 k_pool"), (vq, "E4M3 v_pool"), (err, "device_error")):
        assert g.intact(), f"a write outside {what}"
    ek, ev = k16.copy(), v16.copy()
    oracle.reshape_and_cache(kn, vn, "f16", ek, ev, "f16", slots)
    eqk, eqv = np.zeros(shape, np.uint8), np.zeros(shape, np.uint8)
    oracle.reshape_and_cache(kn, vn, "f16", eqk, eqv, "e4m3", slots, 0.05, 0.05)
    oracle.copy_blocks(ek, ev, cow)
    hk_ref, hv_ref = np.zeros_like(ek), np.zeros_like(ev)
    oracle.swap_blocks(ek, ev, hk_ref, hv_ref, out_pairs)
    oracle.swap_blocks(hk_ref, hv_ref, ek, ev, in_pairs)
    assert np.array_equal(H.to_host_bits(kp.t), ek) and np.array_equal(H.to_host_bits(vp.t), ev)
    assert np.array_equal(H.to_host_bits(kq.t), eqk) and np.array_equal(H.to_host_bits(vq.t), eqv)
