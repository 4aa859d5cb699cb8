"""The decode step and the chunked prefill captured in CUDA graphs and replayed.

A serving loop replays one graph per step instead of launching each kernel: the
library's launches (programmatic-dependent-launch attributes, tensor maps passed
by value, a caller-provided workspace) must be capturable, and every replay must
read the inputs copied into the graph's static buffers.  Each replay is checked
against the oracle on that replay's inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_324_b200 import binding as B
from paged_kv_cache_324_b200 import workload as wl
from tests import harness as H
from tests.parity import attention_close, prefill_close

pytestmark = pytest.mark.gpu


def _bits_to(dst: torch.Tensor, bits: np.ndarray):
    dst.view(torch.int16).copy_(torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)))


def test_decode_step_graph_replays_with_new_inputs():
    dev = torch.device("cuda:0")
    w = wl.make("gqa", small=True)
    rng = np.random.default_rng(90)
    kp_h, vp_h = w.initial_pool("k"), w.initial_pool("v")
    kp, vp = H.to_dev_bits(kp_h, w.kv_dtype, dev), H.to_dev_bits(vp_h, w.kv_dtype, dev)
    for op in w.setup:
        B.reshape_and_cache(H.to_dev_bits(op.k, w.src_dtype, dev), H.to_dev_bits(op.v, w.src_dtype, dev), kp, vp,
                            torch.from_numpy(op.slots).to(dev))
        oracle.reshape_and_cache(op.k, op.v, w.src_dtype, kp_h, vp_h, w.kv_dtype, op.slots)
    S, Hq, D, Hkv = w.num_seqs, w.num_heads, w.head_dim, w.num_kv_heads
    q = torch.empty((S, Hq, D), dtype=torch.bfloat16, device=dev)
    kn = torch.empty((S, Hkv, D), dtype=torch.bfloat16, device=dev)
    vn = torch.empty_like(kn)
    slots = torch.from_numpy(w.step_scatter.slots).to(dev)
    tables = torch.from_numpy(w.block_tables).to(dev)
    lens = torch.from_numpy(w.context_lens).to(dev)
    out = torch.empty_like(q)
    ws_bytes = B.decode_workspace_bytes(S, Hq, Hkv, D, w.kv_dtype, w.block_size, w.max_context_len, 0)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def step():
        B.reshape_and_cache(kn, vn, kp, vp, slots, device_error=err)
        B.paged_attn_decode(out, q, kp, vp, tables, lens, float(w.scale), max_context_len=w.max_context_len,
                            workspace=ws, device_error=err)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):                     # one eager run before capture
        step()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(3):
        qb = wl.normal_bits(rng, (S, Hq, D), "bf16")
        kb = wl.normal_bits(rng, (S, Hkv, D), "bf16")
        vb = wl.normal_bits(rng, (S, Hkv, D), "bf16")
        _bits_to(q, qb)
        _bits_to(kn, kb)
        _bits_to(vn, vb)
        g.replay()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        oracle.reshape_and_cache(kb, vb, "bf16", kp_h, vp_h, "bf16", w.step_scatter.slots)
        ref = oracle.paged_attn_decode(qb, "bf16", kp_h, vp_h, "bf16", w.block_tables, w.context_lens, w.scale)
        ok, rep = attention_close(H.out_f64(out), ref, "bf16", "bf16")
        assert ok, rep
    assert np.array_equal(H.to_host_bits(kp), kp_h) and np.array_equal(H.to_host_bits(vp), vp_h)


def test_prefill_graph_replays_with_new_inputs():
    dev = torch.device("cuda:0")
    w = wl.make_prefill(small=True)
    rng = np.random.default_rng(91)
    kp_h, vp_h = w.initial_pool("k"), w.initial_pool("v")
    kp, vp = H.to_dev_bits(kp_h, w.dtype, dev), H.to_dev_bits(vp_h, w.dtype, dev)
    for op in w.setup:
        if op.slots.size:
            B.reshape_and_cache(H.to_dev_bits(op.k, w.dtype, dev), H.to_dev_bits(op.v, w.dtype, dev), kp, vp,
                                torch.from_numpy(op.slots).to(dev))
            oracle.reshape_and_cache(op.k, op.v, w.dtype, kp_h, vp_h, w.dtype, op.slots)
    T, Hq, D, Hkv = w.num_tokens, w.num_heads, w.head_dim, w.num_kv_heads
    q = torch.empty((T, Hq, D), dtype=torch.bfloat16, device=dev)
    kn = torch.empty((T, Hkv, D), dtype=torch.bfloat16, device=dev)
    vn = torch.empty_like(kn)
    slots = torch.from_numpy(w.step_scatter.slots).to(dev)
    tables = torch.from_numpy(w.block_tables).to(dev)
    lens = torch.from_numpy(w.context_lens).to(dev)
    qs = torch.from_numpy(w.query_start).to(dev)
    out = torch.empty_like(q)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = torch.empty(B.prefill_workspace_bytes("bf16", w.num_seqs, w.max_blocks, Hkv, D, w.block_size),
                     dtype=torch.uint8, device=dev)

    def step():
        B.reshape_and_cache(kn, vn, kp, vp, slots, device_error=err)
        B.paged_attn_prefill(out, q, kp, vp, tables, lens, qs, float(w.scale), max_query_len=w.max_query_len,
                             workspace=ws, device_error=err)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(2):
        qb = wl.normal_bits(rng, (T, Hq, D), "bf16")
        kb = wl.normal_bits(rng, (T, Hkv, D), "bf16")
        vb = wl.normal_bits(rng, (T, Hkv, D), "bf16")
        _bits_to(q, qb)
        _bits_to(kn, kb)
        _bits_to(vn, vb)
        g.replay()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        oracle.reshape_and_cache(kb, vb, "bf16", kp_h, vp_h, "bf16", w.step_scatter.slots)
        ref = oracle.paged_attn_prefill(qb, "bf16", kp_h, vp_h, "bf16", w.block_tables, w.context_lens,
                                        w.query_start, w.scale)
        ok, rep = prefill_close(H.out_f64(out), ref, "bf16")
        assert ok, rep
