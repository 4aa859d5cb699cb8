"""pkv_paged_attn_decode_static_ws, the decode call that allocates nothing.

Some callers cannot allocate device memory: code hosted by a framework that
owns every allocation on the GPU, or a serving loop that must not allocate
once it runs because cudaMalloc can synchronise the device.  For them the
library keeps the split-context workspace in a device array of its own.
This test calls that entry point through the C ABI, twice in a row on
different workloads that both need the workspace, and checks each result
against the float64 oracle and against the ordinary entry point (given a
caller-allocated workspace) with the comparison rule the other parity tests
use.  It lives in a file that pytest collects last, so a run that stops at
the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from paged_kv_cache_324_b200 import binding as B
from paged_kv_cache_324_b200 import workload as wl
from tests import harness as H
from tests.parity import attention_close

pytestmark = pytest.mark.gpu

CODES = {"f16": B.F16, "bf16": B.BF16, "e4m3": B.FP8_E4M3}
STATIC_WS_BYTES = 64 << 20


def static_entry():
    f = B.lib().pkv_paged_attn_decode_static_ws
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    f.argtypes = [P, P, I, P, P, I, F, F, P, I, P, I, I, I, I, I, I, I, F, I, P, P]
    f.restype = I
    return f


def device_inputs(w, dev):
    """Pools after the workload's setup and step scatter (library kernels), plus q, tables, lengths."""
    kp = H.to_dev_bits(w.initial_pool("k"), w.kv_dtype, dev)
    vp = H.to_dev_bits(w.initial_pool("v"), w.kv_dtype, dev)
    for op in list(w.setup) + ([w.step_copy] if w.step_copy is not None else []) + [w.step_scatter]:
        if isinstance(op, wl.Scatter):
            B.reshape_and_cache(H.to_dev_bits(op.k, w.src_dtype, dev), H.to_dev_bits(op.v, w.src_dtype, dev),
                                kp, vp, torch.from_numpy(op.slots).to(dev), float(w.k_scale), float(w.v_scale))
        else:
            B.copy_blocks(kp, vp, torch.from_numpy(op.pairs).to(dev))
    return dict(q=H.to_dev_bits(w.q, w.q_dtype, dev), kp=kp, vp=vp,
                tables=torch.from_numpy(w.block_tables).to(dev), lens=torch.from_numpy(w.context_lens).to(dev))


def call_static(f, w, t, out, err, partition_size):
    stream = torch.cuda.current_stream().cuda_stream
    return f(out.data_ptr(), t["q"].data_ptr(), CODES[w.q_dtype], t["kp"].data_ptr(), t["vp"].data_ptr(),
             CODES[w.kv_dtype], float(w.k_scale), float(w.v_scale), t["tables"].data_ptr(), w.max_blocks,
             t["lens"].data_ptr(), w.max_context_len, w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim,
             w.block_size, w.num_blocks, float(w.scale), partition_size, err.data_ptr(), stream)


def test_static_workspace_matches_caller_workspace_on_two_calls():
    dev = torch.device("cuda:0")
    f = static_entry()
    cases = [(wl.make("gqa", small=True), 64), (wl.make("fp8", small=True), 512)]
    for w, ps in cases:
        need = B.decode_workspace_bytes(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.kv_dtype, w.block_size,
                                        w.max_context_len, ps)
        assert 0 < need <= STATIC_WS_BYTES      # the workspace is really used
    for w, ps in cases:                          # two calls in a row, each checked
        t = device_inputs(w, dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        ref = torch.empty_like(t["q"])
        B.paged_attn_decode(ref, t["q"], t["kp"], t["vp"], t["tables"], t["lens"], float(w.scale),
                            max_context_len=w.max_context_len, k_scale=float(w.k_scale),
                            v_scale=float(w.v_scale), partition_size=ps, device_error=err)
        out = torch.full_like(t["q"], float("nan"))
        assert call_static(f, w, t, out, err, ps) == 0
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        ok, rep = attention_close(H.out_f64(out), H.oracle_step(w)["out"], w.kv_dtype, w.q_dtype)
        assert ok, (w.name, "against the oracle", rep)
        ok, rep = attention_close(H.out_f64(out), H.out_f64(ref), w.kv_dtype, w.q_dtype)
        assert ok, (w.name, "against the ordinary entry point", rep)


def test_static_workspace_rejects_oversized_requests():
    dev = torch.device("cuda:0")
    f = static_entry()
    w = wl.make("tiny")
    t = device_inputs(w, dev)
    out = torch.zeros_like(t["q"])
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    # claim a context long enough that the workspace would exceed the library's array
    big_len, ps = 1 << 22, w.block_size
    assert B.decode_workspace_bytes(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.kv_dtype, w.block_size,
                                    big_len, ps) > STATIC_WS_BYTES
    stream = torch.cuda.current_stream().cuda_stream
    status = f(out.data_ptr(), t["q"].data_ptr(), CODES[w.q_dtype], t["kp"].data_ptr(), t["vp"].data_ptr(),
               CODES[w.kv_dtype], 1.0, 1.0, t["tables"].data_ptr(), w.max_blocks, t["lens"].data_ptr(),
               big_len, w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.block_size, w.num_blocks,
               float(w.scale), ps, err.data_ptr(), stream)
    assert status == 3                          # PKV_ERR_WORKSPACE, nothing launched
    torch.cuda.synchronize()
    assert not out.any() and int(err.item()) == 0
