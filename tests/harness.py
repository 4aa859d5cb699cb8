"""Runs one workload's decode step on the GPU (through the binding) and on the
oracle (on the host), from the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

from paged_kv_cache_324_b200 import workload as wl

TORCH16 = {"f16": torch.float16, "bf16": torch.bfloat16}


def to_dev_bits(bits: np.ndarray, dtype: str, dev) -> torch.Tensor:
    """Raw host bits -> device tensor of the named dtype (bit-identical)."""
    if dtype == "e4m3":
        return torch.from_numpy(np.ascontiguousarray(bits)).to(dev)
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev)
    return t.view(TORCH16[dtype])


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.uint8:
        return t.cpu().numpy()
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def out_f64(t: torch.Tensor) -> np.ndarray:
    return t.double().cpu().numpy()


def gpu_step(w: wl.DecodeWorkload, partition_size=None, dev="cuda:0", keep_pools=True,
             block_tables=None, context_lens=None, max_context_len=None):
    from paged_kv_cache_324_b200 import binding as B
    dev = torch.device(dev)
    if partition_size is None:
        partition_size = w.partition_size
    kp = to_dev_bits(w.initial_pool("k"), w.kv_dtype, dev)
    vp = to_dev_bits(w.initial_pool("v"), w.kv_dtype, dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def scatter(op):
        B.reshape_and_cache(to_dev_bits(op.k, w.src_dtype, dev), to_dev_bits(op.v, w.src_dtype, dev),
                            kp, vp, torch.from_numpy(op.slots).to(dev), float(w.k_scale), float(w.v_scale),
                            device_error=err)

    def copy(op):
        B.copy_blocks(kp, vp, torch.from_numpy(op.pairs).to(dev), device_error=err)

    for op in w.setup:
        scatter(op) if isinstance(op, wl.Scatter) else copy(op)
    if w.step_copy is not None:
        copy(w.step_copy)
    scatter(w.step_scatter)
    q = to_dev_bits(w.q, w.q_dtype, dev)
    out = torch.empty_like(q)
    bt = w.block_tables if block_tables is None else block_tables
    cl = w.context_lens if context_lens is None else context_lens
    B.paged_attn_decode(out, q, kp, vp, torch.from_numpy(bt).to(dev), torch.from_numpy(cl).to(dev),
                        float(w.scale), max_context_len=w.max_context_len if max_context_len is None else max_context_len,
                        k_scale=float(w.k_scale), v_scale=float(w.v_scale),
                        partition_size=partition_size, device_error=err)
    torch.cuda.synchronize()
    res = {"out": out_f64(out), "err": int(err.item())}
    if keep_pools:
        res["k_pool"], res["v_pool"] = to_host_bits(kp), to_host_bits(vp)
    del kp, vp
    return res


def oracle_pools(w: wl.DecodeWorkload):
    import oracle
    kp, vp = w.initial_pool("k"), w.initial_pool("v")
    for op in w.setup:
        if isinstance(op, wl.Scatter):
            oracle.reshape_and_cache(op.k, op.v, w.src_dtype, kp, vp, w.kv_dtype, op.slots, w.k_scale, w.v_scale)
        else:
            oracle.copy_blocks(kp, vp, op.pairs)
    if w.step_copy is not None:
        oracle.copy_blocks(kp, vp, w.step_copy.pairs)
    sc = w.step_scatter
    oracle.reshape_and_cache(sc.k, sc.v, w.src_dtype, kp, vp, w.kv_dtype, sc.slots, w.k_scale, w.v_scale)
    return kp, vp


def oracle_step(w: wl.DecodeWorkload, block_tables=None, context_lens=None):
    import oracle
    kp, vp = oracle_pools(w)
    out = oracle.paged_attn_decode(w.q, w.q_dtype, kp, vp, w.kv_dtype,
                                   w.block_tables if block_tables is None else block_tables,
                                   w.context_lens if context_lens is None else context_lens,
                                   w.scale, w.k_scale, w.v_scale)
    return {"out": out, "k_pool": kp, "v_pool": vp}


def gpu_prefill(w, dev="cuda:0", block_tables=None, context_lens=None, query_start=None, q_bits=None,
                workspace="auto"):
    """Build the cache (setup scatter), scatter the chunk's K/V, run the prefill; returns
    (out tensor, device error word, k pool, v pool).  workspace: "auto" (bf16: V narrowed to f16
    in a workspace) or None (bf16: the two-part weights, no workspace)."""
    from paged_kv_cache_324_b200 import binding as B
    dev = torch.device(dev)
    kp = to_dev_bits(w.initial_pool("k"), w.dtype, dev)
    vp = to_dev_bits(w.initial_pool("v"), w.dtype, dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for op in list(w.setup) + [w.step_scatter]:
        if op.slots.size:
            B.reshape_and_cache(to_dev_bits(op.k, w.dtype, dev), to_dev_bits(op.v, w.dtype, dev), kp, vp,
                                torch.from_numpy(op.slots).to(dev), device_error=err)
    q = to_dev_bits(w.q if q_bits is None else q_bits, w.dtype, dev)
    out = torch.full_like(q, float("nan"))
    bt = w.block_tables if block_tables is None else block_tables
    cl = w.context_lens if context_lens is None else context_lens
    qs = w.query_start if query_start is None else query_start
    B.paged_attn_prefill(out, q, kp, vp, torch.from_numpy(np.ascontiguousarray(bt)).to(dev),
                         torch.from_numpy(np.ascontiguousarray(cl)).to(dev),
                         torch.from_numpy(np.ascontiguousarray(qs)).to(dev), float(w.scale),
                         max_query_len=w.max_query_len, workspace=workspace, device_error=err)
    torch.cuda.synchronize()
    return out, int(err.item()), kp, vp


def oracle_prefill_pools(w):
    """Host pools after the setup and chunk scatters (oracle arithmetic)."""
    import oracle
    kp, vp = w.initial_pool("k"), w.initial_pool("v")
    for op in list(w.setup) + [w.step_scatter]:
        if op.slots.size:
            oracle.reshape_and_cache(op.k, op.v, w.dtype, kp, vp, w.dtype, op.slots)
    return kp, vp


class Guarded:
    """A buffer with guard bytes on both sides, to catch writes just outside it: the tensor
    ``t`` (shape, dtype) sits between two GUARD-byte runs of PATTERN inside one allocation.
    GUARD is a multiple of 256, so ``t`` keeps the allocation's alignment."""
    GUARD = 4096
    PATTERN = 0xA5

    def __init__(self, shape, dtype, dev, init=None):
        shape = tuple(int(x) for x in shape)
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.n = n
        self.raw = torch.full((self.GUARD + n + self.GUARD,), self.PATTERN, dtype=torch.uint8, device=dev)
        self.t = self.raw[self.GUARD:self.GUARD + n].view(dtype).view(shape)
        if init is not None:
            self.t.copy_(init)

    def intact(self) -> bool:
        g = self.GUARD
        return bool((self.raw[:g] == self.PATTERN).all()) and bool((self.raw[g + self.n:] == self.PATTERN).all())
