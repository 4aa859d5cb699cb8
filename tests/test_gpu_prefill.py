"""Chunked prefill on the GPU (tcgen05 kernel, through the C ABI) against the oracle.

Small cases compare every output row with the float64 oracle: MHA and GQA
groups of 2, 4, 8 and 16, head_dim 64 and 128, blocks of 16 and 32 tokens,
f16 and bf16, whole prompts, chunks after earlier context that start inside a
partially filled block, single-token chunks, empty chunks, chunk lengths that
leave ragged query and key tiles, a long context, and logits wide enough that
the running maximum moves many times.  The full-size workload is checked on
every row.  Data-dependent errors (a bad block id, a chunk longer than its
context) must give NaN rows and the documented error bits while the other
sequences stay correct.  A prefill of one-token chunks must agree with the
decode kernel.  E4M3 caches go through the widening gather and the same
kernel, compared with the oracle on the dequantised cache, a bad block id
included.
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


def oracle_out(w, kp, vp, block_tables=None, context_lens=None, query_start=None, q_bits=None):
    return oracle.paged_attn_prefill(
        w.q if q_bits is None else q_bits, w.dtype, kp, vp, w.dtype,
        w.block_tables if block_tables is None else block_tables,
        w.context_lens if context_lens is None else context_lens,
        w.query_start if query_start is None else query_start, w.scale)


CASES = {
    # name: (H, Hkv, D, B, dtype, prior, chunks, NB)
    "small_workload": None,
    "mha_f16": (4, 4, 128, 16, "f16", [0, 130, 5], [300, 1, 64], 256),
    "g8_b32_bf16": (16, 2, 128, 32, "bf16", [1000, 0], [150, 33], 256),
    "d64_g2_f16": (4, 2, 64, 16, "f16", [17, 500], [90, 260], 256),
    "g16_bf16": (32, 2, 128, 16, "bf16", [64, 3], [40, 129], 64),
    "empty_chunk": (8, 2, 128, 16, "bf16", [50, 10, 0], [0, 20, 1], 64),
    "long_context": (8, 2, 128, 16, "f16", [5000], [130], 512),
    "d64_b32_bf16": (8, 8, 64, 32, "bf16", [31, 300], [97, 128], 128),
}


def make_case(name):
    if name == "small_workload":
        return wl.make_prefill(small=True)
    Hq, Hkv, D, Bs, dt, prior, chunks, NB = CASES[name]
    return wl.chunked_prefill(name, 100 + len(name), Hq, Hkv, D, Bs, NB, dt, prior, chunks)


@pytest.mark.parametrize("ws", ["auto", None], ids=["workspace", "no_workspace"])
@pytest.mark.parametrize("name", list(CASES))
def test_prefill_matches_oracle(name, ws):
    """bf16 runs both ways: V narrowed to f16 in a workspace, and the two-part weights without one."""
    w = make_case(name)
    if ws is None and w.dtype != "bf16":
        pytest.skip("f16 takes no workspace")
    out, err, _, _ = H.gpu_prefill(w, workspace=ws)
    assert err == 0
    kp, vp = H.oracle_prefill_pools(w)
    ref = oracle_out(w, kp, vp)
    ok, rep = prefill_close(H.out_f64(out), ref, w.dtype)
    assert ok, (name, rep)


def scaled_v(w, factor):
    """The workload with every scattered V row of KV head h multiplied by factor[h] (bf16 bits)."""
    import dataclasses

    def scale(op):
        v = H.out_f64(H.to_dev_bits(op.v, w.dtype, "cpu")) * np.asarray(factor, np.float64)[None, :, None]
        bits = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        return dataclasses.replace(op, v=bits.reshape(op.v.shape))

    return dataclasses.replace(w, setup=[scale(op) for op in w.setup], step_scatter=scale(w.step_scatter))


@pytest.mark.parametrize("ws", ["auto", None], ids=["workspace", "no_workspace"])
def test_bf16_v_far_outside_the_f16_range(ws):
    """KV heads whose V values lie far above the f16 range (x 3e5 and x 2^60) or far below it
    (x 1e-6 and x 2^-100): narrowing scales each (sequence, KV head) by its own power of two, so
    every head keeps the accuracy of a unit-scale one.  Checked per head against the oracle,
    relative to the head's largest |v| (the 2e-3 bound of a unit-scale V)."""
    factors = [3e5, 1e-6, 2.0 ** 60, 2.0 ** -100, 1.0, 7.0, 0.01, 1.0]
    w = scaled_v(wl.chunked_prefill("vrange", 12, 16, 8, 128, 16, 256, "bf16", [300, 40, 0], [200, 150, 90]),
                 factors)
    out, err, _, _ = H.gpu_prefill(w, workspace=ws)
    assert err == 0
    o = H.out_f64(out)
    assert np.isfinite(o).all()
    kp, vp = H.oracle_prefill_pools(w)
    ref = oracle_out(w, kp, vp)
    G = w.num_heads // w.num_kv_heads
    ops = [op for op in list(w.setup) + [w.step_scatter] if op.slots.size]
    vmax = [max(np.abs(H.out_f64(H.to_dev_bits(op.v, "bf16", "cpu"))[:, h]).max() for op in ops)
            for h in range(w.num_kv_heads)]
    for h in range(w.num_kv_heads):
        d = np.abs(o[:, h * G:(h + 1) * G] - ref[:, h * G:(h + 1) * G]).max()
        assert d <= 4e-3 * vmax[h], (h, factors[h], d, vmax[h])


def test_wide_logits_move_the_running_maximum():
    """q scaled by 6: logits spread over ~+-100, so the lagging maximum moves often."""
    w = wl.chunked_prefill("wide", 7, 8, 2, 128, 16, 256, "bf16", [700, 0], [260, 200])
    qf = H.out_f64(H.to_dev_bits(w.q, "bf16", "cpu")) * 6.0
    q6 = torch.from_numpy(qf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    out, err, _, _ = H.gpu_prefill(w, q_bits=q6)
    assert err == 0
    kp, vp = H.oracle_prefill_pools(w)
    ref = oracle_out(w, kp, vp, q_bits=q6)
    ok, rep = prefill_close(H.out_f64(out), ref, "bf16")
    assert ok, rep


def test_bad_block_id_gives_nan_rows_and_flag():
    w = wl.chunked_prefill("bad", 8, 8, 2, 128, 16, 128, "f16", [40, 100], [30, 60])
    tab = w.block_tables.copy()
    tab[1, 2] = w.num_blocks + 5                 # a block sequence 1 needs
    out, err, _, _ = H.gpu_prefill(w, block_tables=tab)
    assert err & 0x1
    o = H.out_f64(out)
    r0, r1 = int(w.query_start[1]), int(w.query_start[2])
    assert np.isnan(o[r0:r1]).any()              # the tiles that needed the block
    kp, vp = H.oracle_prefill_pools(w)
    ref = oracle_out(w, kp, vp)
    ok, rep = prefill_close(o[:r0], ref[:r0], "f16")   # sequence 0 untouched
    assert ok, rep


@pytest.mark.parametrize("ws", ["auto", None], ids=["workspace", "no_workspace"])
def test_bf16_bad_block_id_gives_nan_rows_and_flag(ws):
    """A bad id in a bf16 call: with a workspace the narrowing passes skip that block and leave -1
    in the workspace table (NaN rows for the tiles that need it, PKV_DEVERR_BLOCK_ID), without one
    the prefill kernel finds it; the other sequence is unaffected either way."""
    w = wl.chunked_prefill("badbf", 18, 8, 2, 128, 16, 128, "bf16", [40, 100], [30, 60])
    tab = w.block_tables.copy()
    tab[1, 3] = -7                               # a block sequence 1 needs
    out, err, _, _ = H.gpu_prefill(w, block_tables=tab, workspace=ws)
    assert err & 0x1
    o = H.out_f64(out)
    r0, r1 = int(w.query_start[1]), int(w.query_start[2])
    assert np.isnan(o[r0:r1]).any()
    kp, vp = H.oracle_prefill_pools(w)
    ref = oracle_out(w, kp, vp)
    ok, rep = prefill_close(o[:r0], ref[:r0], "bf16")
    assert ok, rep


def test_chunk_longer_than_context_is_flagged():
    w = wl.chunked_prefill("ctx", 9, 4, 4, 128, 16, 64, "bf16", [20, 5], [10, 12])
    lens = w.context_lens.copy()
    lens[1] = 7                                  # chunk of 12 in a context of 7
    out, err, _, _ = H.gpu_prefill(w, context_lens=lens)
    assert err & 0x8
    o = H.out_f64(out)
    r0 = int(w.query_start[1])
    assert np.isnan(o[r0:]).all()
    kp, vp = H.oracle_prefill_pools(w)
    ref = oracle_out(w, kp, vp)
    ok, rep = prefill_close(o[:r0], ref[:r0], "bf16")
    assert ok, rep


def test_single_token_chunks_agree_with_the_decode_kernel():
    """Every sequence prefills one token: the same operation as decode, two different kernels."""
    rng = np.random.default_rng(10)
    prior = rng.integers(0, 900, size=12)
    w = wl.chunked_prefill("c1", 10, 32, 8, 128, 16, 1024, "bf16", prior, np.ones(12, np.int64))
    out, err, kp, vp = H.gpu_prefill(w)
    assert err == 0
    dev = torch.device("cuda:0")
    q = H.to_dev_bits(w.q, "bf16", dev)
    dec = torch.empty_like(q)
    B.paged_attn_decode(dec, q, kp, vp, torch.from_numpy(w.block_tables).to(dev),
                        torch.from_numpy(w.context_lens).to(dev), float(w.scale),
                        max_context_len=int(w.context_lens.max()))
    torch.cuda.synchronize()
    ok, rep = prefill_close(H.out_f64(out), H.out_f64(dec), "bf16")
    assert ok, rep


def test_full_size_every_row():
    """The full chunked-prefill workload (16 sequences, 23,714 query rows x 32 heads): every output
    row against the oracle, under the same rule as decode."""
    w = wl.make_prefill()
    out, err, _, _ = H.gpu_prefill(w)
    assert err == 0
    o = H.out_f64(out)
    assert np.isfinite(o).all()
    kp, vp = H.oracle_prefill_pools(w)
    ref = oracle_out(w, kp, vp)
    ok, rep = prefill_close(o, ref, w.dtype)
    assert ok, rep


def fp8_pools(w, dev):
    """E4M3 pools (random bytes outside the written slots) filled by the library's scatter and by
    the oracle's, with per-tensor amax / 448 scales over everything written."""
    ops = [op for op in list(w.setup) + [w.step_scatter] if op.slots.size]
    ks = max(wl.amax_scale(op.k, w.dtype) for op in ops)
    vs = max(wl.amax_scale(op.v, w.dtype) for op in ops)
    rng = np.random.default_rng(7)
    n = int(np.prod(w.pool_shape))
    kp_h = wl.garbage_bytes(rng, n).reshape(w.pool_shape)
    vp_h = wl.garbage_bytes(rng, n).reshape(w.pool_shape)
    kp, vp = torch.from_numpy(kp_h.copy()).to(dev), torch.from_numpy(vp_h.copy()).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for op in ops:
        B.reshape_and_cache(H.to_dev_bits(op.k, w.dtype, dev), H.to_dev_bits(op.v, w.dtype, dev), kp, vp,
                            torch.from_numpy(op.slots).to(dev), float(ks), float(vs), device_error=err)
        oracle.reshape_and_cache(op.k, op.v, w.dtype, kp_h, vp_h, "e4m3", op.slots, ks, vs)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(kp.cpu().numpy(), kp_h) and np.array_equal(vp.cpu().numpy(), vp_h)
    return kp, vp, kp_h, vp_h, float(ks), float(vs)


def gpu_prefill_fp8(w, kp, vp, ks, vs, dev, block_tables=None):
    q = H.to_dev_bits(w.q, w.dtype, dev)
    out = torch.full_like(q, float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    tab = w.block_tables if block_tables is None else block_tables
    B.paged_attn_prefill_fp8(out, q, kp, vp, torch.from_numpy(tab).to(dev),
                             torch.from_numpy(w.context_lens).to(dev), torch.from_numpy(w.query_start).to(dev),
                             float(w.scale), ks, vs, max_query_len=w.max_query_len, device_error=err)
    torch.cuda.synchronize()
    return H.out_f64(out), int(err.item())


@pytest.mark.parametrize("dtype,Hq,Hkv,Bs,prior,chunks", [
    ("f16", 8, 2, 16, [100, 0, 300], [60, 129, 1]),
    ("bf16", 16, 2, 32, [700, 37], [150, 90]),
])
def test_fp8_cache_prefill_matches_oracle(dtype, Hq, Hkv, Bs, prior, chunks):
    """E4M3 pools written by the library's scatter (per-tensor amax scales), prefilled through the
    widening gather and the tensor-core kernel, against the oracle on the dequantised values (the
    FP8 comparison rule: max-abs 3e-2, relative L2 1e-2)."""
    dev = torch.device("cuda:0")
    w = wl.chunked_prefill("fp8", 120 + Hq, Hq, Hkv, 128, Bs, 256, dtype, prior, chunks)
    kp, vp, kp_h, vp_h, ks, vs = fp8_pools(w, dev)
    o, err = gpu_prefill_fp8(w, kp, vp, ks, vs, dev)
    assert err == 0
    ref = oracle.paged_attn_prefill(w.q, dtype, kp_h, vp_h, "e4m3", w.block_tables, w.context_lens, w.query_start,
                                    w.scale, k_scale=ks, v_scale=vs)
    ok, rep = attention_close(o, ref, "e4m3", dtype)
    assert ok, rep


def test_fp8_bad_block_id_gives_nan_rows_and_flag():
    """A table entry outside the E4M3 pool: the widening gather marks the workspace entry invalid,
    the prefill reports PKV_DEVERR_BLOCK_ID with NaN rows, and the other sequence is unaffected."""
    dev = torch.device("cuda:0")
    w = wl.chunked_prefill("fp8bad", 8, 8, 2, 128, 16, 128, "f16", [40, 100], [30, 60])
    kp, vp, kp_h, vp_h, ks, vs = fp8_pools(w, dev)
    tab = w.block_tables.copy()
    tab[1, 2] = w.num_blocks + 5
    o, err = gpu_prefill_fp8(w, kp, vp, ks, vs, dev, block_tables=tab)
    assert err & 0x1
    r0, r1 = int(w.query_start[1]), int(w.query_start[2])
    assert np.isnan(o[r0:r1]).any()
    ref = oracle.paged_attn_prefill(w.q, "f16", kp_h, vp_h, "e4m3", w.block_tables, w.context_lens, w.query_start,
                                    w.scale, k_scale=ks, v_scale=vs)
    ok, rep = attention_close(o[:r0], ref[:r0], "e4m3", "f16")
    assert ok, rep
