"""Shared-prefix decode (each shared prompt read once per unit) against the oracle.

The oracle is the plain definition; the shared-prefix call must reach the same
result as attending each sequence on its own (glossary "PagedAttention",
section "Sharing blocks across sequences": shared blocks give the result of
private copies)."""
import numpy as np
import pytest
import torch

from paged_kv_cache_324_b200 import binding as B
from paged_kv_cache_324_b200 import workload as wl
from tests import harness as H
from tests.parity import attention_close

pytestmark = pytest.mark.gpu


def run_shared(w, ps=0, drop_units=False):
    dev = torch.device("cuda:0")
    g = H.gpu_step(w, keep_pools=True, partition_size=ps)       # builds the pools through the library
    kp = H.to_dev_bits(g["k_pool"], w.kv_dtype, dev)
    vp = H.to_dev_bits(g["v_pool"], w.kv_dtype, dev)
    G = w.num_heads // w.num_kv_heads
    spl, us, ul, mp = B.find_shared_prefixes(w.block_tables, w.context_lens, w.block_size, 16 // G)
    if drop_units:                       # a caller may leave some groups unshared
        keep = np.arange(len(ul)) % 2 == 0
        for u in np.nonzero(~keep)[0]:
            for s in us[u]:
                if s >= 0:
                    spl[s] = 0
        us, ul = us[keep], ul[keep]
    out = torch.empty((w.num_seqs, w.num_heads, w.head_dim), dtype=H.TORCH16[w.q_dtype], device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    B.paged_attn_decode_shared_prefix(
        out, H.to_dev_bits(w.q, w.q_dtype, dev), kp, vp, torch.from_numpy(w.block_tables).to(dev),
        torch.from_numpy(w.context_lens).to(dev), float(w.scale), max_context_len=w.max_context_len,
        seq_prefix_len=torch.from_numpy(spl).to(dev), unit_seqs=torch.from_numpy(us).to(dev),
        unit_len=torch.from_numpy(ul).to(dev), max_prefix_len=mp, k_scale=float(w.k_scale),
        v_scale=float(w.v_scale), partition_size=ps, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return H.out_f64(out), g["out"], len(ul), mp


@pytest.mark.parametrize("samples,H_,Hkv,dtype,B_,ps", [
    (8, 32, 8, 'f16', 16, 0), (8, 32, 8, 'f16', 16, 128), (3, 16, 2, 'bf16', 16, 64),
    (2, 16, 2, 'f16', 32, 0), (5, 8, 8, 'f16', 16, 64), (6, 32, 4, 'bf16', 32, 128)])
def test_shared_prefix_matches_oracle(samples, H_, Hkv, dtype, B_, ps):
    w = wl.shared_prefix_sampling("sp", 40 + samples, 3, samples, H_, Hkv, 128, B_, 1200, dtype,
                                  prefix_blocks=12 if B_ == 16 else 6, tail_max=90)
    out, plain, units, mp = run_shared(w, ps)
    assert units > 0 and mp > 0
    ref = H.oracle_step(w)["out"]
    ok, rep = attention_close(out, ref, w.kv_dtype, w.q_dtype)
    assert ok, rep
    assert attention_close(plain, ref, w.kv_dtype, w.q_dtype)[0]


def test_shared_prefix_with_unshared_groups():
    w = wl.make("prefix", small=True)
    out, _, units, _ = run_shared(w, drop_units=True)
    ref = H.oracle_step(w)["out"]
    ok, rep = attention_close(out, ref, w.kv_dtype, w.q_dtype)
    assert ok, rep


def test_shared_prefix_long_prompts_small():
    w = wl.make("prefix_long", small=True)
    out, _, units, mp = run_shared(w)
    assert units == 4 and mp == 80 * 16
    ref = H.oracle_step(w)["out"]
    ok, rep = attention_close(out, ref, w.kv_dtype, w.q_dtype)
    assert ok, rep


def test_shared_prefix_full_size_workload():
    w = wl.make("prefix")
    out, _, units, mp = run_shared(w)
    assert units == 32 and mp == 512
    ref = H.oracle_step(w)["out"]
    ok, rep = attention_close(out, ref, w.kv_dtype, w.q_dtype)
    assert ok, rep
