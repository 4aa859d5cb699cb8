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


def shared_call(w, kp, vp, spl, us, ul, mp, ps=0, plan="shared"):
    """One shared-prefix call on device copies of the arrays; (output in float64, error word)."""
    dev = torch.device("cuda:0")
    out = torch.empty((w.num_seqs, w.num_heads, w.head_dim), dtype=H.TORCH16[w.q_dtype], device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    B.paged_attn_decode_shared_prefix(
        out, H.to_dev_bits(w.q, w.q_dtype, dev), kp, vp, torch.from_numpy(w.block_tables).to(dev),
        torch.from_numpy(w.context_lens).to(dev), float(w.scale), max_context_len=w.max_context_len,
        seq_prefix_len=torch.from_numpy(spl).to(dev), unit_seqs=torch.from_numpy(us).to(dev),
        unit_len=torch.from_numpy(ul).to(dev), max_prefix_len=mp, k_scale=float(w.k_scale),
        v_scale=float(w.v_scale), partition_size=ps, plan=plan, device_error=err)
    torch.cuda.synchronize()
    return H.out_f64(out), int(err.item())


def device_pools(w, ps=0):
    dev = torch.device("cuda:0")
    g = H.gpu_step(w, keep_pools=True, partition_size=ps)       # builds the pools through the library
    return H.to_dev_bits(g["k_pool"], w.kv_dtype, dev), H.to_dev_bits(g["v_pool"], w.kv_dtype, dev), g["out"]


def run_shared(w, ps=0, drop_units=False, plan="shared"):
    kp, vp, plain = device_pools(w, ps)
    G = w.num_heads // w.num_kv_heads
    spl, us, ul, mp = B.find_shared_prefixes(w.block_tables, w.context_lens, w.block_size, 16 // G)
    if drop_units:                       # a caller may leave some groups unshared
        keep = np.arange(len(ul)) % 2 == 0
        for u in np.nonzero(~keep)[0]:
            for s in us[u]:
                if s >= 0:
                    spl[s] = 0
        us, ul = us[keep], ul[keep]
    out, err = shared_call(w, kp, vp, spl, us, ul, mp, ps, plan)
    assert err == 0
    return out, plain, len(ul), mp


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


@pytest.mark.parametrize("plan", ["auto", "plain"])
def test_other_plans_give_the_same_result(plan):
    """The automatic plan (on this workload the prefixes fit in L2, so the plain call runs) and the
    plain plan reach the oracle's result too."""
    w = wl.make("prefix", small=True)
    out, _, units, _ = run_shared(w, plan=plan)
    ref = H.oracle_step(w)["out"]
    ok, rep = attention_close(out, ref, w.kv_dtype, w.q_dtype)
    assert ok, rep


def broken_units_case():
    w = wl.make("prefix", small=True)
    kp, vp, _ = device_pools(w)
    G = w.num_heads // w.num_kv_heads
    spl, us, ul, mp = B.find_shared_prefixes(w.block_tables, w.context_lens, w.block_size, 16 // G)
    assert len(ul) >= 3 and mp > w.block_size
    return w, kp, vp, spl, us, ul, mp


def check_nan_only(out, ref, w, bad):
    """NaN in exactly the rows of the sequences in ``bad``; every other sequence matches the oracle."""
    bad = sorted(set(int(s) for s in bad))
    good = [s for s in range(w.num_seqs) if s not in bad]
    assert np.isnan(out[bad]).all()
    ok, rep = attention_close(out[good], ref[good], w.kv_dtype, w.q_dtype)
    assert ok, rep


def test_prefix_longer_than_the_bound_is_flagged():
    """One sequence claims a prefix beyond max_prefix_len: its merge would index past its row of
    partitions, so it is refused on the device before any read; it and its unit's other members
    (whose unit no longer matches them all) get NaN, the rest is exact."""
    w, kp, vp, spl, us, ul, mp = broken_units_case()
    s0 = int(us[0][0])
    spl[s0] = mp + w.block_size
    out, err = shared_call(w, kp, vp, spl, us, ul, mp)
    assert err & 0x8
    check_nan_only(out, H.oracle_step(w)["out"], w, [m for m in us[0] if m >= 0])


def test_unit_longer_than_the_bound_is_flagged():
    w, kp, vp, spl, us, ul, mp = broken_units_case()
    ul[1] = mp + w.block_size
    out, err = shared_call(w, kp, vp, spl, us, ul, mp)
    assert err & 0x8
    check_nan_only(out, H.oracle_step(w)["out"], w, [m for m in us[1] if m >= 0])


def test_sequence_with_a_prefix_but_no_unit_is_flagged():
    """A unit is dropped while its members keep their prefix lengths: their prefix slots are never
    written, so their merges must not read stale partials."""
    w, kp, vp, spl, us, ul, mp = broken_units_case()
    dropped = [m for m in us[2] if m >= 0]
    keep = np.arange(len(ul)) != 2
    out, err = shared_call(w, kp, vp, spl, us[keep], ul[keep], mp)
    assert err & 0x8
    check_nan_only(out, H.oracle_step(w)["out"], w, dropped)


def test_member_whose_prefix_differs_from_its_unit_is_flagged():
    w, kp, vp, spl, us, ul, mp = broken_units_case()
    s0 = int(us[1][0])
    spl[s0] -= w.block_size            # still a valid prefix length, but not the unit's
    out, err = shared_call(w, kp, vp, spl, us, ul, mp)
    assert err & 0x8
    check_nan_only(out, H.oracle_step(w)["out"], w, [m for m in us[1] if m >= 0])
