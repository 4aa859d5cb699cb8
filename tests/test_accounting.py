"""The byte and FLOP accounting behind every roofline figure, on CPU.

Each counting function is checked against a brute-force count on small
workloads (every token, slot and causal (query, key) pair enumerated), and the
full-size figures the design notes quote are reproduced exactly.
"""
import numpy as np
import pytest

from paged_kv_cache_324_b200 import workload as wl


@pytest.mark.parametrize("name", ["tiny", "gqa", "prefix", "fp8"])
def test_decode_bytes_by_enumeration(name):
    w = wl.make(name, small=True)
    e, eq = wl.ELEM_BYTES[w.kv_dtype], wl.ELEM_BYTES[w.q_dtype]
    kv = table = 0
    distinct = set()
    for s in range(w.num_seqs):
        L = int(w.context_lens[s])
        for t in range(L):
            kv += 2 * w.num_kv_heads * w.head_dim * e                  # K and V rows of every head
            distinct.add((int(w.block_tables[s, t // w.block_size]), t % w.block_size))
        table += 4 * len({t // w.block_size for t in range(L)})        # each used table entry once
    q_out = 2 * w.num_seqs * w.num_heads * w.head_dim * eq
    assert wl.decode_algorithmic_bytes(w) == kv + q_out + table + 4 * w.num_seqs
    kv_distinct = len(distinct) * 2 * w.num_kv_heads * w.head_dim * e
    assert wl.decode_distinct_bytes(w) == kv_distinct + q_out + table + 4 * w.num_seqs
    if name != "prefix":                                               # no sharing: nothing counted twice
        assert wl.decode_distinct_bytes(w) == wl.decode_algorithmic_bytes(w)
    else:
        assert wl.decode_distinct_bytes(w) < wl.decode_algorithmic_bytes(w)


def test_prefill_flops_by_enumeration():
    w = wl.make_prefill(small=True)
    pairs = 0
    for s in range(w.num_seqs):
        L, C = int(w.context_lens[s]), int(w.chunk_lens[s])
        for j in range(C):
            pairs += (L - C + j) + 1                                   # row j attends to positions 0..L-C+j
    assert wl.prefill_flops(w) == 4 * w.head_dim * w.num_heads * pairs
    kv = int(w.context_lens.sum()) * 2 * w.num_kv_heads * w.head_dim * 2
    assert wl.prefill_bytes(w) == kv + 2 * w.num_tokens * w.num_heads * w.head_dim * 2


def test_full_size_figures_quoted_in_the_design_notes():
    w = wl.make("opt13b")
    assert wl.decode_algorithmic_bytes(w) == 1_302_626_168
    assert wl.step_algorithmic_bytes(w) == 1_305_248_120
    p = wl.make_prefill()
    assert p.num_tokens == 23_714
    assert wl.prefill_flops(p) == 948_108_214_272
    assert round(wl.prefill_bytes(p) / 1e6) == 594
