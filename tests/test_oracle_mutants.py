"""The oracle's pins have teeth: each test plants one plausible mistake in a copy
of the oracle's C source, builds the copy, loads it in place of the oracle, and
checks that the pin named for that mistake fails (and that the unchanged oracle
passes the same pin).  Every mistake keeps all memory accesses in bounds.

Pins come from tests/test_oracle_pins.py and tests/test_oracle_prefill_pins.py;
each is independent of the oracle (library softmax, closed forms, the pages'
worked example, library number-format casts).
"""
import contextlib
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins
from tests import test_oracle_prefill_pins as ppins

SRC = os.path.join(os.path.dirname(oracle.__file__), "pagedkv_oracle.c")

# name: (text in the source, replacement, the pin expected to catch it)
MUTANTS = {
    "decode drops each sequence's last token": (
        "const int L = context_lens[s];\n            double* o = out",
        "const int L = context_lens[s] > 1 ? context_lens[s] - 1 : context_lens[s];\n            double* o = out",
        lambda: pins.test_matches_library_softmax_on_contiguous_cache(16, 1)),
    "decode pairs query heads with KV heads round-robin": (
        "            const int kvh = h / G;",
        "            const int kvh = h % num_kv_heads;",
        lambda: pins.test_matches_library_softmax_on_contiguous_cache(4, 4)),
    "decode drops the softmax scale": (
        "load_elem(k_pool, row + d, kv_dtype, ks);\n                x[t] = scale * dot;",
        "load_elem(k_pool, row + d, kv_dtype, ks);\n                x[t] = dot;",
        lambda: pins.test_matches_library_softmax_on_contiguous_cache(4, 1)),
    "decode reads V rows in reverse order inside a block": (
        "t % block_size) * head_dim;\n                for (int d = 0; d < head_dim; ++d)\n                    o[d] += p",
        "(block_size - 1 - t % block_size)) * head_dim;\n                for (int d = 0; d < head_dim; ++d)\n"
        "                    o[d] += p",
        lambda: pins.test_matches_block_form(16)),
    "decode normalises by l + 1": (
        "o[d] += p * load_elem(v_pool, row + d, kv_dtype, vs);\n            }\n"
        "            for (int d = 0; d < head_dim; ++d)\n                o[d] /= l;",
        "o[d] += p * load_elem(v_pool, row + d, kv_dtype, vs);\n            }\n"
        "            for (int d = 0; d < head_dim; ++d)\n                o[d] /= l + 1.0;",
        pins.test_single_token_returns_its_value),
    "decode ignores the V scale of an E4M3 cache": (
        "const double vs = kv_dtype == ORC_E4M3 ? v_scale : 1.0;\n\n    /* validate",
        "const double vs = 1.0;\n\n    /* validate",
        lambda: pins.test_fp8_cache_error_against_the_unquantised_cache("fp8")),
    "decode ignores the K scale of an E4M3 cache": (
        "const double ks = kv_dtype == ORC_E4M3 ? k_scale : 1.0;\n    const double vs = kv_dtype == ORC_E4M3 ? "
        "v_scale : 1.0;\n\n    /* validate",
        "const double ks = 1.0;\n    const double vs = kv_dtype == ORC_E4M3 ? v_scale : 1.0;\n\n    /* validate",
        lambda: pins.test_fp8_cache_error_against_the_unquantised_cache("fp8")),
    "prefill ignores the K scale of an E4M3 cache": (
        "const double ks = kv_dtype == ORC_E4M3 ? k_scale : 1.0;\n    const double vs = kv_dtype == ORC_E4M3 ? "
        "v_scale : 1.0;\n    for (int s = 0;",
        "const double ks = 1.0;\n    const double vs = kv_dtype == ORC_E4M3 ? v_scale : 1.0;\n    for (int s = 0;",
        ppins.test_fp8_cache_uses_the_dequantised_values),
    "prefill ignores the V scale of an E4M3 cache": (
        "const double vs = kv_dtype == ORC_E4M3 ? v_scale : 1.0;\n    for (int s = 0;",
        "const double vs = 1.0;\n    for (int s = 0;",
        ppins.test_fp8_cache_uses_the_dequantised_values),
    "E4M3 subnormals decoded one binade low": (
        "v = ldexp((double)m, -9);",
        "v = ldexp((double)m, -10);",
        pins.test_e4m3_decode_exhaustive_against_library),
    "E4M3 encoder rounds ties away from zero": (
        "double r = nearbyint(q);",
        "double r = floor(q + 0.5);",
        pins.test_e4m3_encode_against_library_and_roundtrip),
    "E4M3 encoder saturates to NaN": (
        "return sign | 0x7e;",
        "return sign | 0x7f;",
        pins.test_e4m3_encode_saturates),
    "f16 subnormals decoded one binade high": (
        "v = ldexp((double)m, -24);",
        "v = ldexp((double)m, -23);",
        pins.test_f16_decode_exhaustive),
    "scatter writes the pool as [block][offset][head]": (
        "size_t dst = (((size_t)blk * num_kv_heads + h) * block_size + off) * head_dim;",
        "size_t dst = (((size_t)blk * block_size + off) * num_kv_heads + h) * head_dim;",
        pins.test_scatter_fp8_quantises_each_element),
    "prefill without the causal mask inside the chunk": (
        "const int p = L - C + (int)(r - query_start[s]);",
        "const int p = L - 1;",
        lambda: ppins.test_matches_library_causal_softmax(4, 1)),
    "prefill rows attend one key too few": (
        "const int p = L - C + (int)(r - query_start[s]);",
        "const int p = L - C + (int)(r - query_start[s]) - (r > query_start[s]);",
        lambda: ppins.test_matches_library_causal_softmax(16, 1)),
    "prefill pairs query heads with KV heads round-robin": (
        "const int h = (int)(u % num_heads), kvh = h / G;",
        "const int h = (int)(u % num_heads), kvh = h % num_kv_heads;",
        lambda: ppins.test_matches_library_causal_softmax(4, 4)),
    "bf16 normals decoded with the wrong exponent bias": (
        "v = ldexp((double)(128 + m), e - 134);",
        "v = ldexp((double)(128 + m), e - 133);",
        pins.test_bf16_decode_exhaustive),
    "gather reads the rows of a block in reverse": (
        "t % block_size) * head_dim;\n        memcpy(",
        "(block_size - 1 - t % block_size)) * head_dim;\n        memcpy(",
        pins.test_worked_example_block_table_and_gather),
    "swap writes the V block over the K block": (
        "memcpy((char*)dst_v + (size_t)d * block_bytes, (const char*)src_v",
        "memcpy((char*)dst_k + (size_t)d * block_bytes, (const char*)src_v",
        pins.test_swap_blocks_round_trip_and_untouched_blocks),
    "copy-on-write copies destination onto source": (
        "memmove((char*)k_pool + (size_t)d * block_bytes, (char*)k_pool + (size_t)s * block_bytes, block_bytes);",
        "memmove((char*)k_pool + (size_t)s * block_bytes, (char*)k_pool + (size_t)d * block_bytes, block_bytes);",
        pins.test_copy_blocks_copies_only_destinations),
}


@contextlib.contextmanager
def oracle_from_source(text, tmp_path):
    """Build ``text`` as the oracle library and make the wrapper load it until the block exits."""
    c = tmp_path / "oracle_mutant.c"
    so = tmp_path / "liboracle_mutant.so"
    c.write_text(text)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(c), "-lm"])
    saved_lib, saved_build = oracle._lib, oracle.build
    oracle._lib = None
    oracle.build = lambda force=False: str(so)
    try:
        yield
    finally:
        oracle._lib, oracle.build = saved_lib, saved_build


@pytest.mark.parametrize("name", list(MUTANTS))
def test_pin_catches_planted_mistake(name, tmp_path):
    old, new, pin = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, "the mutation must name one place in the source"
    pin()                                              # the oracle as it is passes the pin
    with oracle_from_source(src.replace(old, new), tmp_path):
        with pytest.raises(AssertionError):
            pin()
    pin()                                              # and the real oracle is back afterwards
