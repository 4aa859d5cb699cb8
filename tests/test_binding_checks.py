"""Host-side argument checks of the Python binding, on CPU.

The kernels read num_seqs rows of the block tables and num_seqs context lengths,
and atomically OR into a 4-byte device error word; the binding rejects tensors
too small for that before it takes any pointer (so CPU tensors reach the checks).
"""
import pytest
import torch

from paged_kv_cache_324_b200 import binding as B


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_324_b200 import build
    build.build()


S, H, Hkv, D, NB, Bs = 4, 8, 2, 128, 16, 16


def decode_args(tables_rows=S, lens_n=S, tables_dtype=torch.int32):
    q = torch.zeros((S, H, D), dtype=torch.float16)
    pool = torch.zeros((NB, Hkv, Bs, D), dtype=torch.float16)
    return (torch.empty_like(q), q, pool, pool.clone(), torch.zeros((tables_rows, 4), dtype=tables_dtype),
            torch.ones(lens_n, dtype=torch.int32), 0.1)


def test_decode_rejects_short_tables_and_lengths():
    with pytest.raises(ValueError, match="block_tables must be"):
        B.paged_attn_decode(*decode_args(tables_rows=S - 1), max_context_len=16)
    with pytest.raises(ValueError, match="context_lens must hold"):
        B.paged_attn_decode(*decode_args(lens_n=S - 1), max_context_len=16)
    with pytest.raises(TypeError, match="int32"):
        B.paged_attn_decode(*decode_args(tables_dtype=torch.int64), max_context_len=16)
    # well-formed (extra table rows allowed): passes the checks, then needs GPU tensors
    with pytest.raises(ValueError, match="CUDA tensor"):
        B.paged_attn_decode(*decode_args(tables_rows=S + 2), max_context_len=16)


def test_prefill_rejects_short_tables_and_bad_offsets():
    T = 10
    q = torch.zeros((T, H, D), dtype=torch.bfloat16)
    pool = torch.zeros((NB, Hkv, Bs, D), dtype=torch.bfloat16)
    lens = torch.tensor([5, 5], dtype=torch.int32)
    qs = torch.tensor([0, 5, 10], dtype=torch.int32)
    with pytest.raises(ValueError, match="block_tables must be"):
        B.paged_attn_prefill(torch.empty_like(q), q, pool, pool, torch.zeros((1, 2), dtype=torch.int32), lens, qs,
                             0.1, max_query_len=5)
    with pytest.raises(ValueError, match="num_seqs \\+ 1"):
        B.paged_attn_prefill(torch.empty_like(q), q, pool, pool, torch.zeros((2, 2), dtype=torch.int32), lens,
                             qs[:2], 0.1, max_query_len=5)
    p8 = torch.zeros((NB, Hkv, Bs, D), dtype=torch.uint8)
    with pytest.raises(ValueError, match="block_tables must be"):
        B.paged_attn_prefill_fp8(torch.empty_like(q), q, p8, p8, torch.zeros(2, dtype=torch.int32), lens, qs,
                                 0.1, 1.0, 1.0, max_query_len=5)
    with pytest.raises(ValueError, match="num_seqs \\+ 1"):
        B.paged_attn_prefill_fp8(torch.empty_like(q), q, p8, p8, torch.zeros((2, 2), dtype=torch.int32), lens,
                                 qs[:2], 0.1, 1.0, 1.0, max_query_len=5)
    qf = torch.zeros((T, H, D), dtype=torch.float32)
    with pytest.raises(TypeError, match="float16 or bfloat16"):
        B.paged_attn_prefill_fp8(torch.empty_like(qf), qf, p8, p8, torch.zeros((2, 2), dtype=torch.int32), lens,
                                 qs, 0.1, 1.0, 1.0, max_query_len=5)


def test_prefill_workspace_choice():
    """workspace is a tensor, "auto" (a bf16 call gets one of prefill_workspace_bytes) or None (the
    two-part weights); anything else is refused before a pointer is taken."""
    T = 10
    q = torch.zeros((T, H, D), dtype=torch.bfloat16)
    pool = torch.zeros((NB, Hkv, Bs, D), dtype=torch.bfloat16)
    lens = torch.tensor([5, 5], dtype=torch.int32)
    qs = torch.tensor([0, 5, 10], dtype=torch.int32)
    tables = torch.zeros((2, 2), dtype=torch.int32)
    with pytest.raises(ValueError, match="workspace must be"):
        B.paged_attn_prefill(torch.empty_like(q), q, pool, pool, tables, lens, qs, 0.1, max_query_len=5,
                             workspace="none")
    for ws in ("auto", None):   # well-formed: passes the checks, then needs GPU tensors
        with pytest.raises(ValueError, match="CUDA tensor"):
            B.paged_attn_prefill(torch.empty_like(q), q, pool, pool, tables, lens, qs, 0.1, max_query_len=5,
                                 workspace=ws)
    assert B.prefill_workspace_bytes(torch.bfloat16, 2, 2, Hkv, D, Bs) > 0
    assert B.prefill_workspace_bytes(torch.float16, 2, 2, Hkv, D, Bs) == 0


def test_shared_prefix_rejects_inconsistent_arguments():
    out, q, kp, vp, tables, lens, scale = decode_args()
    i32 = torch.zeros(S, dtype=torch.int32)
    units = torch.zeros((1, 2), dtype=torch.int32)
    ulen = torch.zeros(1, dtype=torch.int32)
    with pytest.raises(ValueError, match="inconsistent"):
        B.paged_attn_decode_shared_prefix(out[:2], q, kp, vp, tables, lens, scale, max_context_len=16,
                                          seq_prefix_len=i32, unit_seqs=units, unit_len=ulen, max_prefix_len=16)
    with pytest.raises(ValueError, match="block_tables must be"):
        B.paged_attn_decode_shared_prefix(out, q, kp, vp, tables[:2], lens, scale, max_context_len=16,
                                          seq_prefix_len=i32, unit_seqs=units, unit_len=ulen, max_prefix_len=16)
    with pytest.raises(TypeError, match="unit_seqs must be int32"):
        B.paged_attn_decode_shared_prefix(out, q, kp, vp, tables, lens, scale, max_context_len=16,
                                          seq_prefix_len=i32, unit_seqs=units.long(), unit_len=ulen,
                                          max_prefix_len=16)
    with pytest.raises(ValueError, match="seq_prefix_len must hold"):
        B.paged_attn_decode_shared_prefix(out, q, kp, vp, tables, lens, scale, max_context_len=16,
                                          seq_prefix_len=i32[:1], unit_seqs=units, unit_len=ulen,
                                          max_prefix_len=16)


def test_device_error_word_must_be_a_4_byte_integer():
    assert B._err(None) is None
    for bad in (torch.zeros(1, dtype=torch.float32), torch.zeros(0, dtype=torch.int32),
                torch.zeros(1, dtype=torch.int64), torch.zeros(4, dtype=torch.uint8)):
        with pytest.raises(TypeError, match="device_error"):
            B._err(bad)
    with pytest.raises(ValueError, match="CUDA tensor"):       # right type, but on the host
        B._err(torch.zeros(1, dtype=torch.int32))


def test_copy_blocks_needs_matching_pools():
    k = torch.zeros((8, 2, 16, 64), dtype=torch.float16)
    pairs = torch.tensor([[0, 1]], dtype=torch.int64)
    with pytest.raises(ValueError, match="one shape and dtype"):
        B.copy_blocks(k, torch.zeros((4, 2, 16, 64), dtype=torch.float16), pairs)
    with pytest.raises(ValueError, match="one shape and dtype"):
        B.copy_blocks(k, torch.zeros((8, 2, 16, 64), dtype=torch.bfloat16), pairs)


def test_decode_needs_one_pool_dtype():
    out, q, kp, vp, tables, lens, scale = decode_args()
    with pytest.raises(ValueError, match="inconsistent"):
        B.paged_attn_decode(out, q, kp, vp.to(torch.bfloat16), tables, lens, scale, max_context_len=16)
    with pytest.raises(ValueError, match="inconsistent"):
        B.paged_attn_decode_shared_prefix(out, q, kp, vp.to(torch.bfloat16), tables, lens, scale, max_context_len=16,
                                          seq_prefix_len=torch.zeros(S, dtype=torch.int32),
                                          unit_seqs=torch.zeros((1, 2), dtype=torch.int32),
                                          unit_len=torch.zeros(1, dtype=torch.int32), max_prefix_len=16)


def test_scatter_and_swap_need_one_dtype_per_pair():
    k = torch.zeros((3, Hkv, D), dtype=torch.float16)
    pool = torch.zeros((NB, Hkv, Bs, D), dtype=torch.float16)
    slots = torch.zeros(3, dtype=torch.int64)
    with pytest.raises(ValueError, match="share a dtype"):
        B.reshape_and_cache(k, k.to(torch.bfloat16), pool, pool, slots)
    with pytest.raises(ValueError, match="share a dtype"):
        B.reshape_and_cache(k, k, pool, pool.to(torch.bfloat16), slots)
    pairs = torch.zeros((1, 2), dtype=torch.int64)
    with pytest.raises(ValueError, match="one layout and dtype"):
        B.swap_blocks(pool, pool.to(torch.bfloat16), pool, pool, pairs)
