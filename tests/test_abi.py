"""The C-ABI library: it builds for sm_100a, loads, exports every entry point
declared in include/pagedkv.h, and rejects bad host-side arguments with the
documented status codes before touching the GPU (no GPU needed here)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedkv.h")


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_324_b200 import binding, build
    build.build()
    return binding.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ("pkv_paged_attn_decode", "pkv_reshape_and_cache", "pkv_copy_blocks",
                 "pkv_decode_workspace_bytes", "pkv_status_string", "pkv_version"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    from paged_kv_cache_324_b200 import binding
    out = subprocess.run(["nm", "-D", "--defined-only", binding._LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (pkv_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(lib, n)


def test_library_is_built_for_sm100a(lib):
    from paged_kv_cache_324_b200 import binding
    out = subprocess.run(["cuobjdump", "--list-elf", binding._LIB_PATH], capture_output=True, text=True).stdout
    assert "sm_100a" in out


def test_version_and_status_strings(lib):
    from paged_kv_cache_324_b200 import binding
    assert binding.version() >= 100
    assert binding.status_string(0) == "ok"
    assert "workspace" in binding.status_string(3)


def _decode(lib, **over):
    P = ctypes.c_void_p
    args = dict(out=P(16), q=P(16), q_dtype=0, k_pool=P(16), v_pool=P(16), kv_dtype=0, k_scale=1.0,
                v_scale=1.0, block_tables=P(16), max_blocks=4, context_lens=P(16), max_len=64, S=2, H=8,
                Hkv=2, D=128, B=16, NB=10, scale=0.1, ps=0, ws=None, ws_bytes=0, err=None, stream=None)
    args.update(over)
    return lib.pkv_paged_attn_decode(*args.values())


@pytest.mark.parametrize("over,status", [
    (dict(H=0), 1), (dict(H=6, Hkv=4), 1), (dict(S=-1), 1), (dict(ps=24), 1),
    (dict(B=8), 2), (dict(D=96), 2), (dict(H=34, Hkv=2), 2), (dict(q_dtype=0, kv_dtype=1), 2),
    (dict(kv_dtype=2, D=64), 2), (dict(kv_dtype=2, k_scale=0.0), 1), (dict(q_dtype=2), 2),
    (dict(scale=float("inf")), 1), (dict(scale=float("-inf")), 1), (dict(scale=float("nan")), 1),
    (dict(kv_dtype=2, k_scale=float("inf")), 1), (dict(kv_dtype=2, v_scale=float("inf")), 1),
    (dict(kv_dtype=2, v_scale=float("nan")), 1),
])
def test_decode_rejects_bad_arguments(lib, over, status):
    """Host-side checks of pkv_paged_attn_decode, non-finite scales included: nothing is launched."""
    assert _decode(lib, **over) == status


def test_static_workspace_call_checks_arguments_before_its_size(lib):
    """The allocation-free decode call answers a bad argument with the same status as the ordinary
    call, even when the (meaningless) request would also be too large for its array."""
    f = lib.pkv_paged_attn_decode_static_ws
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    f.argtypes = [P, P, I, P, P, I, F, F, P, I, P, I, I, I, I, I, I, I, F, I, P, P]
    f.restype = I
    big = 1 << 24                      # 16M tokens in 16-token partitions: far beyond the 64 MiB array
    base = [P(16), P(16), 0, P(16), P(16), 0, 1.0, 1.0, P(16), big // 16, P(16), big, 64, 8, 2, 128, 16, 10, 0.1,
            16, None, None]
    assert f(*base) == 3               # well-formed: refused for its size
    bad_q = list(base)
    bad_q[1] = None
    assert f(*bad_q) == 1
    bad_scale = list(base)
    bad_scale[18] = float("inf")
    assert f(*bad_scale) == 1
    bad_group = list(base)
    bad_group[13], bad_group[14] = 34, 2
    assert f(*bad_group) == 2


def test_shared_prefix_rejects_an_unknown_plan(lib):
    f = lib.pkv_paged_attn_decode_shared_prefix
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    f.argtypes = [P, P, I, P, P, I, F, F, P, I, P, I, I, I, I, I, I, I, F, I, P, P, P, I, I, I, I, P, Z, P, P]
    f.restype = I
    args = [P(16), P(16), 0, P(16), P(16), 0, 1.0, 1.0, P(16), 4, P(16), 64, 2, 8, 2, 128, 16, 10, 0.1, 0,
            P(16), P(16), P(16), 1, 2, 32, 0, P(256), 1 << 20, None, None]
    for plan in (3, -1):
        args[26] = plan
        assert f(*args) == 1


def test_decode_rejects_null_and_misaligned(lib):
    assert _decode(lib, q=None) == 1
    assert _decode(lib, out=ctypes.c_void_p(18)) == 5


def _prefill(lib, **over):
    P = ctypes.c_void_p
    args = dict(out=P(16), q=P(16), dtype=1, k_pool=P(16), v_pool=P(16), block_tables=P(16), max_blocks=4,
                context_lens=P(16), query_start=P(16), max_q=64, S=2, T=100, H=8, Hkv=2, D=128, B=16, NB=10,
                scale=0.1, ws=None, ws_bytes=0, err=None, stream=None)
    args.update(over)
    f = lib.pkv_paged_attn_prefill
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    f.argtypes = [P, P, I, P, P, P, I, P, P, I, I, I, I, I, I, I, I, F, P, Z, P, P]
    f.restype = I
    return f(*args.values())


@pytest.mark.parametrize("over,status", [
    (dict(H=6, Hkv=4), 1), (dict(S=-1), 1), (dict(scale=0.0), 1), (dict(scale=-1.0), 1),
    (dict(scale=float("inf")), 1), (dict(max_q=-1), 1), (dict(H=0), 1),
    (dict(dtype=2), 2), (dict(D=96), 2), (dict(B=8), 2), (dict(H=6, Hkv=2), 2), (dict(H=64, Hkv=2), 2),
    (dict(q=None), 1), (dict(query_start=None), 1), (dict(out=ctypes.c_void_p(24)), 5),
    (dict(query_start=ctypes.c_void_p(18)), 5),
    (dict(T=0), 0), (dict(S=0), 0), (dict(max_q=0), 0),
    # bf16 with a workspace: too small, or not 256-byte aligned (the workspace path's own checks)
    (dict(ws=ctypes.c_void_p(256), ws_bytes=1024), 3), (dict(ws=ctypes.c_void_p(272), ws_bytes=1 << 20), 5),
])
def test_prefill_rejects_bad_arguments(lib, over, status):
    """Host-side checks of pkv_paged_attn_prefill (group size 3 and 32, FP8, odd sizes, a
    non-positive scale, null and misaligned pointers; empty problems succeed at once)."""
    assert _prefill(lib, **over) == status


def test_reshape_and_copy_reject_bad_arguments(lib):
    P = ctypes.c_void_p
    assert lib.pkv_reshape_and_cache(P(16), P(16), 0, P(16), P(16), 1, 1.0, 1.0, P(16), 4, 2, 128, 16, 10,
                                     None, None) == 2   # f16 in, bf16 pool
    assert lib.pkv_reshape_and_cache(P(16), P(16), 0, P(16), P(16), 0, 1.0, 1.0, P(16), 4, 2, 100, 16, 10,
                                     None, None) == 2   # head_dim not a multiple of 8
    assert lib.pkv_reshape_and_cache(P(16), P(16), 0, P(16), P(16), 0, 1.0, 1.0, P(16), 0, 2, 128, 16, 10,
                                     None, None) == 0   # nothing to do
    for ks, vs in ((0.0, 1.0), (1.0, -1.0), (float("inf"), 1.0), (1.0, float("nan"))):
        assert lib.pkv_reshape_and_cache(P(16), P(16), 0, P(16), P(16), 2, ks, vs, P(16), 4, 2, 128, 16, 10,
                                         None, None) == 1   # E4M3 scales must be positive and finite
    assert lib.pkv_copy_blocks(P(16), P(16), 24, P(16), 3, 10, None, None) == 2
    assert lib.pkv_copy_blocks(P(16), P(16), 32, P(16), -1, 10, None, None) == 1
    assert lib.pkv_copy_blocks(P(16), P(16), 32, P(16), 0, 10, None, None) == 0


def test_workspace_size_rules(lib):
    from paged_kv_cache_324_b200 import binding as B
    # fits one partition: no workspace
    assert B.decode_workspace_bytes(64, 40, 40, 128, "f16", 16, 512, 1024) == 0
    # 32768 tokens in 512-token partitions: 64 partitions of (128 floats + max + sum)
    n = B.decode_workspace_bytes(16, 64, 8, 128, "e4m3", 16, 32768, 512)
    rows = 16 * 64 * 64
    assert n >= rows * (128 * 4 + 8)
    assert B.decode_partition_size(16, 8, 128, "e4m3", 16, 32768, 512) == 512
    assert B.decode_partition_size(16, 8, 128, "f16", 16, 300, 512) == 304    # one partition, rounded to the block
    # automatic choice: ~512 KB of K+V per partition and KV head
    assert B.decode_partition_size(256, 8, 128, "bf16", 16, 4096, 0) == 1024
    assert B.decode_partition_size(16, 8, 128, "e4m3", 16, 32768, 0) == 2048
    # ... shrunk when there are few work units, never below 4 blocks
    assert B.decode_partition_size(4, 8, 64, "f16", 16, 256, 0) == 64


def test_prefill_workspace_size(lib):
    """The bf16 prefill's narrowing workspace: the f16 V pool (num_seqs x max_blocks_per_seq blocks),
    its table, one factor per (sequence, KV head) and one partial maximum per (sequence, KV head,
    16 table slots), each part rounded up to 256 bytes; none for f16 or E4M3."""
    from paged_kv_cache_324_b200 import binding as B
    assert B.prefill_workspace_bytes("f16", 2, 4, 2, 128, 16) == 0
    assert B.prefill_workspace_bytes("e4m3", 2, 4, 2, 128, 16) == 0
    assert B.prefill_workspace_bytes("bf16", 2, 4, 2, 128, 16) == 8 * 2 * 16 * 128 * 2 + 3 * 256
    S, maxb, Hkv, D, Bs = 16, 320, 8, 128, 16
    pool = S * maxb * Hkv * Bs * D * 2
    parts = -(-(S * Hkv * 20 * 4) // 256) * 256
    assert B.prefill_workspace_bytes(torch.bfloat16, S, maxb, Hkv, D, Bs) == pool + S * maxb * 4 + 512 + parts
    assert B.prefill_workspace_bytes("bf16", 0, 4, 2, 128, 16) == 0


def test_stream_read_checks_its_buffer(lib):
    """The read-only measurement helper refuses a misaligned buffer or size before launching."""
    P = ctypes.c_void_p
    f = lib.pkv_stream_read
    f.argtypes = [P, ctypes.c_size_t, P, P]
    assert f(P(16), 0, None, None) == 0                 # nothing to read
    assert f(None, 64, None, None) == 1
    assert f(P(24), 64, None, None) == 5                # buffer not 16-byte aligned
    assert f(P(16), 40, None, None) == 5                # size not a multiple of 16
    assert f(P(16), 64, P(18), None) == 5               # misaligned sink word
