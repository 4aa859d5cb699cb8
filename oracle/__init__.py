"""ORACLE -- test infrastructure, not product code.

Python access to the float64 CPU oracle in ``pagedkv_oracle.c``: the plain
definition of paged decode attention (gather through the block table, then
textbook two-pass softmax) and of chunked prefill over the same cache, the
scatter of new tokens into the pool, the block copy used for copy-on-write,
the block swap between two pools, and the number-format codecs.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package.  It shares no code with the CUDA
library and never imports it.

Sources are cited in the C file's header: the Ultralytics glossary entry
"PagedAttention" (worked example of the pool, table, scatter and gather), the
Wikipedia article "PagedAttention", section "Mathematical formulation" (token
form of causal attention), the podcast transcript "vLLM and PagedAttention"
(copy of the shared partial block), and the OCP 8-bit floating point
specification (E4M3).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pagedkv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F16, BF16, E4M3 = 0, 1, 2
DTYPE_CODES = {"f16": F16, "bf16": BF16, "e4m3": E4M3}
_ERRORS = {1: "bad argument", 2: "block id out of range", 3: "slot out of range",
           4: "context length beyond table capacity"}


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile the oracle with the host C compiler (never nvcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I, D, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_float, ctypes.c_size_t
        lib.orc_paged_attn_decode.argtypes = [P, P, I, P, P, I, D, D, P, I, P, I, I, I, I, I, I, D, I]
        lib.orc_paged_attn_decode.restype = I
        lib.orc_paged_attn_prefill.argtypes = [P, P, I, P, P, I, D, D, P, I, P, P, I, I, I, I, I, I, D, I]
        lib.orc_paged_attn_prefill.restype = I
        lib.orc_reshape_and_cache.argtypes = [P, P, I, P, P, I, F, F, P, I, I, I, I, I]
        lib.orc_reshape_and_cache.restype = I
        lib.orc_copy_blocks.argtypes = [P, P, Z, P, I, I]
        lib.orc_copy_blocks.restype = I
        lib.orc_swap_blocks.argtypes = [P, P, I, P, P, I, Z, P, I]
        lib.orc_swap_blocks.restype = I
        lib.orc_gather.argtypes = [P, P, I, P, I, I, I, I, I, I, I]
        lib.orc_gather.restype = I
        lib.orc_decode_array.argtypes = [P, P, I, Z]
        lib.orc_decode_array.restype = None
        lib.orc_encode_e4m3_array.argtypes = [P, P, Z]
        lib.orc_encode_e4m3_array.restype = None
        _lib = lib
    return _lib


def _threads(n) -> int:
    """OpenMP threads for one call: n, or every host core when n is 0 (so that an earlier call's
    count does not carry over)."""
    return int(n) if n else (os.cpu_count() or 1)


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int):
    if rc != 0:
        raise OracleError(_ERRORS.get(rc, f"error {rc}"))


def _code(dtype) -> int:
    return DTYPE_CODES[dtype] if isinstance(dtype, str) else int(dtype)


def decode_values(bits: np.ndarray, dtype) -> np.ndarray:
    """Exact float64 values of raw f16 / bf16 (uint16) or e4m3 (uint8) bit patterns."""
    bits = np.ascontiguousarray(bits)
    out = np.empty(bits.shape, np.float64)
    _load().orc_decode_array(_ptr(out), _ptr(bits), _code(dtype), bits.size)
    return out


def encode_e4m3(x: np.ndarray) -> np.ndarray:
    """float32 -> E4M3 bytes, round-to-nearest-even, saturating at +-448."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint8)
    _load().orc_encode_e4m3_array(_ptr(out), _ptr(x), x.size)
    return out


def paged_attn_decode(q_bits, q_dtype, k_pool, v_pool, kv_dtype, block_tables, context_lens,
                      scale, k_scale=1.0, v_scale=1.0, threads=0) -> np.ndarray:
    """float64 out[S, H, D] of decode attention over the paged pool.

    q_bits: uint16 [S, H, D]; pools: uint16 (f16/bf16) or uint8 (e4m3)
    [NB, Hkv, B, D]; block_tables int32 [S, max_blocks]; context_lens int32 [S].
    ``scale``, ``k_scale`` and ``v_scale`` are used exactly as given (pass the
    float32 values the GPU receives).
    """
    q_bits = np.ascontiguousarray(q_bits)
    k_pool = np.ascontiguousarray(k_pool)
    v_pool = np.ascontiguousarray(v_pool)
    block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    S, H, D = q_bits.shape
    NB, Hkv, B, D2 = k_pool.shape
    assert D2 == D and v_pool.shape == k_pool.shape
    out = np.empty((S, H, D), np.float64)
    _check(_load().orc_paged_attn_decode(
        _ptr(out), _ptr(q_bits), _code(q_dtype), _ptr(k_pool), _ptr(v_pool), _code(kv_dtype),
        float(k_scale), float(v_scale), _ptr(block_tables), block_tables.shape[1],
        _ptr(context_lens), S, H, Hkv, D, B, NB, float(scale), _threads(threads)))
    return out


def paged_attn_prefill(q_bits, q_dtype, k_pool, v_pool, kv_dtype, block_tables, context_lens,
                       query_start, scale, k_scale=1.0, v_scale=1.0, threads=0) -> np.ndarray:
    """float64 out[T, H, D] of chunked prefill over the paged pool.

    q_bits: uint16 [T, H, D], the chunks of all sequences packed in order;
    query_start: int32 [S + 1], row offsets of each sequence's chunk (starts at
    0, ends at T); context_lens int32 [S] count the chunk's tokens, which are
    already in the pool.  Row query_start[s] + j attends to positions
    0 .. context_lens[s] - C_s + j of sequence s.
    """
    q_bits = np.ascontiguousarray(q_bits)
    k_pool = np.ascontiguousarray(k_pool)
    v_pool = np.ascontiguousarray(v_pool)
    block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    query_start = np.ascontiguousarray(query_start, dtype=np.int32)
    T, H, D = q_bits.shape
    NB, Hkv, B, D2 = k_pool.shape
    S = context_lens.shape[0]
    assert D2 == D and v_pool.shape == k_pool.shape
    assert query_start.shape == (S + 1,) and int(query_start[-1]) == T
    out = np.empty((T, H, D), np.float64)
    _check(_load().orc_paged_attn_prefill(
        _ptr(out), _ptr(q_bits), _code(q_dtype), _ptr(k_pool), _ptr(v_pool), _code(kv_dtype),
        float(k_scale), float(v_scale), _ptr(block_tables), block_tables.shape[1],
        _ptr(context_lens), _ptr(query_start), S, H, Hkv, D, B, NB, float(scale), _threads(threads)))
    return out


def reshape_and_cache(k_bits, v_bits, in_dtype, k_pool, v_pool, kv_dtype, slot_mapping,
                      k_scale=1.0, v_scale=1.0) -> None:
    """Scatter k/v [T, Hkv, D] into the pools in place through slot_mapping (int64 [T])."""
    k_bits = np.ascontiguousarray(k_bits)
    v_bits = np.ascontiguousarray(v_bits)
    slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    T, Hkv, D = k_bits.shape
    NB, Hkv2, B, D2 = k_pool.shape
    assert (Hkv2, D2) == (Hkv, D)
    _check(_load().orc_reshape_and_cache(
        _ptr(k_bits), _ptr(v_bits), _code(in_dtype), _ptr(k_pool), _ptr(v_pool), _code(kv_dtype),
        float(k_scale), float(v_scale), _ptr(slot_mapping), T, Hkv, D, B, NB))


def copy_blocks(k_pool, v_pool, pairs) -> None:
    """pool[dst] := pool[src] for each row (src, dst) of pairs (int64 [n, 2]), in place."""
    pairs = np.ascontiguousarray(pairs, dtype=np.int64).reshape(-1, 2)
    NB = k_pool.shape[0]
    block_bytes = k_pool[0].nbytes
    _check(_load().orc_copy_blocks(_ptr(k_pool), _ptr(v_pool), block_bytes, _ptr(pairs),
                                   pairs.shape[0], NB))


def swap_blocks(src_k, src_v, dst_k, dst_v, pairs) -> None:
    """dst[d] := src[s] (K and V, whole blocks) for each row (s, d) of pairs, in place in dst."""
    pairs = np.ascontiguousarray(pairs, dtype=np.int64).reshape(-1, 2)
    assert src_k.shape[1:] == dst_k.shape[1:] and src_k.dtype == dst_k.dtype
    _check(_load().orc_swap_blocks(_ptr(np.ascontiguousarray(src_k)), _ptr(np.ascontiguousarray(src_v)),
                                   src_k.shape[0], _ptr(dst_k), _ptr(dst_v), dst_k.shape[0], src_k[0].nbytes,
                                   _ptr(pairs), pairs.shape[0]))


def gather(pool, kv_dtype, table, length, kvh=0) -> np.ndarray:
    """Rows 0..length-1 of one KV head read back through a block table (raw bits)."""
    table = np.ascontiguousarray(table, dtype=np.int32)
    NB, Hkv, B, D = pool.shape
    out = np.empty((length, D), pool.dtype)
    _check(_load().orc_gather(_ptr(out), _ptr(np.ascontiguousarray(pool)), _code(kv_dtype),
                              _ptr(table), table.size, int(length), Hkv, int(kvh), D, B, NB))
    return out
