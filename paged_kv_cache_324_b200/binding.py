"""Thin Python binding over ``libpagedkv.so`` (C ABI in ``include/pagedkv.h``).

Argument marshalling only: shapes, dtypes and pointers of torch tensors are
read here and passed to the C entry points of the same names (without the
``pkv_`` prefix); every step of the computation runs in the library's CUDA
kernels.  There is no fallback: if the library is missing or a call fails,
an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpagedkv.so")

F16, BF16, FP8_E4M3 = 0, 1, 2
DEVERR_BLOCK_ID, DEVERR_SLOT, DEVERR_PAIR, DEVERR_CONTEXT_LEN, DEVERR_TIMEOUT = 1, 2, 4, 8, 16

_TORCH_CODES = {torch.float16: F16, torch.bfloat16: BF16, torch.uint8: FP8_E4M3,
                torch.float8_e4m3fn: FP8_E4M3}


class PagedKVError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m paged_kv_cache_324_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(_LIB_PATH)
        P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.pkv_version.restype = I
        L.pkv_status_string.argtypes = [I]
        L.pkv_status_string.restype = ctypes.c_char_p
        L.pkv_decode_workspace_bytes.argtypes = [I, I, I, I, I, I, I, I]
        L.pkv_decode_workspace_bytes.restype = Z
        L.pkv_decode_partition_size.argtypes = [I, I, I, I, I, I, I]
        L.pkv_decode_partition_size.restype = I
        L.pkv_paged_attn_decode.argtypes = [P, P, I, P, P, I, F, F, P, I, P, I, I, I, I, I, I, I, F, I,
                                            P, Z, P, P]
        L.pkv_paged_attn_decode.restype = I
        L.pkv_prefill_workspace_bytes.argtypes = [I, I, I, I, I, I]
        L.pkv_prefill_workspace_bytes.restype = Z
        L.pkv_paged_attn_prefill.argtypes = [P, P, I, P, P, P, I, P, P, I, I, I, I, I, I, I, I, F, P, Z, P, P]
        L.pkv_paged_attn_prefill.restype = I
        L.pkv_prefill_fp8_workspace_bytes.argtypes = [I, I, I, I, I]
        L.pkv_prefill_fp8_workspace_bytes.restype = Z
        L.pkv_paged_attn_prefill_fp8.argtypes = [P, P, I, P, P, F, F, P, I, P, P, I, I, I, I, I, I, I, I, F, P, Z,
                                                 P, P]
        L.pkv_paged_attn_prefill_fp8.restype = I
        L.pkv_reshape_and_cache.argtypes = [P, P, I, P, P, I, F, F, P, I, I, I, I, I, P, P]
        L.pkv_reshape_and_cache.restype = I
        L.pkv_copy_blocks.argtypes = [P, P, Z, P, I, I, P, P]
        L.pkv_copy_blocks.restype = I
        L.pkv_swap_blocks.argtypes = [P, P, I, P, P, I, Z, P, I, P, P]
        L.pkv_swap_blocks.restype = I
        L.pkv_selftest_bounded_wait.argtypes = [P, ctypes.c_uint, P]
        L.pkv_selftest_bounded_wait.restype = I
        _lib = L
    return _lib


def version() -> int:
    return lib().pkv_version()


def status_string(status: int) -> str:
    return lib().pkv_status_string(status).decode()


def _code(t: torch.Tensor) -> int:
    try:
        return _TORCH_CODES[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}") from None


def _dev(t: Optional[torch.Tensor], name: str):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _err(t: Optional[torch.Tensor]):
    """The device error word: a 4-byte integer tensor on the GPU (element 0 is used), or None."""
    if t is None:
        return None
    if t.element_size() != 4 or t.dtype.is_floating_point or t.numel() < 1:
        raise TypeError("device_error must be an int32 tensor with at least one element")
    return _dev(t, "device_error")


def _tables(block_tables: torch.Tensor, context_lens: torch.Tensor, num_seqs: int):
    """Block tables int32 [>= num_seqs, max_blocks] and context lengths int32 [>= num_seqs]: the
    kernels read num_seqs rows of each."""
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    if block_tables.dim() != 2 or block_tables.shape[0] < num_seqs or block_tables.shape[1] < 1:
        raise ValueError("block_tables must be [num_seqs, max_blocks]")
    if context_lens.numel() < num_seqs:
        raise ValueError("context_lens must hold num_seqs lengths")


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, what: str):
    if status != 0:
        raise PagedKVError(status, what)


_CODES_BY_NAME = {"f16": F16, "bf16": BF16, "e4m3": FP8_E4M3}


def _kv_code(kv_dtype) -> int:
    if isinstance(kv_dtype, torch.dtype):
        return _TORCH_CODES[kv_dtype]
    return _CODES_BY_NAME[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)


def decode_partition_size(num_seqs, num_kv_heads, head_dim, kv_dtype, block_size, max_context_len,
                          partition_size=0) -> int:
    """Partition size the decode call uses; kv_dtype as a torch dtype, 'f16'/'bf16'/'e4m3' or a code."""
    return lib().pkv_decode_partition_size(num_seqs, num_kv_heads, head_dim, _kv_code(kv_dtype), block_size,
                                           max_context_len, partition_size)


def decode_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, kv_dtype, block_size, max_context_len,
                           partition_size=0) -> int:
    return lib().pkv_decode_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, _kv_code(kv_dtype),
                                            block_size, max_context_len, partition_size)


def paged_attn_decode(out: torch.Tensor, q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                      block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float, *,
                      max_context_len: int, k_scale: float = 1.0, v_scale: float = 1.0,
                      partition_size: int = 0, workspace: Optional[torch.Tensor] = None,
                      device_error: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out[S, H, D] = decode attention of q[S, H, D] over pools [NB, Hkv, B, D].

    block_tables int32 [S, max_blocks], context_lens int32 [S].  ``workspace``
    (uint8, >= decode_workspace_bytes) is allocated with torch if not given.
    """
    S, H, D = q.shape
    NB, Hkv, B, D2 = k_pool.shape
    if (out.shape != q.shape or out.dtype != q.dtype or D2 != D or v_pool.shape != k_pool.shape
            or v_pool.dtype != k_pool.dtype):
        raise ValueError("inconsistent shapes or dtypes")
    _tables(block_tables, context_lens, S)
    need = decode_workspace_bytes(S, H, Hkv, D, k_pool.dtype, B, max_context_len, partition_size)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    status = lib().pkv_paged_attn_decode(
        _dev(out, "out"), _dev(q, "q"), _code(q), _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"),
        _code(k_pool), float(k_scale), float(v_scale), _dev(block_tables, "block_tables"),
        block_tables.shape[1], _dev(context_lens, "context_lens"), int(max_context_len), S, H, Hkv, D, B,
        NB, float(scale), int(partition_size), _dev(workspace, "workspace"), ws_bytes,
        _err(device_error), _stream(stream))
    _check(status, "paged_attn_decode")
    return out


def prefill_workspace_bytes(dtype, num_seqs, max_blocks_per_seq, num_kv_heads, head_dim, block_size) -> int:
    """Bytes of device workspace with which a bf16 paged_attn_prefill narrows V to f16 (0 for f16)."""
    return lib().pkv_prefill_workspace_bytes(_kv_code(dtype), num_seqs, max_blocks_per_seq, num_kv_heads, head_dim,
                                             block_size)


def paged_attn_prefill(out: torch.Tensor, q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                       block_tables: torch.Tensor, context_lens: torch.Tensor, query_start: torch.Tensor,
                       scale: float, *, max_query_len: int, workspace="auto",
                       device_error: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out[T, H, D] = chunked causal prefill of q[T, H, D] over pools [NB, Hkv, B, D].

    The chunks of all sequences are packed in q; query_start int32 [S + 1] gives
    their row offsets, context_lens int32 [S] count each chunk's tokens (already
    in the pool).  q, out and the pools share one 16-bit dtype.  ``workspace``
    (bf16 only): a uint8 tensor of at least prefill_workspace_bytes, "auto" to
    allocate one with torch, or None for the call without one (the softmax
    weights then enter P.V as two bf16 parts instead of V being narrowed to f16).
    """
    T, H, D = q.shape
    NB, Hkv, B, D2 = k_pool.shape
    S = context_lens.numel()
    if (out.shape != q.shape or out.dtype != q.dtype or D2 != D or v_pool.shape != k_pool.shape
            or v_pool.dtype != k_pool.dtype):
        raise ValueError("inconsistent shapes or dtypes")
    if k_pool.dtype != q.dtype or v_pool.dtype != q.dtype:
        raise TypeError("prefill needs q and the pools in one 16-bit dtype")
    _tables(block_tables, context_lens, S)
    if query_start.dtype != torch.int32:
        raise TypeError("query_start must be int32")
    if query_start.numel() != S + 1:
        raise ValueError("query_start must hold num_seqs + 1 offsets")
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError('workspace must be a tensor, "auto" or None')
        need = prefill_workspace_bytes(q.dtype, S, block_tables.shape[1], Hkv, D, B)
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device) if need else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    status = lib().pkv_paged_attn_prefill(
        _dev(out, "out"), _dev(q, "q"), _code(q), _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"),
        _dev(block_tables, "block_tables"), block_tables.shape[1], _dev(context_lens, "context_lens"),
        _dev(query_start, "query_start"), int(max_query_len), S, T, H, Hkv, D, B, NB, float(scale),
        _dev(workspace, "workspace"), ws_bytes, _err(device_error), _stream(stream))
    _check(status, "paged_attn_prefill")
    return out


def prefill_fp8_workspace_bytes(num_seqs, max_blocks_per_seq, num_kv_heads, head_dim, block_size) -> int:
    """Bytes of device workspace paged_attn_prefill_fp8 needs (the widened pools and their table)."""
    return lib().pkv_prefill_fp8_workspace_bytes(num_seqs, max_blocks_per_seq, num_kv_heads, head_dim, block_size)


def paged_attn_prefill_fp8(out: torch.Tensor, q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                           block_tables: torch.Tensor, context_lens: torch.Tensor, query_start: torch.Tensor,
                           scale: float, k_scale: float, v_scale: float, *, max_query_len: int,
                           workspace: Optional[torch.Tensor] = None, device_error: Optional[torch.Tensor] = None,
                           stream=None) -> torch.Tensor:
    """Chunked prefill as paged_attn_prefill over E4M3 pools (uint8 [NB, Hkv, B, D]) with per-tensor
    scales; q and out are f16 or bf16.  ``workspace`` (uint8) is allocated with torch if not given."""
    T, H, D = q.shape
    NB, Hkv, B, D2 = k_pool.shape
    S = context_lens.numel()
    if (out.shape != q.shape or out.dtype != q.dtype or D2 != D or v_pool.shape != k_pool.shape
            or v_pool.dtype != k_pool.dtype):
        raise ValueError("inconsistent shapes or dtypes")
    if k_pool.dtype != torch.uint8 or v_pool.dtype != torch.uint8:
        raise TypeError("the pools hold E4M3 bytes (uint8)")
    _tables(block_tables, context_lens, S)
    if query_start.dtype != torch.int32:
        raise TypeError("query_start must be int32")
    if query_start.numel() != S + 1:
        raise ValueError("query_start must hold num_seqs + 1 offsets")
    if q.dtype not in (torch.float16, torch.bfloat16):
        raise TypeError("q and out must be float16 or bfloat16")
    need = prefill_fp8_workspace_bytes(S, block_tables.shape[1], Hkv, D, B)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    status = lib().pkv_paged_attn_prefill_fp8(
        _dev(out, "out"), _dev(q, "q"), _code(q), _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"), float(k_scale),
        float(v_scale), _dev(block_tables, "block_tables"), block_tables.shape[1], _dev(context_lens, "context_lens"),
        _dev(query_start, "query_start"), int(max_query_len), S, T, H, Hkv, D, B, NB, float(scale),
        _dev(workspace, "workspace"), workspace.numel(), _err(device_error), _stream(stream))
    _check(status, "paged_attn_prefill_fp8")
    return out


def reshape_and_cache(k: torch.Tensor, v: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                      slot_mapping: torch.Tensor, k_scale: float = 1.0, v_scale: float = 1.0, *,
                      device_error: Optional[torch.Tensor] = None, stream=None) -> None:
    """Write k, v [T, Hkv, D] into the pools [NB, Hkv, B, D] at slot_mapping (int64 [T])."""
    T, Hkv, D = k.shape
    NB, Hkv2, B, D2 = k_pool.shape
    if (Hkv2, D2) != (Hkv, D) or v.shape != k.shape or v_pool.shape != k_pool.shape:
        raise ValueError("inconsistent shapes")
    if v.dtype != k.dtype or v_pool.dtype != k_pool.dtype:
        raise ValueError("k and v (and the two pools) must share a dtype")
    if slot_mapping.dtype != torch.int64 or slot_mapping.numel() != T:
        raise TypeError("slot_mapping must be int64 [T]")
    status = lib().pkv_reshape_and_cache(
        _dev(k, "k"), _dev(v, "v"), _code(k), _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"),
        _code(k_pool), float(k_scale), float(v_scale), _dev(slot_mapping, "slot_mapping"), T, Hkv, D, B, NB,
        _err(device_error), _stream(stream))
    _check(status, "reshape_and_cache")


def check_block_pairs(pairs, src_num_blocks: int, dst_num_blocks: int, same_pool: bool) -> None:
    """Raise ValueError unless the (src, dst) rows of pairs (int64 [n, 2], any device; copied to the
    host, which synchronises) are in range, the destinations distinct and, within one pool, no
    destination also a source (pkv_check_block_pairs)."""
    import numpy as np
    h = pairs.detach().cpu().numpy() if isinstance(pairs, torch.Tensor) else np.asarray(pairs)
    h = np.ascontiguousarray(h, dtype=np.int64).reshape(-1, 2)
    f = lib().pkv_check_block_pairs
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    f.restype = ctypes.c_int
    if f(h.ctypes.data if h.size else None, h.shape[0], int(src_num_blocks), int(dst_num_blocks),
         1 if same_pool else 0) != 0:
        raise ValueError("block pairs: an id out of range, a repeated destination, or (one pool) a "
                         "destination that is also a source")


def _debug_checks() -> bool:
    return os.environ.get("PKV_DEBUG", "") not in ("", "0")


def copy_blocks(k_pool: torch.Tensor, v_pool: torch.Tensor, pairs: torch.Tensor, *,
                device_error: Optional[torch.Tensor] = None, stream=None, check: Optional[bool] = None) -> None:
    """k_pool[dst] := k_pool[src] (and v) for each row (src, dst) of pairs (int64 [n, 2]).  With
    ``check`` (default: the PKV_DEBUG environment variable) the pairs are first checked on the host."""
    if pairs.dtype != torch.int64 or (pairs.numel() and pairs.shape[-1] != 2):
        raise TypeError("pairs must be int64 [n, 2]")
    if v_pool.shape != k_pool.shape or v_pool.dtype != k_pool.dtype:
        raise ValueError("k_pool and v_pool must have one shape and dtype")
    if check or (check is None and _debug_checks()):
        check_block_pairs(pairs, k_pool.shape[0], k_pool.shape[0], True)
    block_bytes = k_pool[0].numel() * k_pool.element_size()
    status = lib().pkv_copy_blocks(
        _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"), block_bytes, _dev(pairs, "pairs"),
        pairs.numel() // 2, k_pool.shape[0], _err(device_error), _stream(stream))
    _check(status, "copy_blocks")


def swap_blocks(src_k: torch.Tensor, src_v: torch.Tensor, dst_k: torch.Tensor, dst_v: torch.Tensor,
                pairs: torch.Tensor, *, device_error: Optional[torch.Tensor] = None, stream=None,
                check: Optional[bool] = None) -> None:
    """dst[d] := src[s] (K and V pools [NB, Hkv, B, D], whole blocks) for each row (s, d) of pairs
    (int64 [n, 2], on the GPU).  Either side may be pinned host memory (``pin_memory()``).  With
    ``check`` (default: PKV_DEBUG) the pairs are first checked on the host."""
    if pairs.dtype != torch.int64 or (pairs.numel() and pairs.shape[-1] != 2):
        raise TypeError("pairs must be int64 [n, 2]")
    if check or (check is None and _debug_checks()):
        check_block_pairs(pairs, src_k.shape[0], dst_k.shape[0], src_k.data_ptr() == dst_k.data_ptr())
    if src_k.shape[1:] != dst_k.shape[1:] or src_k.dtype != dst_k.dtype or src_v.shape != src_k.shape \
            or dst_v.shape != dst_k.shape or src_v.dtype != src_k.dtype or dst_v.dtype != dst_k.dtype:
        raise ValueError("pools of one layout and dtype")
    for t, name in ((src_k, "src_k"), (src_v, "src_v"), (dst_k, "dst_k"), (dst_v, "dst_v")):
        if not t.is_cuda and not t.is_pinned():
            raise ValueError(f"{name} must be on the GPU or in pinned host memory")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    block_bytes = src_k[0].numel() * src_k.element_size()
    status = lib().pkv_swap_blocks(
        ctypes.c_void_p(src_k.data_ptr()), ctypes.c_void_p(src_v.data_ptr()), src_k.shape[0],
        ctypes.c_void_p(dst_k.data_ptr()), ctypes.c_void_p(dst_v.data_ptr()), dst_k.shape[0], block_bytes,
        _dev(pairs, "pairs"), pairs.numel() // 2, _err(device_error), _stream(stream))
    _check(status, "swap_blocks")


def selftest_bounded_wait(device_error: torch.Tensor, timeout_us: int, stream=None) -> None:
    """Run one bounded wait that nothing completes; it sets DEVERR_TIMEOUT in device_error."""
    _check(lib().pkv_selftest_bounded_wait(_err(device_error), int(timeout_us), _stream(stream)),
           "selftest_bounded_wait")


def stream_read(buf: torch.Tensor, sink: Optional[torch.Tensor] = None, stream=None) -> None:
    """Read every byte of ``buf`` (a contiguous device tensor) once: the read-only HBM rate."""
    if not buf.is_cuda or not buf.is_contiguous():
        raise ValueError("buf must be a contiguous device tensor")
    L = lib()
    L.pkv_stream_read.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]
    _check(L.pkv_stream_read(ctypes.c_void_p(buf.data_ptr()), buf.numel() * buf.element_size(), _err(sink),
                             _stream(stream)), "stream_read")


class BlockManager:
    """Host-side block manager of the library (pkv_bm_* in include/pagedkv.h)."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        import numpy as np
        L = lib()
        P, I, I64, I32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int32
        L.pkv_bm_create.argtypes = [I, I, P]
        L.pkv_bm_create.restype = P
        L.pkv_bm_destroy.argtypes = [P]
        L.pkv_bm_num_free.argtypes = [P]
        L.pkv_bm_add_sequence.argtypes = [P, I64]
        L.pkv_bm_fork.argtypes = [P, I64, I64]
        L.pkv_bm_append_slots.argtypes = [P, P, I, P, P, I, P]
        L.pkv_bm_free_sequence.argtypes = [P, I64]
        L.pkv_bm_block_tables.argtypes = [P, P, I, P, I, I32, P]
        L.pkv_bm_ref_count.argtypes = [P, I32]
        L.pkv_bm_sequence_length.argtypes = [P, I64]
        L.pkv_bm_sequence_length.restype = I64
        L.pkv_bm_num_cached.argtypes = [P]
        L.pkv_bm_add_sequence_cached.argtypes = [P, I64, P, I, P]
        L.pkv_bm_cache_sequence.argtypes = [P, I64, P, I]
        L.pkv_bm_swap.argtypes = [P, P, P, I, P, I, P]
        L.pkv_bm_append_tokens.argtypes = [P, I64, I, P, P, I, P]
        L.pkv_bm_append_tokens.restype = I
        self._L, self._np = L, np
        order = None
        if free_order is not None:
            order = np.ascontiguousarray(free_order, dtype=np.int32).reshape(-1)
            if order.size != num_blocks:            # the library reads num_blocks entries
                raise ValueError("free_order must hold num_blocks entries")
        self.block_size = block_size
        self._h = L.pkv_bm_create(num_blocks, block_size,
                                  order.ctypes.data_as(P) if order is not None else None)
        if not self._h:
            raise ValueError("invalid block manager arguments (free_order must be a permutation)")

    def __del__(self):
        if getattr(self, "_h", None):
            self._L.pkv_bm_destroy(self._h)
            self._h = None

    def _ok(self, status, what):
        _check(status, what)

    @property
    def num_free(self) -> int:
        return self._L.pkv_bm_num_free(self._h)

    def add_sequence(self, seq_id: int):
        self._ok(self._L.pkv_bm_add_sequence(self._h, seq_id), "add_sequence")

    def fork(self, parent: int, child: int):
        self._ok(self._L.pkv_bm_fork(self._h, parent, child), "fork")

    def append_slots(self, seq_ids):
        """One new token per sequence: (slots int64 [n], copy pairs int64 [k, 2])."""
        np = self._np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.size
        slots = np.empty(n, np.int64)
        pairs = np.empty((max(n, 1), 2), np.int64)
        k = ctypes.c_int(0)
        P = ctypes.c_void_p
        self._ok(self._L.pkv_bm_append_slots(self._h, ids.ctypes.data_as(P), n, slots.ctypes.data_as(P),
                                             pairs.ctypes.data_as(P), pairs.shape[0], ctypes.byref(k)),
                 "append_slots")
        return slots, pairs[:k.value].copy()

    def append_tokens(self, seq_id: int, n: int):
        """n new tokens for one sequence (a prefill chunk): (slots int64 [n], copy pairs int64 [k, 2])."""
        np = self._np
        slots = np.empty(max(int(n), 1), np.int64)
        pairs = np.empty((1, 2), np.int64)
        k = ctypes.c_int(0)
        P = ctypes.c_void_p
        self._ok(self._L.pkv_bm_append_tokens(self._h, seq_id, int(n), slots.ctypes.data_as(P),
                                              pairs.ctypes.data_as(P), 1, ctypes.byref(k)), "append_tokens")
        return slots[:int(n)].copy(), pairs[:k.value].copy()

    def free_sequence(self, seq_id: int):
        self._ok(self._L.pkv_bm_free_sequence(self._h, seq_id), "free_sequence")

    def block_tables(self, seq_ids, max_blocks: int, pad: int = -1):
        """(int32 [n, max_blocks] tables, int32 [n] lengths)."""
        np = self._np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        t = np.empty((ids.size, max_blocks), np.int32)
        lens = np.empty(ids.size, np.int32)
        P = ctypes.c_void_p
        self._ok(self._L.pkv_bm_block_tables(self._h, ids.ctypes.data_as(P), ids.size, t.ctypes.data_as(P),
                                             max_blocks, pad, lens.ctypes.data_as(P)), "block_tables")
        return t, lens

    def ref_count(self, block: int) -> int:
        return self._L.pkv_bm_ref_count(self._h, block)

    def sequence_length(self, seq_id: int) -> int:
        return self._L.pkv_bm_sequence_length(self._h, seq_id)

    # prefix caching by block content
    @property
    def num_cached(self) -> int:
        return self._L.pkv_bm_num_cached(self._h)

    def add_sequence_cached(self, seq_id: int, tokens) -> int:
        """A new sequence for a prompt of token ids; returns how many of its leading tokens
        are already cached (whole blocks, shared), which is the sequence's length."""
        np = self._np
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        n = ctypes.c_int(0)
        self._ok(self._L.pkv_bm_add_sequence_cached(self._h, seq_id, t.ctypes.data_as(ctypes.c_void_p), t.size,
                                                    ctypes.byref(n)), "add_sequence_cached")
        return n.value

    def cache_sequence(self, seq_id: int, tokens):
        """Register the full blocks holding tokens[0 .. len(tokens)) of the sequence."""
        np = self._np
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        self._ok(self._L.pkv_bm_cache_sequence(self._h, seq_id, t.ctypes.data_as(ctypes.c_void_p), t.size),
                 "cache_sequence")

    def swap_to(self, other: "BlockManager", seq_ids):
        """Move the sequences to ``other``; returns the (block here, block there) pairs, int64 [k, 2]."""
        np = self._np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        cap = max(1, sum(-(-max(self.sequence_length(int(i)), 0) // self.block_size) for i in ids))
        pairs = np.empty((cap, 2), np.int64)
        k = ctypes.c_int(0)
        P = ctypes.c_void_p
        self._ok(self._L.pkv_bm_swap(self._h, other._h, ids.ctypes.data_as(P), ids.size, pairs.ctypes.data_as(P),
                                     cap, ctypes.byref(k)), "swap")
        return pairs[:k.value].copy()


def find_shared_prefixes(block_tables, context_lens, block_size: int, unit_width: int):
    """Host arrays in, (seq_prefix_len int32 [S], unit_seqs int32 [U, W], unit_len int32 [U], max_prefix_len)."""
    import numpy as np
    L = lib()
    P, I = ctypes.c_void_p, ctypes.c_int
    L.pkv_find_shared_prefixes.argtypes = [P, P, I, I, I, I, P, P, P, I, P, P]
    t = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    S, maxb = t.shape
    cap = max(S, 1)
    spl = np.empty(S, np.int32)
    us = np.empty((cap, unit_width), np.int32)
    ul = np.empty(cap, np.int32)
    nu, mp = ctypes.c_int(0), ctypes.c_int(0)
    _check(L.pkv_find_shared_prefixes(t.ctypes.data_as(P), lens.ctypes.data_as(P), S, maxb, block_size, unit_width,
                                      spl.ctypes.data_as(P), us.ctypes.data_as(P), ul.ctypes.data_as(P), cap,
                                      ctypes.byref(nu), ctypes.byref(mp)), "find_shared_prefixes")
    return spl, us[:nu.value].copy(), ul[:nu.value].copy(), mp.value


def shared_prefix_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, kv_dtype, block_size,
                                  max_context_len, num_units, max_prefix_len, partition_size=0) -> int:
    L = lib()
    I = ctypes.c_int
    L.pkv_shared_prefix_workspace_bytes.argtypes = [I, I, I, I, I, I, I, I, I, I]
    L.pkv_shared_prefix_workspace_bytes.restype = ctypes.c_size_t
    return L.pkv_shared_prefix_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, _kv_code(kv_dtype),
                                               block_size, max_context_len, num_units, max_prefix_len,
                                               partition_size)


#: pkv_prefix_plan codes
PREFIX_PLANS = {"auto": 0, "shared": 1, "plain": 2}


def shared_prefix_plan_used(num_units: int, num_kv_heads: int, head_dim: int, kv_dtype, max_prefix_len: int,
                            plan: str = "auto") -> str:
    """"shared" or "plain": what paged_attn_decode_shared_prefix does for these arguments."""
    L = lib()
    I = ctypes.c_int
    L.pkv_shared_prefix_plan_used.argtypes = [I, I, I, I, I, I]
    L.pkv_shared_prefix_plan_used.restype = I
    r = L.pkv_shared_prefix_plan_used(num_units, num_kv_heads, head_dim, _kv_code(kv_dtype), max_prefix_len,
                                      PREFIX_PLANS[plan])
    return {1: "shared", 2: "plain"}[r]


def paged_attn_decode_shared_prefix(out, q, k_pool, v_pool, block_tables, context_lens, scale, *,
                                    max_context_len: int, seq_prefix_len, unit_seqs, unit_len,
                                    max_prefix_len: int, k_scale: float = 1.0, v_scale: float = 1.0,
                                    partition_size: int = 0, plan: str = "auto", workspace=None, device_error=None,
                                    stream=None):
    """Shared-prefix decode: device tensors; seq_prefix_len int32 [S], unit_seqs int32 [U, W], unit_len int32 [U].
    plan: "auto" (the library picks the shared-prefix passes or the plain call), "shared" or "plain"."""
    L = lib()
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.pkv_paged_attn_decode_shared_prefix.argtypes = [P, P, I, P, P, I, F, F, P, I, P, I, I, I, I, I, I, I, F, I,
                                                      P, P, P, I, I, I, I, P, Z, P, P]
    if plan not in PREFIX_PLANS:
        raise ValueError(f"plan must be one of {sorted(PREFIX_PLANS)}")
    S, H, D = q.shape
    NB, Hkv, B, D2 = k_pool.shape
    if (out.shape != q.shape or out.dtype != q.dtype or D2 != D or v_pool.shape != k_pool.shape
            or v_pool.dtype != k_pool.dtype):
        raise ValueError("inconsistent shapes or dtypes")
    _tables(block_tables, context_lens, S)
    for t, name in ((seq_prefix_len, "seq_prefix_len"), (unit_seqs, "unit_seqs"), (unit_len, "unit_len")):
        if t.dtype != torch.int32:
            raise TypeError(f"{name} must be int32")
    if seq_prefix_len.numel() < S:
        raise ValueError("seq_prefix_len must hold num_seqs entries")
    need = shared_prefix_workspace_bytes(S, H, Hkv, D, k_pool.dtype, B, max_context_len, unit_len.numel(),
                                         max_prefix_len, partition_size)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    U = unit_len.numel()
    W = unit_seqs.shape[1] if unit_seqs.dim() == 2 and U else 1
    status = L.pkv_paged_attn_decode_shared_prefix(
        _dev(out, "out"), _dev(q, "q"), _code(q), _dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"), _code(k_pool),
        float(k_scale), float(v_scale), _dev(block_tables, "block_tables"), block_tables.shape[1],
        _dev(context_lens, "context_lens"), int(max_context_len), S, H, Hkv, D, B, NB, float(scale),
        int(partition_size), _dev(seq_prefix_len, "seq_prefix_len"),
        _dev(unit_seqs, "unit_seqs") if U else None, _dev(unit_len, "unit_len") if U else None, U, W,
        int(max_prefix_len), PREFIX_PLANS[plan], _dev(workspace, "workspace"), workspace.numel(),
        _err(device_error), _stream(stream))
    _check(status, "paged_attn_decode_shared_prefix")
    return out
