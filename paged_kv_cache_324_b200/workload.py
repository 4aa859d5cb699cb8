"""Seeded synthetic workloads for the paged decode path.

This module is shared by the tests (which feed the same inputs to the CUDA
library and to the CPU oracle), the benchmark and the smoke check.  It holds
none of the attention, scatter, copy or quantisation arithmetic: it draws
random numbers (numpy PCG64), rounds them to the input dtype with library
casts, allocates physical blocks from a free list, keeps reference counts for
shared blocks, and lists the operations of a decode step.

Shapes follow the pages' workloads: the OPT-13B layer (40 heads x 128,
fp16; "vLLM and PagedAttention" transcript), GQA and FP8 caches (Ultralytics
glossary "PagedAttention", section "Related methods"), shared-prefix parallel
sampling with copy-on-write of the partially filled shared block
(glossary, section "Sharing blocks across sequences"; transcript), blocks of
16 tokens taken only when the previous block is full (glossary, section
"How paging works").
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Tuple

import numpy as np

ELEM_BYTES = {"f16": 2, "bf16": 2, "e4m3": 1}
#: byte value never produced by an allocator: block-table entries past a
#: sequence's last block are filled with it, so a kernel that reads them fails.
TABLE_POISON = np.int32(0x7FFFFFF0)


# ---------------------------------------------------------------------------
# random values
# ---------------------------------------------------------------------------

def normal_bits(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    """N(0,1) float32 draws rounded (library cast, nearest-even) to f16/bf16; raw uint16 bits."""
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if dtype == "f16":
        return x.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        import torch
        return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    raise ValueError(dtype)


def garbage_bytes(rng: np.random.Generator, nbytes: int) -> np.ndarray:
    """Uniform random bytes: pool content outside the written slots (may decode to NaN/Inf)."""
    return np.frombuffer(rng.bytes(int(nbytes)), dtype=np.uint8).copy()


def amax_scale(bits: np.ndarray, dtype: str) -> np.float32:
    """Per-tensor FP8 scale amax(|x|) / 448 of 16-bit values (a calibration choice of the caller)."""
    if dtype == "f16":
        a = float(np.abs(bits.view(np.float16).astype(np.float32)).max())
    else:
        import torch
        t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().abs().max()
        a = float(t)
    return np.float32(a / 448.0) if a > 0 else np.float32(1.0)


# ---------------------------------------------------------------------------
# block allocation (the host side of paging: free list, tables, ref counts)
# ---------------------------------------------------------------------------

class BlockAllocator:
    """Free list of physical block ids with per-block reference counts.

    A sequence takes a new block only when its last block is full (glossary
    "PagedAttention", section "How paging works"); blocks are popped from the
    front of the free list, as in the glossary's worked example.  A write to a
    block that other sequences also reference (ref count > 1) first gets a
    private copy: the writer is given a fresh block and a (src, dst) copy pair
    (glossary, section "Sharing blocks across sequences"; the transcript says
    only the partially filled shared block is copied).
    """

    def __init__(self, free_ids):
        self.free: List[int] = [int(i) for i in free_ids]
        self.ref = {}

    def allocate(self) -> int:
        if not self.free:
            raise MemoryError("block pool exhausted")
        b = self.free.pop(0)
        self.ref[b] = 1
        return b

    def fork(self, table: List[int]) -> List[int]:
        """A new sequence sharing every block of ``table``."""
        for b in table:
            self.ref[b] += 1
        return list(table)

    def slot_for_append(self, table: List[int], pos: int, block_size: int,
                        pairs: List[Tuple[int, int]]) -> int:
        """Physical slot for token ``pos`` (= current length) of the sequence owning ``table``."""
        j, off = divmod(pos, block_size)
        if j == len(table):
            table.append(self.allocate())
        elif j < len(table) - 1 or j > len(table):
            raise ValueError("append must target the last block")
        b = table[j]
        if self.ref[b] > 1:                      # shared: copy before write
            nb = self.allocate()
            pairs.append((b, nb))
            self.ref[b] -= 1
            table[j] = nb
            b = nb
        return b * block_size + off


def tables_array(tables: List[List[int]], max_blocks: int) -> np.ndarray:
    t = np.full((len(tables), max(1, max_blocks)), TABLE_POISON, dtype=np.int32)
    for s, row in enumerate(tables):
        t[s, :len(row)] = row
    return t


# ---------------------------------------------------------------------------
# a decode step: setup operations, then the step itself
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Scatter:
    """New tokens' K/V ([T, Hkv, D] raw 16-bit bits) and their slots (int64 [T])."""
    k: np.ndarray
    v: np.ndarray
    slots: np.ndarray


@dataclasses.dataclass
class Copy:
    """Block copy pairs (int64 [n, 2], rows (src, dst))."""
    pairs: np.ndarray


@dataclasses.dataclass
class DecodeWorkload:
    name: str
    seed: int
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    q_dtype: str                 # 'f16' | 'bf16'
    kv_dtype: str                # 'f16' | 'bf16' | 'e4m3'
    src_dtype: str               # 16-bit type of the K/V values before any FP8 storage
    scale: np.float32
    k_scale: np.float32
    v_scale: np.float32
    context_lens: np.ndarray     # int32 [S], includes the step's new token
    block_tables: np.ndarray     # int32 [S, max_blocks]
    q: np.ndarray                # uint16 [S, H, D]
    setup: list                  # Scatter / Copy operations that build the cache
    step_copy: Optional[Copy]    # block copies inside the step (None = none)
    step_scatter: Scatter        # the step's appended tokens (one per sequence)
    partition_size: int = 0      # split-context partition (tokens) the workload states; 0 = automatic
    description: str = ""
    kv_head_range: Optional[Tuple[int, int]] = None   # a head shard: its KV heads in the full pools
    pool_heads: int = 0          # KV heads of the full pools a shard is cut from (0 = num_kv_heads)

    @property
    def max_blocks(self) -> int:
        return self.block_tables.shape[1]

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def pool_shape(self):
        return (self.num_blocks, self.num_kv_heads, self.block_size, self.head_dim)

    @property
    def pool_bytes(self) -> int:
        return int(np.prod(self.pool_shape)) * ELEM_BYTES[self.kv_dtype]

    def initial_pool(self, which: str) -> np.ndarray:
        """Pool content before any write: random bytes (seeded per pool; a 32 MiB random
        chunk repeated, so that large pools are cheap to make).  Unwritten slots therefore
        hold arbitrary bit patterns, NaN and Inf included."""
        rng = np.random.default_rng([self.seed, 1 if which == "k" else 2])
        full = (self.num_blocks, self.pool_heads or self.num_kv_heads, self.block_size, self.head_dim)
        nbytes = int(np.prod(full)) * ELEM_BYTES[self.kv_dtype]
        chunk = garbage_bytes(rng, min(nbytes, 32 << 20))
        raw = np.resize(chunk, nbytes)
        dt = np.uint8 if self.kv_dtype == "e4m3" else np.uint16
        pool = raw.view(dt).reshape(full)
        if self.kv_head_range is None:
            return pool
        k0, k1 = self.kv_head_range
        return np.ascontiguousarray(pool[:, k0:k1])


def shard_heads(w: DecodeWorkload, rank: int, world: int) -> DecodeWorkload:
    """Rank ``rank`` of ``world``'s share of a decode workload split by KV head: KV heads
    [rank * Hkv / world, (rank + 1) * Hkv / world) with the query heads that use them (query head
    h uses KV head h / G), the same sequences, lengths and block tables, and the same slice of
    every pool, new token and query.  Attention of each (sequence, KV head) is independent, so
    the shards' outputs side by side along the head axis are the whole workload's."""
    if w.kv_head_range is not None:
        raise ValueError("already a shard")
    if world <= 0 or not 0 <= rank < world or w.num_kv_heads % world:
        raise ValueError(f"{w.num_kv_heads} KV heads do not split over {world} ranks")
    n = w.num_kv_heads // world
    G = w.num_heads // w.num_kv_heads
    k0, k1 = rank * n, (rank + 1) * n

    def cut(op):
        if not isinstance(op, Scatter):
            return op                                  # block copies move whole blocks: every head
        return Scatter(np.ascontiguousarray(op.k[:, k0:k1]), np.ascontiguousarray(op.v[:, k0:k1]), op.slots)

    return dataclasses.replace(
        w, name=f"{w.name}_kv{k0}-{k1}", num_heads=n * G, num_kv_heads=n,
        q=np.ascontiguousarray(w.q[:, k0 * G:k1 * G]), setup=[cut(op) for op in w.setup],
        step_scatter=cut(w.step_scatter), kv_head_range=(k0, k1), pool_heads=w.num_kv_heads,
        description=f"{w.description}; KV heads {k0}..{k1 - 1} of {w.num_kv_heads}")


def _new_values(rng, tokens, hkv, d, dtype):
    return normal_bits(rng, (tokens, hkv, d), dtype), normal_bits(rng, (tokens, hkv, d), dtype)


def _finish(name, seed, rng, S, H, Hkv, D, B, NB, q_dtype, kv_dtype, lens, tables,
            setup, step_copy, new_slots, description, partition_size=0):
    src_dtype = q_dtype if kv_dtype != "e4m3" else "f16"
    q = normal_bits(rng, (S, H, D), q_dtype)
    nk, nv = _new_values(rng, len(new_slots), Hkv, D, src_dtype)
    step = Scatter(nk, nv, np.asarray(new_slots, dtype=np.int64))
    k_scale = v_scale = np.float32(1.0)
    if kv_dtype == "e4m3":
        ks = [op.k for op in setup if isinstance(op, Scatter)] + [nk]
        vs = [op.v for op in setup if isinstance(op, Scatter)] + [nv]
        k_scale = max(amax_scale(a, src_dtype) for a in ks if a.size)
        v_scale = max(amax_scale(a, src_dtype) for a in vs if a.size)
    maxb = max((len(t) for t in tables), default=1)
    return DecodeWorkload(
        name=name, seed=seed, num_seqs=S, num_heads=H, num_kv_heads=Hkv, head_dim=D,
        block_size=B, num_blocks=NB, q_dtype=q_dtype, kv_dtype=kv_dtype, src_dtype=src_dtype,
        scale=np.float32(1.0 / np.sqrt(D)), k_scale=np.float32(k_scale), v_scale=np.float32(v_scale),
        context_lens=np.asarray(lens, dtype=np.int32), block_tables=tables_array(tables, maxb),
        q=q, setup=setup, step_copy=step_copy, step_scatter=step,
        partition_size=partition_size, description=description)


def independent_sequences(name, seed, S, H, Hkv, D, B, NB, q_dtype, kv_dtype, lens,
                          description="", partition_size=0) -> DecodeWorkload:
    """Sequences with private blocks; the step appends token L_s - 1 of each sequence.

    Blocks come from a seeded shuffle of range(NB) popped from the front.
    Tokens 0..L_s-2 are written by one setup scatter; the pool starts as
    random bytes, so unwritten slots hold arbitrary bit patterns.
    """
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, dtype=np.int64)
    alloc = BlockAllocator(rng.permutation(NB))
    src_dtype = q_dtype if kv_dtype != "e4m3" else "f16"
    tables, ctx_slots, new_slots = [], [], []
    for L in lens:
        table: List[int] = []
        for pos in range(int(L)):
            slot = alloc.slot_for_append(table, pos, B, [])
            (ctx_slots if pos < L - 1 else new_slots).append(slot)
        tables.append(table)
    ck, cv = _new_values(rng, len(ctx_slots), Hkv, D, src_dtype)
    setup = [Scatter(ck, cv, np.asarray(ctx_slots, dtype=np.int64))]
    return _finish(name, seed, rng, S, H, Hkv, D, B, NB, q_dtype, kv_dtype, lens, tables,
                   setup, None, new_slots, description, partition_size)


def shared_prefix_sampling(name, seed, prompts, samples, H, Hkv, D, B, NB, dtype,
                           prefix_blocks, tail_max, description="",
                           partition_size=0) -> DecodeWorkload:
    """Parallel sampling: ``samples`` sequences per prompt share the prompt's blocks.

    Prompt p has ``prefix_blocks * B + r_p`` tokens, r_p ~ U{1..B-1}, so its
    last block is partially filled and shared by all samples (ref count =
    samples).  At the first append each sample writes into that block: all but
    the last writer get a private copy (copy pairs, applied before any tail
    token is written), the last writes in place.  Each sample then has a
    private tail of U{1..tail_max} tokens; the step appends its last one.  The
    step also forks each prompt's shared partial block into ``samples - 1``
    spare blocks, the per-step block copy of beam-style forking.
    """
    rng = np.random.default_rng(seed)
    alloc = BlockAllocator(rng.permutation(NB))
    S = prompts * samples
    prompt_lens = prefix_blocks * B + rng.integers(1, B, size=prompts)
    tails = rng.integers(1, tail_max + 1, size=S)
    tables, lens = [], []
    prompt_slots, prompt_tables = [], []
    for p in range(prompts):
        t: List[int] = []
        for pos in range(int(prompt_lens[p])):
            prompt_slots.append(alloc.slot_for_append(t, pos, B, []))
        prompt_tables.append(t)
    cow_pairs: List[Tuple[int, int]] = []
    seq_tables = []
    for p in range(prompts):
        for i in range(samples):
            seq_tables.append(alloc.fork(prompt_tables[p]) if i < samples - 1 else prompt_tables[p])
    # the prompt's own reference is handed to its last sample: refs = samples
    first_tail_slots = []
    for s in range(S):
        p = s // samples
        first_tail_slots.append(alloc.slot_for_append(seq_tables[s], int(prompt_lens[p]), B, cow_pairs))
    tail_slots, new_slots = [], []
    for s in range(S):
        p = s // samples
        L = int(prompt_lens[p]) + int(tails[s])
        lens.append(L)
        for pos in range(int(prompt_lens[p]), L):
            slot = first_tail_slots[s] if pos == prompt_lens[p] else \
                alloc.slot_for_append(seq_tables[s], pos, B, [])
            (tail_slots if pos < L - 1 else new_slots).append(slot)
        tables.append(seq_tables[s])
    shared_partial = [prompt_tables[p][prefix_blocks] for p in range(prompts)]
    # the last sample of each prompt kept the original partial block
    fork_pairs = [(shared_partial[p], alloc.allocate()) for p in range(prompts)
                  for _ in range(samples - 1)]
    pk, pv = _new_values(rng, len(prompt_slots), Hkv, D, dtype)
    tk, tv = _new_values(rng, len(tail_slots), Hkv, D, dtype)
    setup = [Scatter(pk, pv, np.asarray(prompt_slots, dtype=np.int64)),
             Copy(np.asarray(cow_pairs, dtype=np.int64).reshape(-1, 2)),
             Scatter(tk, tv, np.asarray(tail_slots, dtype=np.int64))]
    step_copy = Copy(np.asarray(fork_pairs, dtype=np.int64).reshape(-1, 2))
    return _finish(name, seed, rng, S, H, Hkv, D, B, NB, dtype, dtype, lens, tables,
                   setup, step_copy, new_slots, description, partition_size)


# ---------------------------------------------------------------------------
# the five workloads
# ---------------------------------------------------------------------------

def lognormal_lens(rng, n, median, sigma, cap):
    return np.clip(np.rint(rng.lognormal(np.log(median), sigma, size=n)), 1, cap).astype(np.int64)


def make(name: str, small: bool = False) -> DecodeWorkload:
    """One of the named workloads; ``small`` shrinks batch and lengths for fast parity runs
    while keeping head shapes, dtypes and the length distribution's shape.  A name with the
    suffix ``_compact`` is the same workload (same sequences, lengths and values) with the
    pool cut down to the blocks in use plus 64, which keeps profiler captures small."""
    if name.endswith("_compact"):
        w = make(name[: -len("_compact")], small)
        if w.name.startswith("prefix"):
            raise KeyError(name)
        nblk = int(((w.context_lens.astype(np.int64) + w.block_size - 1) // w.block_size).sum())
        rng = np.random.default_rng(w.seed)
        return independent_sequences(
            name, w.seed, w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.block_size, nblk + 64,
            w.q_dtype, w.kv_dtype, w.context_lens, w.description + f" (pool cut to {nblk + 64} blocks)",
            partition_size=w.partition_size)
    if name == "tiny":
        rng = np.random.default_rng(0)
        lens = rng.integers(1, 257, size=4)
        w = independent_sequences("tiny", 0, 4, 8, 8, 64, 16, 128, "f16", "f16", lens,
                                  "batch 4, MHA 8 heads, head_dim 64, B=16, fp16, L~U[1,256]")
        return w
    if name == "opt13b":
        S, maxL, NB = (8, 700, 1024) if small else (64, 2048, 16384)
        rng = np.random.default_rng(1)
        lens = rng.integers(1, maxL + 1, size=S)
        return independent_sequences(
            "opt13b", 1, S, 40, 40, 128, 16, NB, "f16", "f16", lens,
            f"OPT-13B layer: batch {S}, 40 heads MHA, head_dim 128, B=16, fp16, "
            f"L~U[1,{maxL}], {NB}-block pool")
    if name == "gqa":
        S, NB, cap = (24, 4096, 1300) if small else (256, 65536, 4096)
        rng = np.random.default_rng(2)
        lens = lognormal_lens(rng, S, 800 if not small else 300, 1.0, cap)
        return independent_sequences(
            "gqa", 2, S, 32, 8, 128, 16, NB, "bf16", "bf16", lens,
            f"GQA layer: batch {S}, 32 q / 8 KV heads, head_dim 128, bf16, B=16, "
            f"L~lognormal(median {'300' if small else '800'}, sigma 1) capped {cap}, {NB}-block pool")
    if name == "prefix":
        prompts, tail_max = (4, 100) if small else (16, 256)
        return shared_prefix_sampling(
            "prefix", 3, prompts, 8, 32, 8, 128, 16, 4096 if not small else 1024, "f16",
            prefix_blocks=32, tail_max=tail_max,
            description=f"shared-prefix sampling: {prompts} prompts x 8 samples, 32 q / 8 KV heads, "
                        f"head_dim 128, fp16, 512+r token prompts, tails U[1,{tail_max}]")
    if name == "prefix_long":
        prompts, tail_max, pblocks = (2, 100, 80) if small else (16, 256, 256)
        return shared_prefix_sampling(
            "prefix_long", 5, prompts, 8, 32, 8, 128, 16, 8192 if not small else 1024, "f16",
            prefix_blocks=pblocks, tail_max=tail_max,
            description=f"long shared prompts: {prompts} prompts x 8 samples, 32 q / 8 KV heads, head_dim 128, "
                        f"fp16, {pblocks * 16}+r token prompts, tails U[1,{tail_max}]")
    if name in ("fp8", "fp8_b32"):
        B = 32 if name == "fp8_b32" else 16
        S, L = (4, 3000) if small else (16, 32768)
        per_seq = -(-L // B)
        NB = per_seq * S + per_seq * S // 4
        return independent_sequences(
            name, 4, S, 64, 8, 128, B, NB, "f16", "e4m3", np.full(S, L),
            f"long-context FP8: batch {S}, L={L}, 64 q / 8 KV heads, head_dim 128, "
            f"q fp16, K/V e4m3 per-tensor scale, B={B}, 512-token partitions", partition_size=512)
    raise KeyError(name)


# ---------------------------------------------------------------------------
# chunked prefill: prior context in the cache, then a chunk of new tokens
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class PrefillWorkload:
    """A prefill step: each sequence holds ``context_lens - chunk_lens`` earlier tokens in the
    cache (written by the setup scatter); the step scatters the chunk's K/V, then every chunk
    token attends causally to the cache up to its own position."""
    name: str
    seed: int
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    dtype: str                   # q, K/V and output: 'f16' | 'bf16'
    scale: np.float32
    context_lens: np.ndarray     # int32 [S], the chunk included
    chunk_lens: np.ndarray       # int32 [S]
    query_start: np.ndarray      # int32 [S + 1]
    block_tables: np.ndarray     # int32 [S, max_blocks]
    q: np.ndarray                # uint16 [T, H, D], the chunks packed in order
    setup: list                  # Scatter of the earlier tokens
    step_scatter: Scatter        # the chunk's K/V
    description: str = ""

    @property
    def num_tokens(self) -> int:
        return int(self.query_start[-1])

    @property
    def max_query_len(self) -> int:
        return int(self.chunk_lens.max()) if self.num_seqs else 0

    @property
    def max_blocks(self) -> int:
        return self.block_tables.shape[1]

    @property
    def pool_shape(self):
        return (self.num_blocks, self.num_kv_heads, self.block_size, self.head_dim)

    def initial_pool(self, which: str) -> np.ndarray:
        """Random bytes, as for decode: unwritten slots hold arbitrary bit patterns."""
        rng = np.random.default_rng([self.seed, 1 if which == "k" else 2])
        nbytes = int(np.prod(self.pool_shape)) * 2
        raw = np.resize(garbage_bytes(rng, min(nbytes, 32 << 20)), nbytes)
        return raw.view(np.uint16).reshape(self.pool_shape)


def chunked_prefill(name, seed, H, Hkv, D, B, NB, dtype, prior_lens, chunk_lens,
                    description="") -> PrefillWorkload:
    """Sequences with ``prior_lens`` cached tokens each receive a chunk of ``chunk_lens`` new
    tokens.  Blocks come from a seeded shuffle of range(NB), taken only when the last block is
    full; tokens are written in position order, so chunks start inside partially filled blocks."""
    rng = np.random.default_rng(seed)
    prior = np.asarray(prior_lens, dtype=np.int64)
    chunks = np.asarray(chunk_lens, dtype=np.int64)
    S = len(prior)
    alloc = BlockAllocator(rng.permutation(NB))
    tables, ctx_slots, new_slots = [], [], []
    for P, C in zip(prior, chunks):
        table: List[int] = []
        for pos in range(int(P + C)):
            slot = alloc.slot_for_append(table, pos, B, [])
            (ctx_slots if pos < P else new_slots).append(slot)
        tables.append(table)
    ck, cv = _new_values(rng, len(ctx_slots), Hkv, D, dtype)
    nk, nv = _new_values(rng, len(new_slots), Hkv, D, dtype)
    qs = np.zeros(S + 1, np.int32)
    qs[1:] = np.cumsum(chunks)
    q = normal_bits(rng, (int(qs[-1]), H, D), dtype)
    maxb = max((len(t) for t in tables), default=1)
    return PrefillWorkload(
        name=name, seed=seed, num_seqs=S, num_heads=H, num_kv_heads=Hkv, head_dim=D, block_size=B,
        num_blocks=NB, dtype=dtype, scale=np.float32(1.0 / np.sqrt(D)),
        context_lens=(prior + chunks).astype(np.int32), chunk_lens=chunks.astype(np.int32), query_start=qs,
        block_tables=tables_array(tables, maxb), q=q,
        setup=[Scatter(ck, cv, np.asarray(ctx_slots, dtype=np.int64))],
        step_scatter=Scatter(nk, nv, np.asarray(new_slots, dtype=np.int64)), description=description)


def make_prefill(name: str = "prefill", small: bool = False) -> PrefillWorkload:
    """The chunked-prefill workload: 16 sequences, 32 q / 8 KV heads x 128, bf16, B=16, each
    with U{0..3072} cached tokens and a chunk of U{512..2048} new ones (small: 3 sequences)."""
    if name != "prefill":
        raise KeyError(name)
    rng = np.random.default_rng(6)
    if small:
        prior, chunks, NB = [0, 37, 300], [200, 77, 129], 256
    else:
        prior, chunks, NB = rng.integers(0, 3073, size=16), rng.integers(512, 2049, size=16), 4096
    return chunked_prefill(
        "prefill", 6, 32, 8, 128, 16, NB, "bf16", prior, chunks,
        f"chunked prefill: {len(prior)} sequences, 32 q / 8 KV heads, head_dim 128, bf16, B=16, "
        + ("cached 0/37/300 + chunks 200/77/129" if small else "cached U[0,3072] + chunk U[512,2048]")
        + f", {NB}-block pool")


def prefill_flops(w: PrefillWorkload) -> int:
    """Multiply-adds x 2 of Q K^T and P V over the causal pairs: 4 * D * H * sum of attended keys."""
    L = w.context_lens.astype(np.int64)
    C = w.chunk_lens.astype(np.int64)
    keys = int((C * (L - C) + C * (C + 1) // 2).sum())
    return 4 * w.head_dim * w.num_heads * keys


def prefill_bytes(w: PrefillWorkload) -> int:
    """Bytes a prefill call must move at least: each sequence's K/V once, q and out."""
    kv = int(w.context_lens.astype(np.int64).sum()) * kv_bytes_per_token(1, w.num_kv_heads, w.head_dim, 2)
    return kv + 2 * w.num_tokens * w.num_heads * w.head_dim * 2


NAMES = ("tiny", "opt13b", "gqa", "prefix", "fp8", "fp8_b32")
EXTRA_NAMES = ("prefix_long",)
COMPACT_NAMES = tuple(n + "_compact" for n in NAMES if n != "prefix")


# ---------------------------------------------------------------------------
# byte accounting (measurement, not the method)
# ---------------------------------------------------------------------------

def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    """K and V bytes one token occupies across all layers."""
    return 2 * num_layers * num_kv_heads * head_dim * elem_bytes


def decode_algorithmic_bytes(w: DecodeWorkload) -> int:
    """KV actually needed (valid tokens only) + q + out + used table entries + lengths."""
    kv = int(w.context_lens.astype(np.int64).sum()) * kv_bytes_per_token(
        1, w.num_kv_heads, w.head_dim, ELEM_BYTES[w.kv_dtype])
    qo = 2 * w.num_seqs * w.num_heads * w.head_dim * ELEM_BYTES[w.q_dtype]
    nblk = int(((w.context_lens.astype(np.int64) + w.block_size - 1) // w.block_size).sum())
    return kv + qo + 4 * nblk + 4 * w.num_seqs


def decode_distinct_bytes(w: DecodeWorkload) -> int:
    """decode_algorithmic_bytes with each physical KV slot counted once, however many
    sequences attend to it: the least a decode call over shared blocks has to read."""
    B = w.block_size
    slots = []
    for s in range(w.num_seqs):
        L = int(w.context_lens[s])
        p = np.arange(L, dtype=np.int64)
        slots.append(w.block_tables[s, p // B].astype(np.int64) * B + p % B)
    n = int(np.unique(np.concatenate(slots)).size) if slots else 0
    kv = n * kv_bytes_per_token(1, w.num_kv_heads, w.head_dim, ELEM_BYTES[w.kv_dtype])
    return decode_algorithmic_bytes(w) - int(w.context_lens.astype(np.int64).sum()) * kv_bytes_per_token(
        1, w.num_kv_heads, w.head_dim, ELEM_BYTES[w.kv_dtype]) + kv


def scatter_algorithmic_bytes(w: DecodeWorkload, sc: Scatter) -> int:
    """Read k, v; write both into the pool; read the slots."""
    n = sc.k.shape[0] * w.num_kv_heads * w.head_dim
    return n * 2 * ELEM_BYTES[w.src_dtype] + n * 2 * ELEM_BYTES[w.kv_dtype] + 8 * sc.k.shape[0]


def copy_algorithmic_bytes(w: DecodeWorkload, cp: Optional[Copy]) -> int:
    if cp is None:
        return 0
    blk = w.num_kv_heads * w.block_size * w.head_dim * ELEM_BYTES[w.kv_dtype]
    return cp.pairs.shape[0] * (2 * 2 * blk + 16)


def step_algorithmic_bytes(w: DecodeWorkload) -> int:
    return (decode_algorithmic_bytes(w) + scatter_algorithmic_bytes(w, w.step_scatter)
            + copy_algorithmic_bytes(w, w.step_copy))
