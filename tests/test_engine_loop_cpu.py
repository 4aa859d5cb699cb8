"""A serving loop's host logic end to end, on CPU: the native block manager hands out
slots, tables and copy-on-write pairs; the oracle does the memory operations and
the attention on the paged pool; every output is compared with attention over
that sequence's own contiguous token history (no paging), so a wrong slot, table
entry, copy pair or cache hit shows up as a wrong result.

The loop: prompts appended as whole chunks (pkv_bm_append_tokens) and prefilled,
forks into parallel samples (shared blocks), decode steps with copy-on-write, a
finished sequence whose blocks are reused, and a request whose prompt hits the
prefix cache and prefills only the rest.
"""
import numpy as np
import scipy.special

import oracle
from paged_kv_cache_324_b200 import workload as wl
from tests.test_oracle_pins import f64

H, Hkv, D, BS, NB = 4, 2, 16, 4, 96
G = H // Hkv
SCALE = 0.25


def reference(q_bits, hist_k, hist_v, positions):
    """Rows of q [n, H, D] attend causally to the contiguous history up to their positions."""
    K = np.repeat(f64(np.stack(hist_k), "f16"), G, axis=1)        # [L, H, D]
    V = np.repeat(f64(np.stack(hist_v), "f16"), G, axis=1)
    out = []
    for row, p in zip(f64(q_bits, "f16"), positions):
        logits = np.einsum("hd,thd->ht", row, K[:p + 1]) * SCALE
        out.append(np.einsum("ht,thd->hd", scipy.special.softmax(logits, axis=1), V[:p + 1]))
    return np.stack(out)


def test_block_manager_driven_loop_matches_contiguous_attention():
    from paged_kv_cache_324_b200 import binding as B
    from paged_kv_cache_324_b200 import build
    build.build()
    rng = np.random.default_rng(31)
    bm = B.BlockManager(NB, BS, rng.permutation(NB))
    kp = wl.garbage_bytes(rng, NB * Hkv * BS * D * 2).view(np.uint16).reshape(NB, Hkv, BS, D)
    vp = wl.garbage_bytes(rng, NB * Hkv * BS * D * 2).view(np.uint16).reshape(NB, Hkv, BS, D)
    hist = {}                                                     # seq -> (keys, values, token ids)

    def write(slots, k, v):
        oracle.reshape_and_cache(k, v, "f16", kp, vp, "f16", slots)

    def tables(ids):
        t, lens = bm.block_tables(ids, 32, pad=int(wl.TABLE_POISON))
        return t, lens

    def prefill(ids, starts):
        """Prefill the tokens of each sequence from starts[i] on; compare with the reference."""
        t, lens = tables(ids)
        chunks = [int(lens[i]) - starts[i] for i in range(len(ids))]
        qs = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
        q = wl.normal_bits(rng, (int(qs[-1]), H, D), "f16")
        out = oracle.paged_attn_prefill(q, "f16", kp, vp, "f16", t, lens, qs, SCALE)
        for i, s in enumerate(ids):
            ref = reference(q[qs[i]:qs[i + 1]], hist[s][0], hist[s][1], range(starts[i], int(lens[i])))
            np.testing.assert_allclose(out[qs[i]:qs[i + 1]], ref, rtol=1e-10, atol=1e-12)

    def decode(ids):
        slots, pairs = bm.append_slots(ids)
        if len(pairs):
            oracle.copy_blocks(kp, vp, pairs)
        k = wl.normal_bits(rng, (len(ids), Hkv, D), "f16")
        v = wl.normal_bits(rng, (len(ids), Hkv, D), "f16")
        write(slots, k, v)
        for i, s in enumerate(ids):
            hist[s][0].append(k[i])
            hist[s][1].append(v[i])
        t, lens = tables(ids)
        q = wl.normal_bits(rng, (len(ids), H, D), "f16")
        out = oracle.paged_attn_decode(q, "f16", kp, vp, "f16", t, lens, SCALE)
        for i, s in enumerate(ids):
            ref = reference(q[i:i + 1], hist[s][0], hist[s][1], [int(lens[i]) - 1])
            np.testing.assert_allclose(out[i:i + 1], ref, rtol=1e-10, atol=1e-12)
        return len(pairs)

    def add_prompt(s, tokens):
        bm.add_sequence(s)
        slots, pairs = bm.append_tokens(s, len(tokens))
        assert len(pairs) == 0
        k = wl.normal_bits(rng, (len(tokens), Hkv, D), "f16")
        v = wl.normal_bits(rng, (len(tokens), Hkv, D), "f16")
        write(slots, k, v)
        hist[s] = (list(k), list(v), list(tokens))

    prompts = {0: rng.integers(0, 50, 13), 1: rng.integers(0, 50, 8), 2: rng.integers(0, 50, 3)}
    for s, toks in prompts.items():
        add_prompt(s, toks)
    prefill([0, 1, 2], [0, 0, 0])
    bm.cache_sequence(0, prompts[0])                              # sequence 0's full blocks: 3 of them

    nxt = 3
    for s in (0, 1):                                              # two more samples each
        for _ in range(2):
            bm.fork(s, nxt)
            hist[nxt] = (list(hist[s][0]), list(hist[s][1]), list(hist[s][2]))
            nxt += 1
    live = [0, 1, 2, 3, 4, 5, 6]
    copies = 0
    for it in range(9):
        copies += decode(live)
        if it == 4:                                               # a sequence finishes
            bm.free_sequence(2)
            live.remove(2)
    # sequence 0's 13-token prompt leaves a partial block held by 3 samples: the first 2 writers
    # copy it, the last writes in place; sequence 1's 8 tokens fill whole blocks: no copy
    assert copies == 2

    # a new request whose prompt starts with sequence 0's: the cached full blocks are shared
    toks = np.concatenate([prompts[0][:12], rng.integers(0, 50, 6)])
    s = nxt
    got = bm.add_sequence_cached(s, toks)
    assert got == 12
    t0, _ = tables([0])
    ts, _ = tables([s])
    assert np.array_equal(ts[0, :3], t0[0, :3])
    hist[s] = (hist[0][0][:12], hist[0][1][:12], list(toks[:12]))
    rest = len(toks) - got
    slots, pairs = bm.append_tokens(s, rest)
    assert len(pairs) == 0                                        # 12 tokens fill whole blocks
    k = wl.normal_bits(rng, (rest, Hkv, D), "f16")
    v = wl.normal_bits(rng, (rest, Hkv, D), "f16")
    write(slots, k, v)
    hist[s][0].extend(k)
    hist[s][1].extend(v)
    prefill([s], [got])                                           # only the uncached tokens are computed
    decode(live + [s])
