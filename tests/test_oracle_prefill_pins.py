"""Pins of the oracle's chunked prefill to what the pages and the mathematics fix.

Prefill computes, for every token of a chunk, the causal attention of the
token form in the Wikipedia article "PagedAttention" (section "Mathematical
formulation"): query position i attends to positions 0..i.  The pins: a
library softmax over the contiguous cache with a causal mask (rows of a chunk
that follows earlier context included, so a wrong position offset fails),
closed forms (the first token of a prompt returns its own value; equal keys
give the mean of the values up to the query's position, which counts the
attended tokens), pure-Python brute force on tiny inputs, equality of each row
with the separately written decode definition truncated at its position, and
the rejection of malformed chunk layouts.
"""
import math

import numpy as np
import pytest
import scipy.special

import oracle
from paged_kv_cache_324_b200 import workload as wl
from tests.test_oracle_pins import f64


def chunked_cache(seed, H, Hkv, D, B, lens, chunks, dtype="f16", NB=None):
    """Contiguous K/V/q for every position of each sequence, the pool holding K/V through a
    shuffled table, and q rows of the last ``chunks[s]`` positions packed in order."""
    rng = np.random.default_rng(seed)
    S = len(lens)
    Lmax = max(max(lens), 1)
    K = wl.normal_bits(rng, (S, Lmax, Hkv, D), dtype)
    V = wl.normal_bits(rng, (S, Lmax, Hkv, D), dtype)
    Q = wl.normal_bits(rng, (S, Lmax, H, D), dtype)
    need = sum(-(-L // B) for L in lens)
    NB = NB or need + 3
    perm = rng.permutation(NB)
    kp = wl.garbage_bytes(rng, NB * Hkv * B * D * 2).view(np.uint16).reshape(NB, Hkv, B, D)
    vp = wl.garbage_bytes(rng, NB * Hkv * B * D * 2).view(np.uint16).reshape(NB, Hkv, B, D)
    maxb = max(1, max(-(-L // B) for L in lens))
    tables = np.full((S, maxb), wl.TABLE_POISON, np.int32)
    nxt = 0
    for s, L in enumerate(lens):
        for j in range(-(-L // B)):
            tables[s, j] = perm[nxt]
            nxt += 1
        for t in range(L):
            kp[tables[s, t // B], :, t % B, :] = K[s, t]
            vp[tables[s, t // B], :, t % B, :] = V[s, t]
    qs = np.zeros(S + 1, np.int32)
    qs[1:] = np.cumsum(chunks)
    q = np.concatenate([Q[s, L - C:L] for s, (L, C) in enumerate(zip(lens, chunks))], axis=0) \
        if qs[-1] else np.zeros((0, H, D), np.uint16)
    return dict(q=np.ascontiguousarray(q), K=K, V=V, Q=Q, kp=kp, vp=vp, tables=tables,
                lens=np.asarray(lens, np.int32), qs=qs)


def run(c, scale, dtype="f16"):
    return oracle.paged_attn_prefill(c["q"], dtype, c["kp"], c["vp"], dtype, c["tables"], c["lens"],
                                     c["qs"], scale)


def causal_reference(c, s, G, scale, shift=0, dtype="f16"):
    """scipy softmax over the contiguous cache, row j of the chunk masked to t <= L - C + j + shift."""
    L = int(c["lens"][s])
    C = int(c["qs"][s + 1] - c["qs"][s])
    Kf = np.repeat(f64(c["K"][s, :L], dtype), G, axis=1)     # [L, H, D]; head h uses KV head h // G
    Vf = np.repeat(f64(c["V"][s, :L], dtype), G, axis=1)
    qf = f64(c["Q"][s, L - C:L], dtype)                       # [C, H, D]
    logits = np.einsum("jhd,thd->jht", qf, Kf) * scale
    pos = (L - C + np.arange(C) + shift)[:, None, None]
    logits = np.where(np.arange(L)[None, None, :] <= pos, logits, -np.inf)
    return np.einsum("jht,thd->jhd", scipy.special.softmax(logits, axis=2), Vf)


@pytest.mark.parametrize("B", [1, 4, 16])
@pytest.mark.parametrize("G", [1, 4])
def test_matches_library_causal_softmax(B, G):
    lens = [7, 40, 33, 16, 1]
    chunks = [7, 13, 1, 16, 1]          # a whole prompt, chunks after context, single tokens
    c = chunked_cache(40 + B + G, 2 * G, 2, 8, B, lens, chunks)
    out = run(c, 0.3)
    for s in range(len(lens)):
        ref = causal_reference(c, s, G, 0.3)
        np.testing.assert_allclose(out[c["qs"][s]:c["qs"][s + 1]], ref, rtol=1e-12, atol=1e-13)


def test_position_offset_is_pinned():
    """The same reference with the causal limit moved by one token differs far beyond rounding."""
    c = chunked_cache(47, 2, 2, 8, 4, [30], [10])
    out = run(c, 0.5)
    for shift in (-1, 1):
        ref = causal_reference(c, 0, 1, 0.5, shift=shift)
        assert np.abs(out - ref).max() > 1e-3


def test_first_token_of_a_prompt_returns_its_value():
    c = chunked_cache(48, 4, 2, 8, 4, [9, 12], [9, 12])
    out = run(c, 0.5)
    for s in range(2):
        r = c["qs"][s]
        for h in range(4):
            assert np.array_equal(out[r, h], f64(c["V"][s, 0, h // 2]))


def test_equal_keys_give_mean_of_values_up_to_the_position():
    c = chunked_cache(49, 2, 1, 8, 4, [21], [8])
    one = c["K"][0, 0].copy()
    B = 4
    for t in range(21):
        c["kp"][c["tables"][0, t // B], :, t % B, :] = one
    out = run(c, 0.5)
    Vf = f64(c["V"][0, :, 0])
    for j in range(8):
        p = 21 - 8 + j
        ref = Vf[:p + 1].mean(axis=0)
        for h in range(2):
            np.testing.assert_allclose(out[j, h], ref, rtol=1e-12, atol=1e-14)


def test_brute_force_pure_python():
    """Scalar loops with math.exp on D=4: two sequences, chunks after context."""
    lens, chunks = [6, 9], [3, 9]
    c = chunked_cache(50, 2, 1, 4, 2, lens, chunks)
    out = run(c, 0.7)
    r = 0
    for s, (L, C) in enumerate(zip(lens, chunks)):
        for j in range(C):
            p = L - C + j
            for h in range(2):
                qv = [float(x) for x in c["Q"][s, p, h].view(np.float16)]
                ks = [[float(x) for x in c["K"][s, t, 0].view(np.float16)] for t in range(p + 1)]
                vs = [[float(x) for x in c["V"][s, t, 0].view(np.float16)] for t in range(p + 1)]
                e = [math.exp(0.7 * sum(a * b for a, b in zip(qv, k))) for k in ks]
                o = [sum(e[t] * vs[t][d] for t in range(p + 1)) / sum(e) for d in range(4)]
                np.testing.assert_allclose(out[r, h], o, rtol=1e-12, atol=1e-14)
            r += 1


def test_each_row_is_decode_truncated_at_its_position():
    lens, chunks = [50, 19], [17, 19]
    c = chunked_cache(51, 8, 2, 16, 16, lens, chunks, dtype="bf16")
    out = run(c, 0.25, dtype="bf16")
    for s, (L, C) in enumerate(zip(lens, chunks)):
        rows = c["q"][c["qs"][s]:c["qs"][s + 1]]
        tab = np.repeat(c["tables"][s:s + 1], C, axis=0)
        plen = (L - C + 1 + np.arange(C)).astype(np.int32)
        dec = oracle.paged_attn_decode(rows, "bf16", c["kp"], c["vp"], "bf16", tab, plen, 0.25)
        np.testing.assert_allclose(out[c["qs"][s]:c["qs"][s + 1]], dec, rtol=1e-12, atol=1e-14)


def test_fp8_cache_uses_the_dequantised_values():
    """E4M3 pools: the result equals the 16-bit oracle run on the dequantised values."""
    rng = np.random.default_rng(52)
    c = chunked_cache(52, 4, 2, 8, 4, [20, 11], [6, 11])
    kf, vf = f64(c["kp"]), f64(c["vp"])
    kf = np.where(np.isfinite(kf), kf, 0.0)
    vf = np.where(np.isfinite(vf), vf, 0.0)
    ks, vs = np.float32(0.01), np.float32(0.02)
    kq = oracle.encode_e4m3((kf / 4).astype(np.float32) / ks)
    vq = oracle.encode_e4m3((vf / 4).astype(np.float32) / vs)
    out = oracle.paged_attn_prefill(c["q"], "f16", kq, vq, "e4m3", c["tables"], c["lens"], c["qs"], 0.5,
                                    k_scale=ks, v_scale=vs)
    # the same cache written as exact float64 values into a wide-type pool is not expressible in
    # 16 bits, so compare with the definition written out here on the dequantised values
    kd, vd = f64(kq, "e4m3") * float(ks), f64(vq, "e4m3") * float(vs)
    r = 0
    for s, (L, C) in enumerate(zip([20, 11], [6, 11])):
        for j in range(C):
            p = L - C + j
            for h in range(4):
                qv = f64(c["q"][r, h])
                kk = np.stack([kd[c["tables"][s, t // 4], h // 2, t % 4] for t in range(p + 1)])
                vv = np.stack([vd[c["tables"][s, t // 4], h // 2, t % 4] for t in range(p + 1)])
                w = scipy.special.softmax(kk @ qv * 0.5)
                np.testing.assert_allclose(out[r, h], w @ vv, rtol=1e-12, atol=1e-14)
            r += 1


def test_malformed_chunks_are_rejected():
    c = chunked_cache(53, 2, 2, 8, 4, [5, 9], [5, 9])
    bad = c["qs"].copy()
    bad[1] = 6                       # first chunk longer than its sequence
    with pytest.raises(oracle.OracleError):
        oracle.paged_attn_prefill(c["q"], "f16", c["kp"], c["vp"], "f16", c["tables"], c["lens"], bad, 0.5)
    tab = c["tables"].copy()
    tab[1, 1] = c["kp"].shape[0]     # a table entry the definition reads is out of range
    with pytest.raises(oracle.OracleError):
        oracle.paged_attn_prefill(c["q"], "f16", c["kp"], c["vp"], "f16", tab, c["lens"], c["qs"], 0.5)


def test_prefill_tolerance_rejects_planted_mistakes():
    """Mistakes planted in the oracle's inputs (each a plausible kernel bug) fail the prefill
    comparison rule: attending one key too few, ignoring causality inside the chunk, and
    pairing query heads with the wrong KV head."""
    from tests import harness as H
    from tests.parity import prefill_close
    w = wl.chunked_prefill("planted", 60, 8, 2, 128, 16, 128, "bf16", [40, 90], [70, 33])
    kp, vp = H.oracle_prefill_pools(w)
    ref = oracle.paged_attn_prefill(w.q, "bf16", kp, vp, "bf16", w.block_tables, w.context_lens, w.query_start,
                                    w.scale)
    assert prefill_close(ref, ref, "bf16")[0]
    # one key too few: the same chunks in contexts one token shorter
    short = oracle.paged_attn_prefill(w.q, "bf16", kp, vp, "bf16", w.block_tables, w.context_lens - 1,
                                      w.query_start, w.scale)
    assert not prefill_close(short, ref, "bf16")[0]
    # no causal mask inside the chunk: every row sees its sequence's whole context
    rows = []
    for s in range(w.num_seqs):
        n = int(w.chunk_lens[s])
        tab = np.repeat(w.block_tables[s:s + 1], n, axis=0)
        lens = np.full(n, w.context_lens[s], np.int32)
        q = w.q[w.query_start[s]:w.query_start[s + 1]]
        rows.append(oracle.paged_attn_decode(q, "bf16", kp, vp, "bf16", tab, lens, w.scale))
    assert not prefill_close(np.concatenate(rows), ref, "bf16")[0]
    # query head h paired with KV head h % Hkv instead of h // G
    Hq, Hkv = w.num_heads, w.num_kv_heads
    G = Hq // Hkv
    perm = np.array([(h % Hkv) * G + h // Hkv for h in range(Hq)])
    qp = np.empty_like(w.q)
    qp[:, perm] = w.q
    outp = oracle.paged_attn_prefill(qp, "bf16", kp, vp, "bf16", w.block_tables, w.context_lens, w.query_start,
                                     w.scale)
    assert not prefill_close(outp[:, perm], ref, "bf16")[0]
