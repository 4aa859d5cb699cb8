"""Pins of the float64 oracle to what the pages and the mathematics fix.

Each test ties the oracle to something other than itself: the worked example
printed in the Ultralytics glossary entry "PagedAttention" (section "How
paging works"), closed forms of softmax attention, the block form of the
Wikipedia article "PagedAttention" (section "Mathematical formulation")
written out independently, a library softmax on a contiguous [B, L, H, D]
cache (the pre-paging layout of the same article's vAttention section),
brute force on tiny inputs, invariants of paging (permutation of physical
ids, shared blocks versus private copies), and library codecs for the number
formats.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from paged_kv_cache_324_b200 import workload as wl
from tests.parity import attention_close

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# helpers (test-side construction of small caches)
# --------------------------------------------------------------------------

def small_cache(seed, S, H, Hkv, D, B, lens, NB=None, dtype="f16"):
    """Contiguous K/V [S, Lmax, Hkv, D] and q, placed into a shuffled pool with the test's own loop."""
    rng = np.random.default_rng(seed)
    Lmax = max(int(max(lens)), 1)
    K = wl.normal_bits(rng, (S, Lmax, Hkv, D), dtype)
    V = wl.normal_bits(rng, (S, Lmax, Hkv, D), dtype)
    q = wl.normal_bits(rng, (S, H, D), dtype)
    need = sum(-(-int(L) // B) for L in lens)
    NB = NB or need + 5
    perm = rng.permutation(NB)
    kp = wl.garbage_bytes(rng, NB * Hkv * B * D * 2).view(np.uint16).reshape(NB, Hkv, B, D)
    vp = wl.garbage_bytes(rng, NB * Hkv * B * D * 2).view(np.uint16).reshape(NB, Hkv, B, D)
    maxb = max(1, max(-(-int(L) // B) for L in lens))
    tables = np.full((S, maxb), wl.TABLE_POISON, np.int32)
    nxt = 0
    for s, L in enumerate(lens):
        for j in range(-(-int(L) // B)):
            tables[s, j] = perm[nxt]
            nxt += 1
        for t in range(int(L)):
            kp[tables[s, t // B], :, t % B, :] = K[s, t]
            vp[tables[s, t // B], :, t % B, :] = V[s, t]
    return q, K, V, kp, vp, tables, np.asarray(lens, np.int32)


def f64(bits, dtype="f16"):
    return oracle.decode_values(bits, dtype)


# --------------------------------------------------------------------------
# the worked example (glossary, "How paging works")
# --------------------------------------------------------------------------

def test_worked_example_block_table_and_gather():
    g = json.load(open(os.path.join(GOLDEN, "ul_worked_example.json")))
    B, D, n = g["block_size"], g["head_dim"], g["num_tokens"]
    exp = g["expected"]
    alloc = wl.BlockAllocator(g["free_blocks"])
    table = []
    slots = [alloc.slot_for_append(table, pos, B, []) for pos in range(n)]
    assert len(table) == exp["blocks_needed"] == -(-n // B)
    assert table == exp["block_table"]
    # scatter exactly as the page writes it: pool[table[pos // B], pos % B] = key
    assert slots == [table[p // B] * B + p % B for p in range(n)]
    rng = np.random.default_rng(7)
    keys = wl.normal_bits(rng, (n, 1, D), "f16")
    pool = np.zeros((g["pool_blocks"], 1, B, D), np.uint16)
    vpool = np.zeros_like(pool)
    oracle.reshape_and_cache(keys, keys, "f16", pool, vpool, "f16", np.asarray(slots))
    gathered = oracle.gather(pool, "f16", table, n)
    assert np.array_equal(gathered, keys[:, 0, :]) == exp["keys_intact"]
    assert len(table) * B - n == exp["unused_slots_paged"]
    assert g["reservation_tokens"] - n == exp["unused_slots_reserved"]
    # no other block of the pool was touched
    others = [b for b in range(g["pool_blocks"]) if b not in table]
    assert not pool[others].any()


def test_waste_is_below_one_block():
    """Only the last block's tail is unused: ceil(L/B)*B - L <= B-1 (glossary, 'How paging works')."""
    rng = np.random.default_rng(11)
    for B in (1, 4, 16, 32):
        alloc = wl.BlockAllocator(range(100000))
        for L in rng.integers(1, 3000, size=50):
            t = []
            for pos in range(int(L)):
                alloc.slot_for_append(t, pos, B, [])
            assert len(t) == -(-int(L) // B)
            assert 0 <= len(t) * B - L <= B - 1


def test_allocator_copy_on_write_rule():
    """A write into a block referenced elsewhere copies it first; the last holder writes in place."""
    alloc = wl.BlockAllocator(range(100))
    base = []
    for pos in range(20):              # 16 + 4 tokens: one full block, one partial
        alloc.slot_for_append(base, pos, 16, [])
    forks = [alloc.fork(base) for _ in range(3)]
    assert alloc.ref[base[1]] == 4 and alloc.ref[base[0]] == 4
    pairs = []
    for t in forks:
        alloc.slot_for_append(t, 20, 16, pairs)
    alloc.slot_for_append(base, 20, 16, pairs)
    assert len(pairs) == 3 and all(p[0] == base[1] for p in pairs)
    assert len({p[1] for p in pairs}) == 3
    assert all(t[0] == base[0] for t in forks)            # full block stays shared
    assert alloc.ref[base[1]] == 1 and alloc.ref[base[0]] == 4


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------

def test_f16_decode_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = f64(bits, "f16")
    lib = bits.view(np.float16).astype(np.float64)
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    m = ~np.isnan(lib)
    assert np.array_equal(ours[m], lib[m])


def test_bf16_decode_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = f64(bits, "bf16")
    lib = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    m = ~np.isnan(lib)
    assert np.array_equal(ours[m], lib[m])


def test_e4m3_decode_exhaustive_against_library():
    bits = np.arange(256, dtype=np.uint8)
    ours = f64(bits, "e4m3")
    lib = torch.from_numpy(bits).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF]) and np.isnan(ours).sum() == 2
    m = ~np.isnan(lib)
    assert np.array_equal(ours[m], lib[m])
    assert ours[0x7E] == 448.0 and ours[0x08] == 2.0 ** -6 and ours[0x01] == 2.0 ** -9


def test_e4m3_encode_against_library_and_roundtrip():
    finite = np.array([b for b in range(256) if b not in (0x7F, 0xFF)], np.uint8)
    vals = f64(finite, "e4m3").astype(np.float32)
    assert np.array_equal(oracle.encode_e4m3(vals), finite)          # encode(decode(b)) == b
    # every midpoint between neighbours, and points just either side of it
    pos = np.sort(f64(np.arange(0, 0x7F, dtype=np.uint8), "e4m3"))
    mids = (pos[1:] + pos[:-1]) / 2
    probe = np.concatenate([mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9)]).astype(np.float32)
    rng = np.random.default_rng(5)
    probe = np.concatenate([probe, rng.uniform(-447.9, 447.9, 200000).astype(np.float32),
                            (rng.standard_normal(200000) * 0.05).astype(np.float32)])
    probe = np.concatenate([probe, -probe])
    probe = probe[np.abs(probe) < 448]                # the library cast does not saturate
    lib = torch.from_numpy(probe).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.encode_e4m3(probe), lib)


def test_e4m3_encode_saturates():
    x = np.array([448.0, 449.0, 463.9, 464.0, 500.0, 1e30, np.inf, -1e30, -np.inf], np.float32)
    assert oracle.encode_e4m3(x).tolist() == [0x7E] * 7 + [0xFE] * 2
    assert oracle.encode_e4m3(np.array([np.nan], np.float32))[0] & 0x7F == 0x7F


# --------------------------------------------------------------------------
# attention: closed forms, library reference, block form, brute force
# --------------------------------------------------------------------------

def test_single_token_returns_its_value():
    """L = 1: the softmax has one term, so o = v_1 exactly."""
    q, K, V, kp, vp, tab, lens = small_cache(1, 3, 4, 2, 16, 4, [1, 1, 1])
    out = oracle.paged_attn_decode(q, "f16", kp, vp, "f16", tab, lens, scale=0.25)
    G = 2
    for s in range(3):
        for h in range(4):
            assert np.array_equal(out[s, h], f64(V[s, 0, h // G]))


def test_zero_query_gives_mean_of_values():
    """q = 0 makes every score equal, so o is the plain mean of the L values."""
    q, K, V, kp, vp, tab, lens = small_cache(2, 2, 2, 1, 8, 4, [13, 37])
    q[:] = 0
    out = oracle.paged_attn_decode(q, "f16", kp, vp, "f16", tab, lens, scale=0.5)
    for s, L in enumerate(lens):
        mean = f64(V[s, :L, 0]).mean(axis=0)
        for h in range(2):
            np.testing.assert_allclose(out[s, h], mean, rtol=0, atol=1e-14)


def test_equal_keys_give_mean_of_values():
    q, K, V, kp, vp, tab, lens = small_cache(3, 1, 1, 1, 8, 4, [23])
    for t in range(23):
        kp[tab[0, t // 4], 0, t % 4] = K[0, 0, 0]
    out = oracle.paged_attn_decode(q, "f16", kp, vp, "f16", tab, lens, scale=0.3)
    np.testing.assert_allclose(out[0, 0], f64(V[0, :23, 0]).mean(axis=0), rtol=0, atol=1e-14)


def test_dominant_score_selects_its_value():
    """A score larger than all others by g gives o within (L-1) e^-g max|v| of that token's value."""
    q, K, V, kp, vp, tab, lens = small_cache(4, 1, 1, 1, 8, 4, [19])
    kf = f64(K[0, :19, 0])
    qf = f64(q[0, 0])
    scores = kf @ qf
    j = int(np.argmax(scores))
    gap = scores[j] - np.sort(scores)[-2]
    scale = 60.0 / gap
    out = oracle.paged_attn_decode(q, "f16", kp, vp, "f16", tab, lens, scale=scale)
    bound = 18 * math.exp(-60.0) * np.abs(f64(V[0, :19, 0])).max() * 2
    np.testing.assert_allclose(out[0, 0], f64(V[0, j, 0]), rtol=0, atol=bound + 1e-15)


@pytest.mark.parametrize("B", [1, 2, 4, 16])
@pytest.mark.parametrize("G", [1, 2, 4])
def test_matches_library_softmax_on_contiguous_cache(B, G):
    """Equality with softmax(q K^T scale) V on the contiguous [S, L, Hkv, D] cache (scipy softmax)."""
    Hkv = 2
    lens = [1, 5, B, B + 1, 40]
    q, K, V, kp, vp, tab, lens = small_cache(10 + B + G, 5, Hkv * G, Hkv, 8, B, lens)
    scale = 1 / math.sqrt(8)
    out = oracle.paged_attn_decode(q, "f16", kp, vp, "f16", tab, lens, scale=scale)
    Kf, Vf, qf = f64(K), f64(V), f64(q)
    for s, L in enumerate(lens):
        Kr = np.repeat(Kf[s, :L], G, axis=1)       # [L, H, D], head h uses KV head h // G
        Vr = np.repeat(Vf[s, :L], G, axis=1)
        logits = np.einsum("hd,lhd->hl", qf[s], Kr) * scale
        ref = np.einsum("hl,lhd->hd", scipy.special.softmax(logits, axis=1), Vr)
        np.testing.assert_allclose(out[s], ref, rtol=1e-12, atol=1e-13)


def block_form(qf, kp_f, vp_f, table, L, kvh, B, scale):
    """The Wikipedia block form: A_ij = exp(q.K_j/sqrt d) / sum_t sum exp(q.K_t/sqrt d),
    o = sum_j V_j A_ij^T over ceil(L/B) blocks, with slots t >= L of the last block left out."""
    nblk = -(-L // B)
    A = []
    for j in range(nblk):
        Kj = kp_f[table[j], kvh]
        valid = np.arange(j * B, j * B + B) < L
        with np.errstate(over="ignore", invalid="ignore"):
            A.append(np.where(valid, np.exp((Kj @ qf) * scale), 0.0))
    den = sum(a.sum() for a in A)
    o = np.zeros(kp_f.shape[-1])
    for j in range(nblk):
        valid = np.arange(j * B, j * B + B) < L
        Vj = np.where(valid[:, None], vp_f[table[j], kvh], 0.0)
        o += Vj.T @ (A[j] / den)
    return o


@pytest.mark.parametrize("B", [1, 2, 4, 16])
def test_matches_block_form(B):
    lens = [1, B, B + 1, 3 * B - 1, 40]
    q, K, V, kp, vp, tab, lens = small_cache(20 + B, 5, 4, 2, 8, B, lens)
    out = oracle.paged_attn_decode(q, "f16", kp, vp, "f16", tab, lens, scale=0.35)
    kp_f, vp_f, qf = f64(kp), f64(vp), f64(q)
    for s, L in enumerate(lens):
        for h in range(4):
            ref = block_form(qf[s, h], kp_f, vp_f, tab[s], int(L), h // 2, B, 0.35)
            np.testing.assert_allclose(out[s, h], ref, rtol=1e-12, atol=1e-13)


def test_brute_force_pure_python():
    """Scalar loops with math.exp on D=4, L up to 9."""
    q, K, V, kp, vp, tab, lens = small_cache(30, 3, 2, 1, 4, 2, [1, 4, 9])
    out = oracle.paged_attn_decode(q, "f16", kp, vp, "f16", tab, lens, scale=0.7)
    for s, L in enumerate(lens):
        for h in range(2):
            qv = [float(x) for x in q[s, h].view(np.float16)]
            ks = [[float(x) for x in K[s, t, 0].view(np.float16)] for t in range(L)]
            vs = [[float(x) for x in V[s, t, 0].view(np.float16)] for t in range(L)]
            e = [math.exp(0.7 * sum(a * b for a, b in zip(qv, k))) for k in ks]
            o = [sum(e[t] * vs[t][d] for t in range(L)) / sum(e) for d in range(4)]
            np.testing.assert_allclose(out[s, h], o, rtol=1e-12, atol=1e-14)


def test_zero_length_sequence_gives_zero():
    q, K, V, kp, vp, tab, lens = small_cache(31, 2, 2, 2, 8, 4, [0, 3])
    out = oracle.paged_attn_decode(q, "f16", kp, vp, "f16", tab, lens, scale=0.5)
    assert not out[0].any() and np.all(np.isfinite(out[1]))


def test_invalid_table_entry_is_rejected():
    q, K, V, kp, vp, tab, lens = small_cache(32, 1, 1, 1, 8, 4, [9])
    tab[0, 2] = kp.shape[0]
    with pytest.raises(oracle.OracleError):
        oracle.paged_attn_decode(q, "f16", kp, vp, "f16", tab, lens, scale=0.5)


# --------------------------------------------------------------------------
# paging invariants
# --------------------------------------------------------------------------

def test_permutation_of_physical_ids_changes_nothing():
    q, K, V, kp, vp, tab, lens = small_cache(40, 4, 4, 2, 16, 4, [3, 17, 32, 50], NB=60)
    ref = oracle.paged_attn_decode(q, "f16", kp, vp, "f16", tab, lens, scale=0.25)
    perm = np.random.default_rng(41).permutation(kp.shape[0])
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm] = kp
    vp2[perm] = vp
    tab2 = np.where(tab == wl.TABLE_POISON, tab, perm[np.clip(tab, 0, kp.shape[0] - 1)]).astype(np.int32)
    out = oracle.paged_attn_decode(q, "f16", kp2, vp2, "f16", tab2, lens, scale=0.25)
    assert np.array_equal(out, ref)


def test_shared_prefix_equals_private_copies():
    """Sequences whose tables point at the same prefix blocks give the result of private copies."""
    w = wl.make("prefix", small=True)
    kp, vp = w.initial_pool("k"), w.initial_pool("v")
    for op in w.setup:
        if isinstance(op, wl.Scatter):
            oracle.reshape_and_cache(op.k, op.v, w.src_dtype, kp, vp, w.kv_dtype, op.slots)
        else:
            oracle.copy_blocks(kp, vp, op.pairs)
    sc = w.step_scatter
    oracle.reshape_and_cache(sc.k, sc.v, w.src_dtype, kp, vp, w.kv_dtype, sc.slots)
    shared = oracle.paged_attn_decode(w.q, w.q_dtype, kp, vp, w.kv_dtype, w.block_tables,
                                      w.context_lens, w.scale)
    # private copies: every (sequence, block) gets its own physical block
    S = w.num_seqs
    nblk = (w.context_lens + w.block_size - 1) // w.block_size
    total = int(nblk.sum())
    kp2 = np.empty((total,) + kp.shape[1:], kp.dtype)
    vp2 = np.empty_like(kp2)
    tab2 = np.full_like(w.block_tables, wl.TABLE_POISON)
    n = 0
    for s in range(S):
        for j in range(int(nblk[s])):
            kp2[n], vp2[n] = kp[w.block_tables[s, j]], vp[w.block_tables[s, j]]
            tab2[s, j] = n
            n += 1
    private = oracle.paged_attn_decode(w.q, w.q_dtype, kp2, vp2, w.kv_dtype, tab2,
                                       w.context_lens, w.scale)
    assert np.array_equal(shared, private)
    # the shared structure is real: prefix blocks are referenced by all 8 samples
    assert len(set(w.block_tables[:8, 0].tolist())) == 1
    # and the partial block was copied for 7 samples, kept by the 8th
    blk32 = w.block_tables[:8, 32].tolist()
    assert len(set(blk32)) == 8


# --------------------------------------------------------------------------
# scatter and copy
# --------------------------------------------------------------------------

def test_scatter_gather_roundtrip_and_skip():
    rng = np.random.default_rng(50)
    NB, Hkv, B, D, T = 12, 3, 4, 8, 30
    kp = wl.garbage_bytes(rng, NB * Hkv * B * D * 2).view(np.uint16).reshape(NB, Hkv, B, D)
    vp = kp.copy()
    before = kp.copy()
    slots = rng.choice(NB * B, size=T, replace=False).astype(np.int64)
    slots[::7] = -1
    k = wl.normal_bits(rng, (T, Hkv, D), "bf16")
    v = wl.normal_bits(rng, (T, Hkv, D), "bf16")
    oracle.reshape_and_cache(k, v, "bf16", kp, vp, "bf16", slots)
    written = np.zeros((NB, B), bool)
    for t, sl in enumerate(slots):
        if sl < 0:
            continue
        b, o = divmod(int(sl), B)
        assert np.array_equal(kp[b, :, o], k[t]) and np.array_equal(vp[b, :, o], v[t])
        written[b, o] = True
    assert np.array_equal(kp.transpose(0, 2, 1, 3)[~written], before.transpose(0, 2, 1, 3)[~written])


def test_scatter_fp8_quantises_each_element():
    rng = np.random.default_rng(51)
    NB, Hkv, B, D, T = 6, 2, 4, 16, 10
    kp = np.zeros((NB, Hkv, B, D), np.uint8)
    vp = np.zeros_like(kp)
    k = wl.normal_bits(rng, (T, Hkv, D), "f16")
    v = wl.normal_bits(rng, (T, Hkv, D), "f16")
    ks, vs = np.float32(0.01), np.float32(0.0123)
    slots = np.arange(T, dtype=np.int64) * 2
    oracle.reshape_and_cache(k, v, "f16", kp, vp, "e4m3", slots, ks, vs)
    kf = k.view(np.float16).astype(np.float32)
    for t in range(T):
        b, o = divmod(int(slots[t]), B)
        lib = torch.from_numpy(kf[t] / ks).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(kp[b, :, o], lib)
        deq = f64(kp[b, :, o], "e4m3") * float(ks)
        # within half a quantum (relative 2^-4) of the exact value, when not saturated
        np.testing.assert_array_less(np.abs(deq - kf[t]), np.abs(kf[t]) * 2.0 ** -4 + 2.0 ** -10 * float(ks) + 1e-12)


@pytest.mark.parametrize("name", ["fp8", "fp8_b32"])
def test_fp8_cache_error_against_the_unquantised_cache(name):
    """The E4M3 cache against the same f16 values kept in 16 bits (decode, float64 oracle on
    both): the quantisation moves the output by well under the FP8 max-abs budget of 3e-2, and by
    a relative L2 in the range that 3-bit-mantissa rounding of K and V gives (a few per cent:
    an encoder that kept f16 precision would give ~0, a broken one far more).  Printed as
    information; the parity tests compare against the oracle on the dequantised cache."""
    w = wl.make(name, small=True)
    kq, vq = w.initial_pool("k"), w.initial_pool("v")
    k16 = np.zeros(kq.shape, np.uint16)
    v16 = np.zeros(kq.shape, np.uint16)
    for op in list(w.setup) + [w.step_scatter]:
        oracle.reshape_and_cache(op.k, op.v, w.src_dtype, kq, vq, "e4m3", op.slots, w.k_scale, w.v_scale)
        oracle.reshape_and_cache(op.k, op.v, w.src_dtype, k16, v16, "f16", op.slots)
    a = oracle.paged_attn_decode(w.q, w.q_dtype, kq, vq, "e4m3", w.block_tables, w.context_lens, w.scale,
                                 w.k_scale, w.v_scale)
    b = oracle.paged_attn_decode(w.q, w.q_dtype, k16, v16, "f16", w.block_tables, w.context_lens, w.scale)
    max_abs = float(np.abs(a - b).max())
    rel_l2 = float(np.linalg.norm(a - b) / np.linalg.norm(b))
    print(f"{name}: E4M3 vs f16 cache, max-abs {max_abs:.4f}, relative L2 {rel_l2:.4f}")
    assert max_abs < 3e-2
    assert 0.01 < rel_l2 < 0.1


def test_copy_blocks_copies_only_destinations():
    rng = np.random.default_rng(52)
    kp = wl.garbage_bytes(rng, 10 * 2 * 4 * 8 * 2).view(np.uint16).reshape(10, 2, 4, 8)
    vp = wl.garbage_bytes(rng, 10 * 2 * 4 * 8 * 2).view(np.uint16).reshape(10, 2, 4, 8)
    k0, v0 = kp.copy(), vp.copy()
    pairs = np.array([[1, 5], [1, 6], [3, 9]], np.int64)
    oracle.copy_blocks(kp, vp, pairs)
    for s, d in pairs:
        assert np.array_equal(kp[d], k0[s]) and np.array_equal(vp[d], v0[s])
    untouched = [0, 1, 2, 3, 4, 7, 8]
    assert np.array_equal(kp[untouched], k0[untouched]) and np.array_equal(vp[untouched], v0[untouched])


# --------------------------------------------------------------------------
# byte accounting against the pages' numbers
# --------------------------------------------------------------------------

def test_kv_bytes_match_pages():
    cases = json.load(open(os.path.join(GOLDEN, "kv_bytes.json")))["cases"]
    for c in cases:
        if "ratio" in c:
            assert wl.kv_bytes_per_token(1, 8, 128, 1) / wl.kv_bytes_per_token(1, 8, 128, 2) == c["ratio"]
            continue
        n = wl.kv_bytes_per_token(c["layers"], c["kv_heads"], c["head_dim"], c["elem_bytes"]) * c["tokens"]
        if "stated" in c:
            assert abs(n - c["stated"]) / c["stated"] <= c["rel_tol"], (c["what"], n)
        else:
            assert n <= c["stated_max"], (c["what"], n)


# --------------------------------------------------------------------------
# the comparison rule discriminates (mistakes planted in the oracle's inputs)
# --------------------------------------------------------------------------

def _ref_and_bits(w):
    kp, vp = w.initial_pool("k"), w.initial_pool("v")
    for op in w.setup:
        if isinstance(op, wl.Scatter):
            oracle.reshape_and_cache(op.k, op.v, w.src_dtype, kp, vp, w.kv_dtype, op.slots,
                                     w.k_scale, w.v_scale)
        else:
            oracle.copy_blocks(kp, vp, op.pairs)
    sc = w.step_scatter
    oracle.reshape_and_cache(sc.k, sc.v, w.src_dtype, kp, vp, w.kv_dtype, sc.slots, w.k_scale, w.v_scale)
    return kp, vp


@pytest.mark.parametrize("name", ["opt13b", "gqa"])
def test_tolerance_rejects_planted_mistakes(name):
    w = wl.make(name, small=True)
    kp, vp = _ref_and_bits(w)
    args = dict(k_scale=w.k_scale, v_scale=w.v_scale)
    ref = oracle.paged_attn_decode(w.q, w.q_dtype, kp, vp, w.kv_dtype, w.block_tables, w.context_lens,
                                   w.scale, **args)
    ok, _ = attention_close(ref, ref, w.kv_dtype, w.q_dtype)
    assert ok
    # correctly rounded output passes
    if w.q_dtype == "f16":
        rounded = ref.astype(np.float16).astype(np.float64)
    else:
        rounded = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    assert attention_close(rounded, ref, w.kv_dtype, w.q_dtype)[0]
    lens = w.context_lens
    long_seq = int(np.argmax(lens))
    mistakes = {}
    off = lens.copy()
    off[long_seq] -= 1                                          # drop the new token (off-by-one mask)
    mistakes["off_by_one"] = (w.block_tables, off)
    drop = lens.copy()
    drop[long_seq] -= (lens[long_seq] - 1) % w.block_size + 1   # drop the last block
    mistakes["drop_last_block"] = (w.block_tables, drop)
    # swapping two full blocks is invisible (the softmax sum does not depend on token
    # order); swapping a full block with the partial last block changes which slots count
    partial = [s for s in range(w.num_seqs) if lens[s] % w.block_size and lens[s] > w.block_size]
    s0 = max(partial, key=lambda s: lens[s])
    last = (int(lens[s0]) - 1) // w.block_size
    sw = w.block_tables.copy()
    sw[s0, [0, last]] = sw[s0, [last, 0]]
    mistakes["swap_with_partial_block"] = (sw, lens)
    other = w.block_tables.copy()
    s1 = (long_seq + 1) % w.num_seqs
    other[long_seq, 0] = other[s1, 0]                            # a block of another sequence
    mistakes["foreign_block"] = (other, lens)
    for what, (tab, ln) in mistakes.items():
        bad = oracle.paged_attn_decode(w.q, w.q_dtype, kp, vp, w.kv_dtype, tab, ln, w.scale, **args)
        assert not attention_close(bad, ref, w.kv_dtype, w.q_dtype)[0], what


def test_swap_blocks_round_trip_and_untouched_blocks():
    """Swap-out then swap-in through another pool restores the blocks bit for bit; blocks
    that no pair names are unchanged on both sides; a pair outside either pool is rejected."""
    rng = np.random.default_rng(70)
    gk = wl.garbage_bytes(rng, 12 * 2 * 16 * 8 * 2).view(np.uint16).reshape(12, 2, 16, 8)
    gv = wl.garbage_bytes(rng, gk.nbytes).view(np.uint16).reshape(gk.shape)
    hk = wl.garbage_bytes(rng, 5 * gk[0].nbytes).view(np.uint16).reshape(5, 2, 16, 8)
    hv = wl.garbage_bytes(rng, hk.nbytes).view(np.uint16).reshape(hk.shape)
    gk0, gv0, hk0, hv0 = gk.copy(), gv.copy(), hk.copy(), hv.copy()
    out = np.array([[3, 0], [7, 4], [11, 1]])
    oracle.swap_blocks(gk, gv, hk, hv, out)
    for s, d in out:
        assert np.array_equal(hk[d], gk0[s]) and np.array_equal(hv[d], gv0[s])
    for d in (2, 3):
        assert np.array_equal(hk[d], hk0[d]) and np.array_equal(hv[d], hv0[d])
    assert np.array_equal(gk, gk0) and np.array_equal(gv, gv0)            # the source is only read
    gk[[3, 7, 11]] = 0                                                     # the GPU blocks are reused meanwhile
    back = np.array([[0, 9], [4, 2], [1, 5]])                              # swap in to other blocks
    oracle.swap_blocks(hk, hv, gk, gv, back)
    for (s_out, _), (_, d_in) in zip(out, back):
        assert np.array_equal(gk[d_in], gk0[s_out]) and np.array_equal(gv[d_in], gv0[s_out])
    with pytest.raises(oracle.OracleError):
        oracle.swap_blocks(gk, gv, hk, hv, np.array([[0, 5]]))             # destination beyond the host pool
