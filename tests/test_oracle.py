"""Pins for the fp64 oracle: what the pages and the mathematics fix, not the oracle itself.

Each test checks the oracle against something independent of its C code:
values the pages print (golden files), closed forms, invariants the paging
idea implies, or a brute-force formulation that builds each sequence
contiguously first and never touches a pool.
"""
import math
import os

import numpy as np
import pytest

import oracle
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(values):
    """float values that are exactly representable in bf16 -> bit patterns."""
    f = np.asarray(values, dtype=np.float32)
    bits = f.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0), "value not exact in bf16"
    return (bits >> 16).astype(np.uint16)


def _page(seqs_k, seqs_v, block_size, num_blocks, order, fill_seed=7):
    """Scatter contiguous sequences (lists of [Hkv, L, D] float arrays with bf16-exact values)
    into a pool using numpy slicing; physical blocks come from `order`.
    Returns (k_cache, v_cache, tables, lens)."""
    Hkv, _, D = seqs_k[0].shape
    Bs = block_size
    rng = np.random.default_rng(fill_seed)
    junk = lambda: _bf16(np.round(rng.standard_normal((num_blocks, Hkv, Bs, D)) * 8) / 8)
    k_cache, v_cache = junk(), junk()
    lens = np.array([s.shape[1] for s in seqs_k], dtype=np.int32)
    nblocks = [-(-int(L) // Bs) for L in lens]
    MB = max(max(nblocks), 1)
    tables = np.full((len(seqs_k), MB), -1, dtype=np.int32)
    it = iter(order)
    for b, (K, V) in enumerate(zip(seqs_k, seqs_v)):
        L = K.shape[1]
        for i in range(nblocks[b]):
            phys = next(it)
            tables[b, i] = phys
            lo, hi = i * Bs, min(L, (i + 1) * Bs)
            k_cache[phys, :, : hi - lo, :] = _bf16(K[:, lo:hi, :])
            v_cache[phys, :, : hi - lo, :] = _bf16(V[:, lo:hi, :])
    return k_cache, v_cache, tables, lens


def _random_seqs(rng, lens, Hkv, D, quant=16.0):
    """bf16-exact contiguous K/V per sequence (multiples of 1/quant, few significant bits)."""
    ks = [np.round(rng.standard_normal((Hkv, L, D)) * quant) / quant for L in lens]
    vs = [np.round(rng.standard_normal((Hkv, L, D)) * quant) / quant for L in lens]
    return ks, vs


def _brute(q, ks, vs, scale, Hq):
    """Contiguous attention in long double: no pool, no table, no gather."""
    B = len(ks)
    Hkv = ks[0].shape[0]
    D = q.shape[-1]
    g = Hq // Hkv
    out = np.zeros((B, Hq, D), dtype=np.longdouble)
    for b in range(B):
        for kvh in range(Hkv):
            K = ks[b][kvh].astype(np.longdouble)
            V = vs[b][kvh].astype(np.longdouble)
            if K.shape[0] == 0:
                continue
            for i in range(g):
                h = kvh * g + i
                s = (K @ q[b, h].astype(np.longdouble)) * np.longdouble(scale)
                e = np.exp(s - s.max())
                out[b, h] = (e / e.sum()) @ V
    return out.astype(np.float64)


# --------------------------------------------------------------------------------------------
# values the pages print
# --------------------------------------------------------------------------------------------
def test_kv_bytes_matches_page_example():
    line = [l for l in open(os.path.join(GOLDEN, "kv_bytes_llama2_70b.txt")) if not l.startswith("#")][0]
    f = dict(kv.split("=") for kv in line.split())
    n = oracle.kv_bytes(int(f["layers"]), int(f["kv_heads"]), int(f["head_dim"]),
                        int(f["tokens"]), int(f["bytes_per_element"]))
    approx = float(f["approx_bytes"])
    assert abs(n - approx) / approx < 0.08            # "about 10GB"
    assert n == 10 * 2 ** 30                          # the printed factors multiply to 10 GiB
    assert n * int(f["requests"]) > float(f["a100_bytes"])  # ten requests exceed an A100 80GB


def test_bf16_widening_matches_layout():
    for line in open(os.path.join(GOLDEN, "bf16_values.txt")):
        if line.startswith("#") or not line.strip():
            continue
        bits, value = line.split()
        got = oracle.bf16_to_double(int(bits, 16))
        want = float(value)
        if math.isinf(want):
            assert got == want
        else:
            assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want)


def test_slot_matches_worked_example():
    for line in open(os.path.join(GOLDEN, "slot_mapping_example.txt")):
        if line.startswith("#") or not line.strip():
            continue
        table, bs, pos, slot = line.split()
        row = np.array([int(x) for x in table.split(",")], dtype=np.int32)
        assert oracle.slot(row, int(pos), int(bs)) == int(slot)


# --------------------------------------------------------------------------------------------
# closed forms of softmax attention
# --------------------------------------------------------------------------------------------
def _one_seq(K, V, q, scale, block_size=16, Hq=None):
    """K, V: [Hkv, L, D] float (bf16-exact); q: [Hq, D]."""
    Hkv, L, D = K.shape
    N = max(-(-L // block_size), 1) + 2
    order = list(range(N))[::-1]
    kc, vc, tables, lens = _page([K], [V], block_size, N, order)
    qb = _bf16(q)[None]
    return oracle.paged_decode(qb, kc, vc, tables, lens, scale)[0]


def test_context_of_one_returns_that_value():
    rng = np.random.default_rng(1)
    K = np.round(rng.standard_normal((1, 1, 64)) * 16) / 16
    V = np.round(rng.standard_normal((1, 1, 64)) * 16) / 16
    q = np.round(rng.standard_normal((3, 64)) * 16) / 16
    out = _one_seq(K, V, q, 0.125)
    for h in range(3):
        np.testing.assert_array_equal(out[h], V[0, 0])


def test_zero_query_gives_mean_of_values():
    rng = np.random.default_rng(2)
    L = 37
    K = np.round(rng.standard_normal((1, L, 64)) * 16) / 16
    V = np.round(rng.standard_normal((1, L, 64)) * 16) / 16
    out = _one_seq(K, V, np.zeros((1, 64)), 0.125)
    np.testing.assert_allclose(out[0], V[0].mean(axis=0), rtol=0, atol=1e-14)


def test_identical_keys_give_mean_of_values():
    rng = np.random.default_rng(3)
    L = 50
    k = np.round(rng.standard_normal(64) * 16) / 16
    K = np.broadcast_to(k, (1, L, 64)).copy()
    V = np.round(rng.standard_normal((1, L, 64)) * 16) / 16
    q = np.round(rng.standard_normal((2, 64)) * 16) / 16
    out = _one_seq(K, V, q, 0.125)
    for h in range(2):
        np.testing.assert_allclose(out[h], V[0].mean(axis=0), rtol=0, atol=1e-14)


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(4)
    L, D = 40, 64
    q = np.zeros((1, D)); q[0, 5] = 1.0
    K = np.round(rng.standard_normal((1, L, D)) * 4) / 64          # |scores| tiny
    K[0, 23, :] = 0.0; K[0, 23, 5] = 256.0                          # s_23 = 256 * scale
    V = np.round(rng.standard_normal((1, L, D)) * 16) / 16
    out = _one_seq(K, V, q, 1.0)
    np.testing.assert_allclose(out[0], V[0, 23], rtol=0, atol=1e-12)


def test_two_tokens_closed_form_and_scale():
    # q = e_0, K_0 = 0, K_1 = 2 e_0: scores 0 and 2*scale.  With scale = ln(3)/2 the
    # weights are 1/4 and 3/4; doubling the scale gives 1/10 and 9/10.
    D = 64
    q = np.zeros((1, D)); q[0, 0] = 1.0
    K = np.zeros((1, 2, D)); K[0, 1, 0] = 2.0
    V = np.zeros((1, 2, D)); V[0, 0, :] = 1.0; V[0, 1, :] = -2.0; V[0, 1, 3] = 4.0
    out = _one_seq(K, V, q, math.log(3.0) / 2.0)
    want = 0.25 * V[0, 0] + 0.75 * V[0, 1]
    np.testing.assert_allclose(out[0], want, rtol=0, atol=1e-14)
    out2 = _one_seq(K, V, q, math.log(3.0))
    want2 = 0.1 * V[0, 0] + 0.9 * V[0, 1]
    np.testing.assert_allclose(out2[0], want2, rtol=0, atol=1e-14)


def test_query_head_reads_its_group_kv_head():
    # Hq=8, Hkv=2: heads 0-3 must read kv head 0, heads 4-7 kv head 1 (contiguous groups).
    L, D = 20, 64
    rng = np.random.default_rng(5)
    K = np.round(rng.standard_normal((2, L, D)) * 16) / 16
    V = np.zeros((2, L, D)); V[0] = 1.0; V[1] = -1.0
    q = np.round(rng.standard_normal((8, D)) * 16) / 16
    out = _one_seq(K, V, q, 0.125)
    np.testing.assert_allclose(out[:4], np.ones((4, D)), rtol=0, atol=1e-14)
    np.testing.assert_allclose(out[4:], -np.ones((4, D)), rtol=0, atol=1e-14)


def test_weights_sum_to_one():
    b = wl.small_batch(11, [1, 15, 16, 17, 300], num_q_heads=6, num_kv_heads=2)
    out, wsum = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens,
                                    b.scale, return_weight_sums=True)
    np.testing.assert_allclose(wsum, 1.0, rtol=0, atol=1e-13)


def test_empty_sequence_gives_zeros():
    b = wl.small_batch(12, [0, 9], num_q_heads=2, num_kv_heads=1)
    out = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale)
    assert np.all(out[0] == 0.0)
    assert np.any(out[1] != 0.0)


# --------------------------------------------------------------------------------------------
# brute force: contiguous sequences, no pool
# --------------------------------------------------------------------------------------------
@pytest.mark.parametrize("Hq,Hkv,D,Bs,lens", [
    (2, 1, 64, 16, [5, 37]),
    (4, 2, 64, 8, [1, 7, 8, 9, 33]),
    (8, 2, 128, 16, [15, 16, 17, 64]),
    (6, 2, 64, 32, [31, 32, 33, 100]),
    (3, 3, 64, 1, [1, 2, 5]),
    (16, 2, 128, 256, [255, 256, 257]),
])
def test_matches_contiguous_brute_force(Hq, Hkv, D, Bs, lens):
    rng = np.random.default_rng(sum(lens) + Bs)
    ks, vs = _random_seqs(rng, lens, Hkv, D)
    N = sum(-(-L // Bs) for L in lens) + 3
    order = rng.permutation(N)
    kc, vc, tables, L = _page(ks, vs, Bs, N, order)
    q = np.round(rng.standard_normal((len(lens), Hq, D)) * 16) / 16
    scale = 1.0 / math.sqrt(D)
    got = oracle.paged_decode(_bf16(q), kc, vc, tables, L, scale)
    want = _brute(q, ks, vs, scale, Hq)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------------------------
# invariants of paging
# --------------------------------------------------------------------------------------------
def test_physical_block_permutation_changes_nothing():
    b = wl.small_batch(21, [3, 16, 40, 129], num_q_heads=8, num_kv_heads=2)
    ref = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale)
    perm = np.random.default_rng(0).permutation(b.num_blocks).astype(np.int32)  # old -> new id
    kc = np.empty_like(b.k_cache); vc = np.empty_like(b.v_cache)
    kc[perm] = b.k_cache; vc[perm] = b.v_cache
    tables = np.where(b.block_tables >= 0, perm[np.maximum(b.block_tables, 0)], -1).astype(np.int32)
    got = oracle.paged_decode(b.q, kc, vc, tables, b.context_lens, b.scale)
    np.testing.assert_array_equal(got, ref)


def test_block_size_is_a_storage_detail():
    rng = np.random.default_rng(22)
    lens = [1, 17, 40, 300]
    ks, vs = _random_seqs(rng, lens, 2, 64)
    q = _bf16(np.round(rng.standard_normal((4, 4, 64)) * 16) / 16)
    outs = []
    for Bs in (1, 8, 16, 256):
        N = sum(-(-L // Bs) for L in lens) + 2
        kc, vc, tables, L = _page(ks, vs, Bs, N, rng.permutation(N))
        outs.append(oracle.paged_decode(q, kc, vc, tables, L, 0.125))
    for o in outs[1:]:
        np.testing.assert_array_equal(o, outs[0])


def test_shared_prefix_blocks_match_private_copies():
    b = wl.make_batch("prefix", 31, [32 + 5, 32 + 40, 32 + 16], num_q_heads=4, num_kv_heads=2,
                      head_dim=64, block_size=16, shared_prefix_tokens=32)
    assert (b.block_tables[:, :2] == b.block_tables[0, :2]).all()
    ref = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale)
    # give every sequence its own copy of the two prefix blocks
    B = b.batch
    extra = 2 * B
    kc = np.concatenate([b.k_cache, np.zeros((extra,) + b.k_cache.shape[1:], np.uint16)])
    vc = np.concatenate([b.v_cache, np.zeros((extra,) + b.v_cache.shape[1:], np.uint16)])
    tables = b.block_tables.copy()
    for s in range(B):
        for i in range(2):
            new = b.num_blocks + 2 * s + i
            kc[new] = b.k_cache[b.block_tables[s, i]]
            vc[new] = b.v_cache[b.block_tables[s, i]]
            tables[s, i] = new
    got = oracle.paged_decode(b.q, kc, vc, tables, b.context_lens, b.scale)
    np.testing.assert_array_equal(got, ref)


def test_batch_permutation_permutes_outputs():
    b = wl.small_batch(41, [5, 60, 17, 33], num_q_heads=4, num_kv_heads=2)
    ref = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale)
    p = np.array([2, 0, 3, 1])
    got = oracle.paged_decode(b.q[p], b.k_cache, b.v_cache, b.block_tables[p], b.context_lens[p], b.scale)
    np.testing.assert_array_equal(got, ref[p])


# --------------------------------------------------------------------------------------------
# split-KV partial states and their merge
# --------------------------------------------------------------------------------------------
def test_merge_closed_form():
    o = np.array([[1.0, 2.0], [3.0, -4.0]])
    # equal log-sum-exps: plain average
    np.testing.assert_allclose(oracle.merge_partials(o, np.array([0.7, 0.7])), [2.0, -1.0], atol=1e-15)
    # second split carries 3x the mass: weights 1/4, 3/4
    np.testing.assert_allclose(oracle.merge_partials(o, np.array([0.0, math.log(3.0)])),
                               [0.25 * 1 + 0.75 * 3, 0.25 * 2 - 0.75 * 4], atol=1e-15)
    # an empty split (lse = -inf) has no weight
    np.testing.assert_allclose(oracle.merge_partials(o, np.array([-np.inf, 5.0])), o[1], atol=0)
    assert np.all(oracle.merge_partials(o, np.array([-np.inf, -np.inf])) == 0.0)


@pytest.mark.parametrize("cuts", [[0, 1, 64], [0, 16, 32, 48, 64], [0, 5, 6, 63, 64], [0, 64]])
def test_merge_of_partials_equals_unsplit(cuts):
    b = wl.small_batch(51, [64, 64], num_q_heads=8, num_kv_heads=2, head_dim=128)
    full = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale)
    parts = [oracle.paged_decode_partial(b.q, b.k_cache, b.v_cache, b.block_tables,
                                         b.context_lens, b.scale, lo, hi)
             for lo, hi in zip(cuts[:-1], cuts[1:])]
    for s in range(b.batch):
        for h in range(8):
            o = np.stack([p[0][s, h] for p in parts])
            lse = np.array([p[1][s, h] for p in parts])
            np.testing.assert_allclose(oracle.merge_partials(o, lse), full[s, h], rtol=0, atol=1e-12)


def test_partial_lse_is_log_of_exp_sum():
    # one token with score s gives lse = s; two equal scores give s + ln 2
    D = 64
    q = np.zeros((1, D)); q[0, 0] = 1.0
    K = np.zeros((1, 2, D)); K[0, :, 0] = 3.0
    V = np.ones((1, 2, D))
    kc, vc, tables, lens = _page([K], [V], 16, 2, [1, 0])
    o, lse = oracle.paged_decode_partial(_bf16(q)[None], kc, vc, tables, lens, 0.5, 0, 1)
    assert abs(lse[0, 0] - 1.5) < 1e-15
    o, lse = oracle.paged_decode_partial(_bf16(q)[None], kc, vc, tables, lens, 0.5, 0, 2)
    assert abs(lse[0, 0] - (1.5 + math.log(2.0))) < 1e-15
    o, lse = oracle.paged_decode_partial(_bf16(q)[None], kc, vc, tables, lens, 0.5, 2, 9)
    assert lse[0, 0] == -np.inf and np.all(o == 0)


# --------------------------------------------------------------------------------------------
# append through the slot mapping
# --------------------------------------------------------------------------------------------
def test_append_writes_exactly_the_mapped_slots():
    b = wl.small_batch(61, [5, 16, 31], num_q_heads=4, num_kv_heads=2, num_blocks=12)
    N, Hkv, Bs, D = b.k_cache.shape
    T = 5
    k = wl.normal_bf16(99, (T, Hkv, D))
    v = wl.normal_bf16(98, (T, Hkv, D))
    slots = np.array([3, -1, 5 * Bs + 7, N * Bs, N * Bs - 1], dtype=np.int64)
    kc, vc = oracle.append_kv(k, v, slots, b.k_cache, b.v_cache)
    want_k = b.k_cache.copy(); want_v = b.v_cache.copy()
    flat_k = want_k.transpose(0, 2, 1, 3).reshape(N * Bs, Hkv, D)   # slot-major view
    flat_v = want_v.transpose(0, 2, 1, 3).reshape(N * Bs, Hkv, D)
    for t, s in enumerate(slots):
        if 0 <= s < N * Bs:
            flat_k[s] = k[t]; flat_v[s] = v[t]
    want_k = flat_k.reshape(N, Bs, Hkv, D).transpose(0, 2, 1, 3)
    want_v = flat_v.reshape(N, Bs, Hkv, D).transpose(0, 2, 1, 3)
    np.testing.assert_array_equal(kc, want_k)
    np.testing.assert_array_equal(vc, want_v)


def test_append_then_attend_round_trip():
    # append a token whose key dominates at position p, then decode over p+1 tokens:
    # the output must be the appended value (slot mapping and gather agree).
    b = wl.small_batch(62, [16, 47], num_q_heads=2, num_kv_heads=1, num_blocks=8)
    N, Hkv, Bs, D = b.k_cache.shape
    lens_after = b.context_lens + 1
    tables = b.block_tables.copy()
    for s in range(b.batch):     # give the new token a block when the last one is full
        p = int(b.context_lens[s])
        if p % Bs == 0:
            tables[s, p // Bs] = b.free_order[s]
    q = np.zeros((b.batch, 2, D), np.float64); q[:, :, 0] = 1.0
    k = np.zeros((b.batch, 1, D)); k[:, 0, 0] = 256.0
    vnew = np.round(np.random.default_rng(3).standard_normal((b.batch, 1, D)) * 16) / 16
    slots = oracle.slot_mapping(tables, lens_after, Bs)
    kc, vc = oracle.append_kv(_bf16(k), _bf16(vnew), slots, b.k_cache, b.v_cache)
    out = oracle.paged_decode(_bf16(q), kc, vc, tables, lens_after, 1.0)
    for s in range(b.batch):
        np.testing.assert_allclose(out[s, 0], vnew[s, 0], rtol=0, atol=1e-9)


def test_slot_mapping_of_newest_tokens():
    tables = np.array([[7, 2, 5, -1], [3, 0, -1, -1]], dtype=np.int32)
    lens = np.array([41, 9], dtype=np.int32)
    np.testing.assert_array_equal(oracle.slot_mapping(tables, lens, 16), [5 * 16 + 8, 3 * 16 + 8])
    np.testing.assert_array_equal(oracle.slot_mapping(tables, np.array([0, 1], np.int32), 16), [-1, 48])
