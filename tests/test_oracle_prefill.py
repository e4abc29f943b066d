"""Pins of the oracle's paged (chunked) prefill against what its definition fixes.

Reading: sequence b holds context_lens[b] = L tokens after this step's append; its
last Tq tokens are the queries (positions L-Tq .. L-1) and the query at position p
attends to cache tokens 0..p (the causal mask of the Tiny-vLLM summary page, section
"고성능 추론을 위한 고급 최적화 기법").  Pinned by: per-query decodes over the
truncated context (a different loop of the oracle), the one-query case, causality
(keys after p do not matter, keys up to p do), chunk splitting, and two closed forms
computed outside the oracle from hand-gathered V rows: q = 0 gives the running mean of V,
and one dominant key returns its own V from its position on.
"""
import numpy as np

import oracle
import workloads as wl


def _case(seed, lens, q_lens, **kw):
    b = wl.small_batch(seed, lens, **kw)
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q = (rng.standard_normal((int(cu[-1]), b.num_q_heads, b.head_dim)).astype(np.float32)
         .view(np.uint32) >> 16).astype(np.uint16)
    return b, q, cu


def test_each_query_is_a_decode_over_its_prefix():
    lens, q_lens = [37, 90, 16], [5, 33, 16]
    b, q, cu = _case(3, lens, q_lens, num_q_heads=8, num_kv_heads=2, head_dim=64, block_size=16)
    out = oracle.paged_prefill(q, b.k_cache, b.v_cache, b.block_tables, cu, b.context_lens, b.scale)
    for s in range(len(lens)):
        L = int(b.context_lens[s])
        for i in range(q_lens[s]):
            pos = L - q_lens[s] + i
            row = int(cu[s]) + i
            want = oracle.paged_decode(q[row:row + 1], b.k_cache, b.v_cache, b.block_tables[s:s + 1],
                                       np.array([pos + 1], dtype=np.int32), b.scale)
            np.testing.assert_allclose(out[row], want[0], rtol=0, atol=1e-13)


def test_one_query_per_sequence_is_the_decode():
    b = wl.small_batch(4, [20, 7, 100], num_q_heads=4, num_kv_heads=4, head_dim=128, block_size=8)
    cu = np.arange(4, dtype=np.int32)
    out = oracle.paged_prefill(b.q, b.k_cache, b.v_cache, b.block_tables, cu, b.context_lens, b.scale)
    want = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale)
    np.testing.assert_array_equal(out, want)


def test_causality():
    b, q, cu = _case(5, [48], [48], num_q_heads=2, num_kv_heads=1, head_dim=64, block_size=16)
    out = oracle.paged_prefill(q, b.k_cache, b.v_cache, b.block_tables, cu, b.context_lens, b.scale)
    k2, v2 = b.k_cache.copy(), b.v_cache.copy()
    p = 20                                        # change every key and value after position 20
    for pos in range(p + 1, 48):
        blk, off = b.block_tables[0][pos // 16], pos % 16
        k2[blk, :, off, :] ^= 0x0040
        v2[blk, :, off, :] ^= 0x0040
    out2 = oracle.paged_prefill(q, k2, v2, b.block_tables, cu, b.context_lens, b.scale)
    np.testing.assert_array_equal(out2[:p + 1], out[:p + 1])   # queries 0..20 see only 0..p
    assert np.abs(out2[p + 1:] - out[p + 1:]).max() > 1e-6      # later ones see the change


def test_a_prefill_split_into_chunks_gives_the_same_outputs():
    b, q, cu = _case(6, [70], [70], num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16)
    whole = oracle.paged_prefill(q, b.k_cache, b.v_cache, b.block_tables, cu, b.context_lens, b.scale)
    a = 29
    first = oracle.paged_prefill(q[:a], b.k_cache, b.v_cache, b.block_tables, np.array([0, a], dtype=np.int32),
                                 np.array([a], dtype=np.int32), b.scale)
    second = oracle.paged_prefill(q[a:], b.k_cache, b.v_cache, b.block_tables,
                                  np.array([0, 70 - a], dtype=np.int32), np.array([70], dtype=np.int32), b.scale)
    np.testing.assert_array_equal(np.concatenate([first, second]), whole)


def _logical(cache, table_row, L, Bs):
    """The sequence's L tokens [L][Hkv][D] as float64, gathered through its table by hand."""
    idx = np.arange(L)
    rows = cache[table_row[idx // Bs], :, idx % Bs, :]
    return (rows.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_equal_scores_give_the_running_mean_of_v():
    # q = 0: every visible key scores 0, so the query at position p returns mean(V_0 .. V_p)
    lens, q_lens = [45, 70], [45, 20]
    b, q, cu = _case(8, lens, q_lens, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16)
    q[:] = 0
    out = oracle.paged_prefill(q, b.k_cache, b.v_cache, b.block_tables, cu, b.context_lens, b.scale)
    G = b.num_q_heads // b.num_kv_heads
    for s, (L, Tq) in enumerate(zip(lens, q_lens)):
        V = _logical(b.v_cache, b.block_tables[s], L, b.block_size)
        running = np.cumsum(V, axis=0) / np.arange(1, L + 1)[:, None, None]
        for i in range(Tq):
            for h in range(b.num_q_heads):
                np.testing.assert_allclose(out[cu[s] + i, h], running[L - Tq + i, h // G], rtol=0, atol=1e-12)


def test_a_dominant_key_takes_over_from_its_position_on():
    # every query is e_0 and key j has K[j][0] = 1000: from position j on it holds all the
    # weight (score 125 against O(0.1)), before j it is masked and changes nothing
    L, j, Bs = 50, 20, 16
    b, q, cu = _case(9, [L], [L], num_q_heads=2, num_kv_heads=1, head_dim=64, block_size=Bs)
    q[:] = 0
    q[:, :, 0] = 0x3F80                                          # bf16 1.0
    before = oracle.paged_prefill(q, b.k_cache, b.v_cache, b.block_tables, cu, b.context_lens, b.scale)
    k2 = b.k_cache.copy()
    k2[b.block_tables[0][j // Bs], :, j % Bs, 0] = 0x447A        # bf16 1000.0
    out = oracle.paged_prefill(q, k2, b.v_cache, b.block_tables, cu, b.context_lens, b.scale)
    np.testing.assert_array_equal(out[:j], before[:j])
    Vj = _logical(b.v_cache, b.block_tables[0], L, Bs)[j, 0]
    for pos in range(j, L):
        for h in range(2):
            np.testing.assert_allclose(out[pos, h], Vj, rtol=1e-12, atol=1e-12)
