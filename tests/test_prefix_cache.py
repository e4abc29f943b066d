"""Prefix caching and copy-on-write of the C++ block manager against the oracle's
model (CPU): identical tables, lengths, refcounts, free and cached counts,
cached-token counts, slots and copy lists on seeded random traces that mix
admission by token ids (small vocabularies, so prefixes repeat), whole forks,
appends with and without ids, plain admissions and releases."""
import numpy as np
import pytest

import oracle
import pagedattention_kv_cache_pa_b200 as pa


def _same(bm: pa.BlockManager, m: oracle.BlockManagerModel):
    tables = bm.block_tables()
    for s in range(m.max_seqs):
        assert list(tables[s]) == m.table_array(s)
    assert list(bm.context_lens()) == m.lens
    assert bm.num_free() == m.num_free()
    assert bm.num_cached_blocks() == m.num_cached()
    assert [bm.refcount(b) for b in range(m.num_blocks)] == m.ref


def _expect_oom(fn):
    with pytest.raises(pa.PaError) as e:
        fn()
    assert e.value.status == -5


@pytest.mark.parametrize("seed,Bs", [(1, 4), (2, 16), (3, 1), (4, 8)])
def test_random_trace_matches_model(seed, Bs):
    rng = np.random.default_rng(seed)
    N, S, MB = 48, 9, 64
    order = rng.permutation(N).astype(np.int32)
    bm = pa.BlockManager(N, Bs, S, MB, order)
    m = oracle.BlockManagerModel(N, Bs, S, MB, order)
    prompts = [list(rng.integers(0, 2, 80)) for _ in range(3)]   # few distinct prompt stems
    for step in range(500):
        r = rng.random()
        live = [s for s in range(S) if m.live[s]]
        dead = [s for s in range(S) if not m.live[s]]
        if dead and r < 0.25:
            s = int(rng.choice(dead))
            stem = prompts[int(rng.integers(0, 3))]
            ids = [int(t) for t in stem[: int(rng.integers(0, 5 * Bs + 3))]]
            if rng.random() < 0.3 and ids:
                ids[-1] = 7                                      # a different tail
            try:
                want = m.add_seq_tokens(s, ids)
            except oracle.OutOfBlocks:
                _expect_oom(lambda: bm.add_seq_tokens(s, ids))
            else:
                assert bm.add_seq_tokens(s, ids) == want
        elif dead and live and r < 0.35:
            s, src = int(rng.choice(dead)), int(rng.choice(live))
            m.fork_all(s, src)
            bm.fork_all(s, src)
        elif dead and r < 0.4:
            s, n = int(rng.choice(dead)), int(rng.integers(0, 3 * Bs))
            try:
                m.add_seq(s, n)
            except oracle.OutOfBlocks:
                _expect_oom(lambda: bm.add_seq(s, n))
            else:
                bm.add_seq(s, n)
        elif live and r < 0.55:
            s = int(rng.choice(live))
            m.free_seq(s)
            bm.free_seq(s)
        elif live:
            pick = [s for s in live if rng.random() < 0.6 and m.lens[s] < MB * Bs - 1]
            ids = [int(t) for t in rng.integers(0, 2, len(pick))]
            plain = rng.random() < 0.1
            try:
                want = m.append_tokens(pick) if plain else m.append_token_ids(pick, ids)
            except oracle.OutOfBlocks:
                _expect_oom(lambda: bm.append_tokens(pick) if plain else bm.append_token_ids(pick, ids))
            except oracle.SharedBlockWrite:
                with pytest.raises(pa.PaError) as e:
                    bm.append_tokens(pick)
                assert e.value.status == -6
            else:
                if plain:
                    assert list(bm.append_tokens(pick)) == want
                else:
                    slots, copies = bm.append_token_ids(pick, ids)
                    assert list(slots) == want[0]
                    assert [tuple(c) for c in copies.tolist()] == want[1]
        _same(bm, m)
    bm.close()


def test_shared_system_prompt_is_found_cached():
    # C3-like: 32 requests with one 1024-token prefix (4 blocks of 256) and own suffixes
    Bs, N = 256, 400
    bm = pa.BlockManager(N, Bs, 32, 40, np.arange(N, dtype=np.int32))
    rng = np.random.default_rng(7)
    prefix = [int(t) for t in rng.integers(0, 32000, 1024)]
    cached = []
    for s in range(32):
        suffix = [int(t) for t in rng.integers(0, 32000, int(rng.integers(256, 2048)))]
        cached.append(bm.add_seq_tokens(s, prefix + suffix))
    assert cached[0] == 0 and all(c == 1024 for c in cached[1:])
    roots = {tuple(bm.block_tables()[s][:4]) for s in range(32)}
    assert len(roots) == 1 and bm.refcount(int(bm.block_tables()[0][0])) == 32
    bm.close()


def test_invalid_arguments():
    bm = pa.BlockManager(8, 4, 2, 4, np.arange(8, dtype=np.int32))
    with pytest.raises(pa.PaError):
        bm.add_seq_tokens(0, list(range(17)))                 # more than max_blocks_per_seq
    with pytest.raises(pa.PaError):
        bm.fork_all(0, 1)                                     # source not live
    bm.add_seq_tokens(0, [1, 2, 3])
    with pytest.raises(pa.PaError):
        bm.fork_all(0, 0)
    with pytest.raises(pa.PaError):
        bm.append_token_ids([1], [5])                         # not live
    bm.close()
