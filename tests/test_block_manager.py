"""The C++ block manager (libpa, host) against the oracle's model of the same
policy: identical tables, slots, lengths, refcounts and free counts on seeded
random traces and on the continuous-batching trace (CPU only)."""
import numpy as np
import pytest

import oracle
import workloads as wl
import pagedattention_kv_cache_pa_b200 as pa


def _same(bm: pa.BlockManager, m: oracle.BlockManagerModel):
    tables = bm.block_tables()
    for s in range(m.max_seqs):
        assert list(tables[s]) == m.table_array(s)
    assert list(bm.context_lens()) == m.lens
    assert bm.num_free() == m.num_free()
    for blk in range(m.num_blocks):
        assert bm.refcount(blk) == m.ref[blk]


def test_random_trace_matches_model():
    rng = np.random.default_rng(1)
    N, Bs, S, MB = 96, 8, 7, 40
    order = rng.permutation(N).astype(np.int32)
    bm = pa.BlockManager(N, Bs, S, MB, order)
    m = oracle.BlockManagerModel(N, Bs, S, MB, order)
    for step in range(600):
        r = rng.random()
        live = [s for s in range(S) if m.live[s]]
        dead = [s for s in range(S) if not m.live[s]]
        if dead and r < 0.2:
            s, n = int(rng.choice(dead)), int(rng.integers(0, 60))
            try:
                m.add_seq(s, n)
                bm.add_seq(s, n)
            except oracle.OutOfBlocks:
                with pytest.raises(pa.PaError) as e:
                    bm.add_seq(s, n)
                assert e.value.status == -5
        elif live and r < 0.3:
            s = int(rng.choice(live))
            m.free_seq(s)
            bm.free_seq(s)
        elif live:
            pick = [s for s in live if rng.random() < 0.6]
            try:
                want = m.append_tokens(pick)
            except oracle.OutOfBlocks:
                with pytest.raises(pa.PaError) as e:
                    bm.append_tokens(pick)
                assert e.value.status == -5
            else:
                got = bm.append_tokens(pick)
                assert list(got) == want
        _same(bm, m)
    bm.close()


def test_shared_prefix_fork_and_refusal():
    N, Bs = 32, 4
    order = np.arange(N, dtype=np.int32)
    bm = pa.BlockManager(N, Bs, 3, 16, order)
    bm.add_seq(0, 10)                          # blocks 0,1,2 (2 is half full)
    bm.fork_seq(1, 0, 2, 9)                    # shares 0,1; own block for tokens 8
    t = bm.block_tables()
    assert list(t[1][:3]) == [0, 1, 3]
    assert bm.refcount(0) == 2 and bm.refcount(1) == 2 and bm.refcount(3) == 1
    with pytest.raises(pa.PaError):
        bm.fork_seq(2, 0, 3, 12)               # block 2 of seq 0 is not full
    bm.import_seq(2, 10, [0, 1, 2])            # a third table holding seq 0's blocks
    with pytest.raises(pa.PaError) as e:
        bm.append_tokens([0])                  # position 10 lands in shared block 2
    assert e.value.status == -6
    bm.free_seq(0)
    bm.free_seq(2)
    assert bm.refcount(2) == 0 and bm.refcount(0) == 1
    bm.close()


def test_dirty_rows():
    bm = pa.BlockManager(16, 4, 4, 8, np.arange(16, dtype=np.int32))
    bm.add_seq(2, 3)
    bm.add_seq(0, 4)
    assert list(bm.take_dirty_rows()) == [0, 2]
    assert list(bm.take_dirty_rows()) == []
    bm.append_tokens([0, 2])                  # seq 0 takes a block; seq 2 does not
    assert list(bm.take_dirty_rows()) == [0]
    bm.close()


def test_invalid_arguments():
    with pytest.raises(pa.PaError):
        pa.BlockManager(4, 4, 2, 4, [0, 0])    # duplicate free block
    with pytest.raises(pa.PaError):
        pa.BlockManager(4, 4, 2, 4, [7])       # out of range
    bm = pa.BlockManager(4, 4, 2, 4, [0, 1])
    with pytest.raises(pa.PaError):
        bm.import_seq(0, 4, [0])               # block 0 is on the free stack
    with pytest.raises(pa.PaError):
        bm.free_seq(1)                         # not live
    bm.close()


def test_continuous_batching_trace_matches_model():
    t = wl.Trace5(layers=1, steps=100, batch=256)
    Bs, B, MB = t.block_size, t.batch, t.max_blocks_per_seq
    bm = pa.BlockManager(t.num_blocks, Bs, B, MB, t.free_order)
    m = oracle.BlockManagerModel(t.num_blocks, Bs, B, MB, t.free_order)
    for s in range(B):
        bm.add_seq(s, int(t.initial_lens[s]))
        m.add_seq(s, int(t.initial_lens[s]))
    seqs = list(range(B))
    for step, retired, admitted in t.events():
        for s in retired:
            bm.free_seq(s)
            m.free_seq(s)
        for s, n in admitted:
            bm.add_seq(s, n)
            m.add_seq(s, n)
        assert list(bm.append_tokens(seqs)) == m.append_tokens(seqs)
    _same(bm, m)
    bm.close()
