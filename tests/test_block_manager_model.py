"""Pins for the block-manager reference model (oracle side, CPU only).

The model's policy is a stated reading (the pages give none); these tests pin
the properties the pages do fix: blocks are handed out only as tokens arrive,
freed blocks become reusable by any request, a shared block stays alive while
any table holds it, and logical positions map to (block, offset) slots.
"""
import numpy as np
import pytest

from oracle import BlockManagerModel, OutOfBlocks, SharedBlockWrite


def _invariants(m: BlockManagerModel):
    held = {}
    for s in range(m.max_seqs):
        if not m.live[s]:
            assert m.tables[s] == []
            continue
        assert len(m.tables[s]) == -(-m.lens[s] // m.block_size)   # exactly the blocks needed
        for blk in m.tables[s]:
            held[blk] = held.get(blk, 0) + 1
    for blk in range(m.num_blocks):
        assert m.ref[blk] == held.get(blk, 0)
    assert set(m.free).isdisjoint(held)
    assert len(m.free) + len(held) == m.num_blocks
    assert len(set(m.free)) == len(m.free)


def test_blocks_arrive_with_tokens_and_order_is_the_free_order():
    m = BlockManagerModel(6, 4, 2, 4, free_order=[5, 1, 3, 0, 2, 4])
    m.add_seq(0, 0)
    assert m.tables[0] == []
    slots = m.append_tokens([0])          # position 0 needs a block: 5 comes first
    assert m.tables[0] == [5] and slots == [20]
    for p in range(1, 4):
        assert m.append_tokens([0]) == [20 + p]
    assert m.num_free() == 5               # no new block until the first one is full
    assert m.append_tokens([0]) == [4]     # position 4 -> second block, which is 1
    _invariants(m)


def test_freed_blocks_are_reused_by_other_sequences():
    m = BlockManagerModel(4, 2, 3, 4, free_order=[0, 1, 2, 3])
    m.add_seq(0, 3)                        # blocks 0, 1
    m.add_seq(1, 4)                        # blocks 2, 3
    with pytest.raises(OutOfBlocks):
        m.add_seq(2, 1)
    m.free_seq(0)
    m.add_seq(2, 4)
    assert sorted(m.tables[2]) == [0, 1]
    _invariants(m)


def test_batch_append_is_all_or_nothing():
    m = BlockManagerModel(3, 2, 2, 4, free_order=[0, 1, 2])
    m.add_seq(0, 2)
    m.add_seq(1, 2)                        # one block left
    before = (list(m.free), [list(t) for t in m.tables], list(m.lens))
    with pytest.raises(OutOfBlocks):
        m.append_tokens([0, 1])            # both need a block
    assert (list(m.free), [list(t) for t in m.tables], list(m.lens)) == before


def test_shared_block_stays_alive_and_refuses_writes():
    m = BlockManagerModel(8, 4, 3, 4, free_order=list(range(8)))
    m.add_seq(0, 6)                        # blocks 0 (full) and 1 (half)
    m.import_seq(1, 6, m.tables[0])        # shares both blocks
    assert m.ref[0] == 2 and m.ref[1] == 2
    with pytest.raises(SharedBlockWrite):
        m.append_tokens([1])               # position 6 lands in shared block 1
    m.free_seq(0)
    assert m.ref[0] == 1 and 0 not in m.free
    m.append_tokens([1])                   # now exclusive: allowed
    _invariants(m)


def test_random_trace_keeps_invariants():
    rng = np.random.default_rng(0)
    N, Bs, S = 64, 4, 6
    m = BlockManagerModel(N, Bs, S, 64, free_order=rng.permutation(N))
    for step in range(400):
        live = [s for s in range(S) if m.live[s]]
        dead = [s for s in range(S) if not m.live[s]]
        r = rng.random()
        try:
            if dead and r < 0.2:
                m.add_seq(int(rng.choice(dead)), int(rng.integers(0, 20)))
            elif live and r < 0.3:
                m.free_seq(int(rng.choice(live)))
            elif live:
                pick = [s for s in live if rng.random() < 0.7]
                lens = [m.lens[s] for s in pick]
                slots = m.append_tokens(pick)
                for s, p, slot in zip(pick, lens, slots):
                    assert slot // Bs == m.tables[s][p // Bs] and slot % Bs == p % Bs
        except OutOfBlocks:
            pass
        _invariants(m)
