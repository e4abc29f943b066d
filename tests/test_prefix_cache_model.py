"""Pins of the block-manager model's prefix caching and copy-on-write (CPU).

The model is the reference the C++ manager is compared with, so it is pinned
here by what its definition fixes: FNV-1a's published test vectors, hand-worked
admission and eviction scenarios, and invariants over random traces.
"""
import random

import pytest

from oracle.block_manager import BlockManagerModel, OutOfBlocks, block_hash, fnv1a64

Bs = 4


def _model(n=16, seqs=8, mb=16):
    return BlockManagerModel(n, Bs, seqs, mb, list(range(n)))


def test_fnv1a64_published_vectors():
    assert fnv1a64(b"") == 0xCBF29CE484222325
    assert fnv1a64(b"a") == 0xAF63DC4C8601EC8C
    assert fnv1a64(b"foobar") == 0x85944171F73967E8


def test_block_hash_layout():
    # parent as 8 little-endian bytes, then each id as 4 little-endian bytes (two's complement)
    want = fnv1a64(bytes([7, 0, 0, 0, 0, 0, 0, 0, 1, 0, 0, 0, 0xFF, 0xFF, 0xFF, 0xFF]))
    assert block_hash(7, [1, -1]) == want


def test_shared_prompt_reuses_full_blocks():
    m = _model()
    prompt = list(range(100, 114))                      # 3 full blocks + 2 tokens
    assert m.add_seq_tokens(0, prompt) == 0
    assert m.num_cached() == 3
    assert m.add_seq_tokens(1, prompt) == 3 * Bs
    assert m.tables[1][:3] == m.tables[0][:3]
    assert m.tables[1][3] != m.tables[0][3]             # the partial block is private
    assert [m.ref[b] for b in m.tables[0][:3]] == [2, 2, 2]
    assert m.num_free() == 16 - 5


def test_divergence_stops_the_hit_walk():
    m = _model()
    a = list(range(12))
    b = a[:8] + [99, 99, 99, 99]                        # differs in block 2
    m.add_seq_tokens(0, a)
    assert m.add_seq_tokens(1, b) == 2 * Bs
    c = [5] + a[1:]                                     # differs in block 0: nothing cached
    assert m.add_seq_tokens(2, c) == 0


def test_only_full_blocks_hit():
    m = _model()
    m.add_seq_tokens(0, list(range(12)))
    assert m.add_seq_tokens(1, list(range(7))) == 1 * Bs   # 1 full block + 3 tokens


def test_released_cached_blocks_stay_reusable_then_evict_oldest_first():
    m = _model(n=6)
    m.add_seq_tokens(0, list(range(8)))                 # 2 cached blocks: b0 (root), b1
    root, tail = m.tables[0]
    m.free_seq(0)
    assert m.num_cached() == 2 and m.num_free() == 6
    # cached blocks sit at the bottom, the root deepest: the 4 uncached go first, then tail
    assert m.free[:2] == [root, tail]
    assert m.add_seq_tokens(1, list(range(8))) == 8      # hit on free cached blocks
    assert m.tables[1] == [root, tail] and m.num_free() == 4
    m.free_seq(1)
    m.add_seq(2, 4 * Bs + 1)                            # takes the 4 uncached + tail (evicted)
    assert m.num_cached() == 1 and m.bhash[root] is not None and m.bhash[tail] is None


def test_admission_is_all_or_nothing():
    m = _model(n=4)
    m.add_seq_tokens(0, list(range(8)))
    with pytest.raises(OutOfBlocks):
        m.add_seq_tokens(1, list(range(8)) + list(range(50, 62)))   # 2 hits + 3 new > 2 free
    assert m.ref[m.tables[0][0]] == 1 and not m.live[1] and m.num_free() == 2


def test_copy_on_write_after_fork():
    m = _model()
    m.add_seq_tokens(0, list(range(6)))                 # 1 full block + 2 tokens
    m.fork_all(1, 0)
    shared = m.tables[0][1]
    assert m.ref[shared] == 2
    slots, copies = m.append_token_ids([1], [77])
    new = m.tables[1][1]
    assert copies == [(shared, new)] and new != shared
    assert slots == [new * Bs + 2]
    assert m.ref[shared] == 1 and m.ref[new] == 1
    assert m.ids[new][:3] == [4, 5, 77] and m.ids[shared][:2] == [4, 5]
    slots, copies = m.append_token_ids([0], [66])       # no longer shared: in place
    assert copies == [] and slots == [shared * Bs + 2]


def test_blocks_filled_by_decode_register_and_hit():
    m = _model()
    m.add_seq_tokens(0, [1, 2, 3])
    m.append_token_ids([0], [4])                        # block 0 fills: registered
    m.append_token_ids([0], [5])
    assert m.num_cached() == 1
    assert m.add_seq_tokens(1, [1, 2, 3, 4, 5]) == Bs


def test_plain_appends_stop_hashing():
    m = _model()
    m.add_seq_tokens(0, [1, 2, 3])
    m.append_tokens([0])                                # a token without an id
    assert m.num_cached() == 0
    m.append_token_ids([0], [9, ])
    m.append_token_ids([0], [9])
    m.append_token_ids([0], [9])
    m.append_token_ids([0], [9])
    assert m.num_cached() == 0


def test_hash_collision_is_not_a_hit(monkeypatch):
    import oracle.block_manager as bmod
    monkeypatch.setattr(bmod, "block_hash", lambda parent, ids: 42)
    m = _model()
    m.add_seq_tokens(0, [1, 2, 3, 4])
    assert m.add_seq_tokens(1, [5, 6, 7, 8]) == 0       # same hash, other ids
    assert m.tables[1][0] != m.tables[0][0]


def _check_invariants(m):
    held = [0] * m.num_blocks
    for s in range(m.max_seqs):
        if m.live[s]:
            assert len(m.tables[s]) == -(-m.lens[s] // m.block_size)
            for b in m.tables[s]:
                held[b] += 1
    assert held == m.ref
    assert sorted(m.free) == [b for b in range(m.num_blocks) if m.ref[b] == 0]
    for h, b in m.cache.items():
        assert m.bhash[b] == h and None not in m.ids[b]


def test_random_traces_keep_invariants():
    rng = random.Random(5)
    for trial in range(40):
        m = BlockManagerModel(24, Bs, 6, 40, rng.sample(range(24), 24))
        vocab = [rng.randrange(3) for _ in range(64)]   # small alphabet: many shared prefixes
        for step in range(200):
            s = rng.randrange(6)
            op = rng.random()
            try:
                if not m.live[s]:
                    if op < 0.6:
                        m.add_seq_tokens(s, vocab[:rng.randrange(0, 30)])
                    elif op < 0.8:
                        src = [x for x in range(6) if m.live[x] and x != s]
                        if src:
                            m.fork_all(s, rng.choice(src))
                    else:
                        m.add_seq(s, rng.randrange(0, 20))
                elif op < 0.15:
                    m.free_seq(s)
                else:
                    live = [x for x in range(6) if m.live[x] and m.lens[x] < 40 * Bs - 1]
                    if live:
                        m.append_token_ids(live, [rng.randrange(3) for _ in live])
            except OutOfBlocks:
                pass
            _check_invariants(m)
