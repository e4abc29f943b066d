"""Per-block pool (pa_pool_*): pinned model, then the C++ pool matched to it bit for bit.

Pins of the model (oracle.BlockPoolModel), from what the pages fix: blocks are handed out only
on request and serve any request once free again; a shared block stays allocated while any
holder keeps it.  The policy details (stack order, all-or-nothing) are checked on a small
hand-worked sequence.
"""
import numpy as np
import pytest

import oracle
import pagedattention_kv_cache_pa_b200 as pa


def test_model_hand_worked_sequence():
    m = oracle.BlockPoolModel(5, free_order=[3, 1, 4])      # blocks 0 and 2 start allocated
    assert m.num_free() == 3 and m.refcount == [1, 0, 1, 0, 0]
    assert m.alloc(2) == [3, 1]                              # top of the stack first
    m.share(3)                                               # 3 now in two tables
    m.free(3)
    assert m.refcount[3] == 1 and m.num_free() == 1          # still held once
    m.free(1)
    assert m.alloc(1) == [1]                                 # the last freed block comes back first
    with pytest.raises(oracle.OutOfBlocks):
        m.alloc(3)                                           # only 4 is free: nothing changes
    assert m.num_free() == 1 and m.stack == [4]
    with pytest.raises(ValueError):
        m.free(4)                                            # free block
    with pytest.raises(ValueError):
        m.share(4)


def test_model_invariants_on_random_operations():
    rng = np.random.default_rng(11)
    N = 64
    m = oracle.BlockPoolModel(N, free_order=rng.permutation(N))
    holders = {}
    for _ in range(5000):
        op = rng.integers(0, 3)
        if op == 0:
            n = int(rng.integers(0, 5))
            if n <= m.num_free():
                for b in m.alloc(n):
                    holders[b] = 1
        elif op == 1 and holders:
            b = int(rng.choice(list(holders)))
            m.share(b)
            holders[b] += 1
        elif holders:
            b = int(rng.choice(list(holders)))
            m.free(b)
            holders[b] -= 1
            if holders[b] == 0:
                del holders[b]
        # every block is either free (count 0, on the stack once) or held by its holders
        assert sorted(m.stack) == sorted(set(range(N)) - set(holders))
        assert all(m.refcount[b] == holders.get(b, 0) for b in range(N))


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_cpp_pool_matches_the_model(seed):
    rng = np.random.default_rng(seed)
    N = int(rng.integers(8, 200))
    order = rng.permutation(N)[: int(rng.integers(1, N + 1))]
    m = oracle.BlockPoolModel(N, free_order=order)
    p = pa.BlockPool(N, free_order=order.astype(np.int32))
    for _ in range(4000):
        op = rng.integers(0, 4)
        b = int(rng.integers(-2, N + 2))
        if op == 0:
            n = int(rng.integers(0, 6))
            try:
                want = m.alloc(n)
            except oracle.OutOfBlocks:
                want = None
            if want is None:
                with pytest.raises(pa.PaError) as e:
                    p.alloc(n)
                assert e.value.status == -5
            else:
                assert list(p.alloc(n)) == want
        elif op in (1, 2):
            f_model, f_pool = (m.share, p.share) if op == 1 else (m.free, p.free)
            try:
                f_model(b)
                ok = True
            except ValueError:
                ok = False
            if ok:
                f_pool(b)
            else:
                with pytest.raises(pa.PaError) as e:
                    f_pool(b)
                assert e.value.status == -1
        assert p.num_free() == m.num_free()
        assert p.refcount(b) == (m.refcount[b] if 0 <= b < N else -1)
    assert [p.refcount(i) for i in range(N)] == m.refcount
    p.close()


def test_pool_create_rejects_bad_free_orders():
    for n, order in ((4, [0, 0]), (4, [4]), (4, [-1]), (0, [])):
        with pytest.raises(pa.PaError):
            pa.BlockPool(n, free_order=np.array(order, dtype=np.int32))
