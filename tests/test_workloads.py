"""The seeded generators produce the configured shapes, distributions and layouts."""
import math

import numpy as np

import workloads as wl


def test_streams_are_deterministic_and_counter_based():
    a = wl.normal_bf16(123, (1000,))
    b = wl.normal_bf16(123, (1000,))
    np.testing.assert_array_equal(a, b)
    tail = wl.normal_bf16(123, (500,), offset=500)
    np.testing.assert_array_equal(a[500:], tail)
    assert not np.array_equal(a, wl.normal_bf16(124, (1000,)))


def test_normals_are_standard_and_rounded_to_nearest_even():
    x = wl.normal(7, 200000)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    bits = wl.normal_bf16(7, (200000,))
    f32 = x.astype(np.float32).view(np.uint32).astype(np.uint64)
    rne = ((f32 + 0x7FFF + ((f32 >> 16) & 1)) >> 16).astype(np.uint16)
    np.testing.assert_array_equal(bits, rne)


def test_config1_shape():
    b = wl.config1()
    assert list(b.context_lens) == [5, 37]
    assert b.num_blocks == 8 and b.num_q_heads == 2 and b.num_kv_heads == 1
    assert b.head_dim == 64 and b.block_size == 16 and b.scale == 1.0 / 8.0
    used = [int(x) for x in b.block_tables.ravel() if x >= 0]
    assert len(used) == 1 + 3
    assert sorted(used + list(b.free_order)) == list(range(8))


def test_config2_shape_and_pool():
    b = wl.config2(with_pool=False)
    L = b.context_lens
    assert L.shape == (64,) and L.min() >= 128 and L.max() <= 2048
    needed = int(np.sum(-(-(L.astype(np.int64) + 1) // 16)))
    assert b.num_blocks == math.ceil(1.1 * needed)
    used = b.block_tables[b.block_tables >= 0]
    assert len(np.unique(used)) == len(used)           # private blocks only
    assert set(used.tolist()).isdisjoint(b.free_order.tolist())


def test_config3_shares_prefix_blocks():
    b = wl.config3(with_pool=False)
    assert b.block_size == 256 and b.shared_prefix_blocks == 4
    assert (b.block_tables[:, :4] == b.block_tables[0, :4]).all()
    suffix = b.context_lens - 1024
    assert suffix.min() >= 256 and suffix.max() <= 7168
    rest = np.concatenate([r[4:][r[4:] >= 0] for r in b.block_tables])
    assert len(np.unique(rest)) == len(rest)
    assert set(rest.tolist()).isdisjoint(b.block_tables[0, :4].tolist())


def test_config4_lengths():
    b = wl.config4(with_pool=False)
    assert list(b.context_lens) == [32768, 65536, 98304, 131072]
    assert b.head_dim == 128 and b.num_q_heads == 64 and b.num_kv_heads == 8


def test_trace5_distribution():
    t = wl.Trace5()
    assert t.initial_lens.shape == (256,)
    assert t.initial_lens.min() >= 1 and t.initial_lens.max() <= 16384
    assert 350 < np.median(t.initial_lens) < 750          # median 512
    assert not t.finish[0].any()
    rate = t.finish[1:].mean()
    assert 0.005 < rate < 0.02                             # p = 0.01 per step
    n = sum(len(r) for _, r, _ in t.events())
    assert n == len(t.new_lens)
