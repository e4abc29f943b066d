"""Pins of the oracle's FP8 (E4M3) KV cache against the format's definition.

The Tiny-vLLM summary page (section "향후 전망") names FP8 as a data type to add,
with no format or scale scheme.  The reading pinned here is the OCP E4M3
format (1 sign, 4 exponent bits of bias 7, 3 mantissa bits, no infinities,
S.1111.111 = NaN, largest finite 448, subnormals m * 2^-9) with one scale per
cache tensor: code = e4m3(float(x) * float(1/scale)), nearest with ties to
even, saturating at +-448; value = value(code) * scale.
"""
import numpy as np
import pytest

import oracle
import workloads as wl


def _value_by_hand(c: int) -> float:
    s, e, m = c >> 7, (c >> 3) & 15, c & 7
    if e == 15 and m == 7:
        return float("nan")
    v = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
    return -v if s else v


def test_every_code_decodes_per_the_format():
    got = oracle.e4m3_to_double(np.arange(256, dtype=np.uint8))
    want = np.array([_value_by_hand(c) for c in range(256)])
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    keep = ~np.isnan(want)
    np.testing.assert_array_equal(got[keep], want[keep])
    hand = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x3F: 1.875,
            0x40: 2.0, 0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0}
    for c, v in hand.items():
        assert got[c] == v, hex(c)
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF])
    assert np.all(np.diff(got[:0x7F]) > 0)               # positive codes are ordered


def test_round_trip_of_every_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = oracle.e4m3_to_double(codes).astype(np.float32)
    vals[codes == 0x80] = np.float32(-0.0)
    np.testing.assert_array_equal(oracle.e4m3_from_float(vals), codes)


def test_midpoints_round_to_even_and_neighbours_to_nearest():
    vals = oracle.e4m3_to_double(np.arange(0x7F, dtype=np.uint8))   # 0 .. 448, ascending
    lo, hi = vals[:-1], vals[1:]
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.all(mid.astype(np.float64) == (lo + hi) / 2)          # midpoints exact in float
    got = oracle.e4m3_from_float(mid)
    k = np.arange(0x7E)
    even = np.where(k % 2 == 0, k, k + 1)                            # the code with mantissa lsb 0
    np.testing.assert_array_equal(got, even.astype(np.uint8))
    up = np.nextafter(mid, np.float32(np.inf))
    down = np.nextafter(mid, np.float32(0))
    np.testing.assert_array_equal(oracle.e4m3_from_float(up), (k + 1).astype(np.uint8))
    np.testing.assert_array_equal(oracle.e4m3_from_float(down), k.astype(np.uint8))


def test_saturation_and_specials():
    got = oracle.e4m3_from_float(np.array([448.0, 449.0, 464.0, 470.0, 1e30, np.inf, -500.0, -np.inf,
                                           np.nan], dtype=np.float32))
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F]


def test_quantize_is_a_float_product_then_the_code():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal(4096).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    for scale in (1.0, 0.0173, 3.7, 2.0 ** -7):
        y = (x.astype(np.uint32) << 16).view(np.float32) * (np.float32(1) / np.float32(scale))
        np.testing.assert_array_equal(oracle.quantize_e4m3(x, scale), oracle.e4m3_from_float(y))


@pytest.mark.parametrize("ks,vs", [(1.0, 1.0), (2.0, 0.5), (0.25, 4.0)])
def test_e4m3_decode_equals_bf16_decode_on_the_same_values(ks, vs):
    # every E4M3 value, times a power of two, is a bf16 value: build the bf16 pools from the
    # dequantized codes and the two oracle decodes must agree exactly
    b = wl.small_batch(55, [1, 17, 40, 130], num_q_heads=8, num_kv_heads=2, head_dim=64, block_size=16)
    rng = np.random.default_rng(9)
    kq = rng.integers(0, 256, b.k_cache.shape).astype(np.uint8)
    vq = rng.integers(0, 256, b.v_cache.shape).astype(np.uint8)
    kq[(kq & 0x7F) == 0x7F] = 0x3C                       # no NaN codes in the pools
    vq[(vq & 0x7F) == 0x7F] = 0x3C
    to_bf16 = lambda a: (a.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    kb = to_bf16(oracle.e4m3_to_double(kq) * ks)
    vb = to_bf16(oracle.e4m3_to_double(vq) * vs)
    assert np.all(((oracle.e4m3_to_double(kq) * ks).astype(np.float32).view(np.uint32) & 0xFFFF) == 0)
    want = oracle.paged_decode(b.q, kb, vb, b.block_tables, b.context_lens, b.scale)
    got = oracle.paged_decode_e4m3(b.q, kq, vq, ks, vs, b.block_tables, b.context_lens, b.scale)
    np.testing.assert_array_equal(got, want)


def test_append_e4m3_writes_only_the_slots():
    b = wl.small_batch(56, [10, 33], num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16)
    kc = np.zeros(b.k_cache.shape, dtype=np.uint8)
    vc = np.zeros(b.v_cache.shape, dtype=np.uint8)
    kq = oracle.quantize_e4m3(b.k_new, 0.5)
    vq = oracle.quantize_e4m3(b.v_new, 0.25)
    slots = np.array([3, -1], dtype=np.int64)
    k2, v2 = oracle.append_kv_e4m3(kq, vq, slots, kc, vc)
    assert np.array_equal(k2[0, :, 3, :], kq[0]) and np.array_equal(v2[0, :, 3, :], vq[0])
    k2[0, :, 3, :] = 0
    v2[0, :, 3, :] = 0
    assert not k2.any() and not v2.any()
