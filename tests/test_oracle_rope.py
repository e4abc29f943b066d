"""Pins of the oracle's RoPE and bf16 rounding against what mathematics fixes.

RoPE is named as a per-layer kernel of the Llama 3.2 1B model on the Tiny-vLLM
summary page (section "핵심 LLM 연산의 CUDA 커널 구현"), without a formula.  The
reading pinned here is RoFormer's rotation in the rotate-half pairing: for i < D/2,
the pair (x[i], x[i + D/2]) at position p turns by p * theta^(-2i/D).  The pins
are closed forms (unit vectors, a chosen frequency schedule), invariants of a
rotation (pair norms, relative position) and the identity at position 0.  bf16
rounding is pinned by the page's own bit layout (tests/golden/bf16_values.txt),
by exhaustive round trips and by hand-placed ties.
"""
import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(values):
    """bf16 bit patterns of values that are exactly representable (numpy, not the oracle)."""
    f = np.asarray(values, dtype=np.float32)
    bits = f.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0), "not a bf16 value"
    return (bits >> 16).astype(np.uint16)


def _widen(bits):
    with np.errstate(invalid="ignore"):   # NaN patterns stay NaN
        return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


# ---- bf16 rounding ----------------------------------------------------------------------

def test_round_bf16_golden_values():
    for line in open(os.path.join(GOLDEN, "bf16_values.txt")):
        if line.startswith("#") or not line.strip():
            continue
        bits, value = line.split()
        got = int(oracle.round_bf16(np.array([float(value)]))[0])
        assert got == int(bits, 16), (value, hex(got))


def test_round_bf16_round_trips_every_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = _widen(bits)
    keep = ~np.isnan(vals)
    got = oracle.round_bf16(vals[keep])
    np.testing.assert_array_equal(got, bits[keep])


def test_round_bf16_ties_and_edges():
    cases = [
        (1 + 2.0 ** -8, 0x3F80),               # halfway between 1 and 1 + 2^-7: even (1)
        (1 + 3 * 2.0 ** -8, 0x3F82),           # halfway above 1 + 2^-7: even (1 + 2^-6)
        (1 + 2.0 ** -8 + 2.0 ** -30, 0x3F81),  # just above half: up
        (1 + 2.0 ** -8 - 2.0 ** -30, 0x3F80),  # just below half: down
        (-(1 + 3 * 2.0 ** -8), 0xBF82),        # sign carried through
        (2.0 ** -134, 0x0000),                 # half the smallest subnormal: even (0)
        (3 * 2.0 ** -134, 0x0002),             # 1.5 x smallest subnormal: even (2)
        (2.0 ** -126 * (1 - 2.0 ** -9), 0x0080),  # rounds up into the normal range
        ((2 - 2.0 ** -7) * 2.0 ** 127, 0x7F7F),   # largest finite
        ((2 - 2.0 ** -8) * 2.0 ** 127, 0x7F80),   # tie at the top goes to even: infinity
        (255.5, 0x4380),                       # 255.5 lies between 255 and 256: tie to even 256
    ]
    got = oracle.round_bf16(np.array([c[0] for c in cases]))
    for (v, want), g in zip(cases, got):
        assert int(g) == want, (v, hex(int(g)), hex(want))


# ---- RoPE ---------------------------------------------------------------------------------

def _rand_bf16(rng, shape):
    """Random bf16 bit patterns (normal draws truncated to bf16)."""
    return (rng.standard_normal(shape).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_rope_position_zero_is_identity():
    x = _rand_bf16(np.random.default_rng(1), (5, 3, 64))
    out = oracle.rope(x, np.zeros(5, dtype=np.int32), 10000.0)
    np.testing.assert_array_equal(out, _widen(x))
    np.testing.assert_array_equal(oracle.rope_bf16(x, np.zeros(5, dtype=np.int32), 500000.0), x)


def test_rope_unit_vectors_closed_form():
    # D = 4, theta = 10^4: pairs (0, 2) turn by p, pairs (1, 3) by p * 10^4^(-1/2) = p / 100
    e = _bf16(np.eye(4, dtype=np.float32)).reshape(4, 1, 4)
    for p in (1, 3, 17, 1000, 123457):
        pos = np.full(4, p, dtype=np.int32)
        out = oracle.rope(e, pos, 10000.0)[:, 0, :]
        a, b = float(p), p / 100.0
        want = np.array([
            [math.cos(a), 0.0, math.sin(a), 0.0],     # e0 -> (cos a, 0, sin a, 0)
            [0.0, math.cos(b), 0.0, math.sin(b)],     # e1 -> (0, cos b, 0, sin b)
            [-math.sin(a), 0.0, math.cos(a), 0.0],    # e2 -> (-sin a, 0, cos a, 0)
            [0.0, -math.sin(b), 0.0, math.cos(b)],    # e3 -> (0, -sin b, 0, cos b)
        ])
        np.testing.assert_allclose(out, want, rtol=0, atol=1e-12)


def test_rope_frequency_schedule():
    # theta = 16, D = 8: pair i turns by p * 16^(-2i/8) = p * 2^-i; read the angle back
    x = np.zeros((1, 1, 8), dtype=np.float32)
    x[0, 0, :4] = 1.0
    xb = _bf16(x)
    p = 1
    out = oracle.rope(xb, np.array([p], dtype=np.int32), 16.0)[0, 0]
    for i in range(4):
        ang = math.atan2(out[i + 4], out[i])
        assert abs(ang - p * 2.0 ** -i) < 1e-12, (i, ang)


def test_rope_preserves_pair_norms():
    rng = np.random.default_rng(2)
    x = _rand_bf16(rng, (7, 4, 128))
    pos = rng.integers(0, 131072, 7).astype(np.int32)
    out = oracle.rope(x, pos, 500000.0)
    xi = _widen(x)
    n_in = xi[..., :64] ** 2 + xi[..., 64:] ** 2
    n_out = out[..., :64] ** 2 + out[..., 64:] ** 2
    np.testing.assert_allclose(n_out, n_in, rtol=1e-12, atol=1e-300)


def test_rope_scores_depend_on_relative_position_only():
    rng = np.random.default_rng(3)
    q = _rand_bf16(rng, (1, 1, 64))
    k = _rand_bf16(rng, (1, 1, 64))
    m, n = 900, 37

    def score(a, b):
        rq = oracle.rope(q, np.array([a], dtype=np.int32), 10000.0)[0, 0]
        rk = oracle.rope(k, np.array([b], dtype=np.int32), 10000.0)[0, 0]
        return float(rq @ rk)

    base = score(m, n)
    for s in (1, 10, 4096, 70000):
        assert abs(score(m + s, n + s) - base) <= 1e-9 * max(1.0, abs(base)), s
    assert abs(score(m + 1, n) - base) > 1e-6      # not shift-invariant in one argument


def test_rope_rows_are_independent():
    rng = np.random.default_rng(4)
    x = _rand_bf16(rng, (6, 5, 64))
    pos = rng.integers(0, 5000, 6).astype(np.int32)
    whole = oracle.rope(x, pos, 10000.0)
    for t in range(6):
        for h in range(5):
            one = oracle.rope(x[t:t + 1, h:h + 1], pos[t:t + 1], 10000.0)
            np.testing.assert_array_equal(one[0, 0], whole[t, h])
