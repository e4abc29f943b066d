"""The planted-key inputs have teeth, shown on the CPU with the oracle alone.

A decode that loses one 16-token slab, or one of the merge's piece groups, of a long
context stays inside the parity tolerance on N(0,1) inputs.  On the planted inputs
(tests/planted.py) it must not: here the oracle runs over the same context with that slab, or
every piece of that group, cut out of the table row, and the result must leave the tolerance
against the oracle over the whole context.  The partition is the one the stream kernel takes
on a B200 for these shapes (148 SMs: one CTA per SM at D = 128, two at D = 64).

The planted construction is pinned too: each head's exact output is the mean of its planted
V rows (the ordinary keys' weight is below 1e-4 in total).
"""
import numpy as np
import pytest

import oracle
import workloads as wl
from tests import planted as pl

B200_SMS = 148


def _after_append(b):
    """Tables, lengths and slots after this step's append, from the block manager model."""
    B, Bs, MB = b.batch, b.block_size, b.max_blocks_per_seq
    m = oracle.BlockManagerModel(b.num_blocks, Bs, B, MB, b.free_order)
    for s in range(B):
        L = int(b.context_lens[s])
        m.import_seq(s, L, b.block_tables[s, : -(-L // Bs)])
    slots = np.array(m.append_tokens(list(range(B))), dtype=np.int64)
    tables = np.array([m.table_array(s) for s in range(B)], dtype=np.int32)
    return tables, np.array(m.lens, dtype=np.int32), slots


@pytest.fixture(scope="module")
def c4():
    b = wl.config4()
    tables, lens, slots = _after_append(b)
    plants = pl.assign(pl.stream_positions(lens, b.num_kv_heads, B200_SMS), b.batch, b.num_q_heads,
                       b.num_kv_heads, lens)
    pb = pl.plant(b, tables, lens, plants, copy=False)
    kc, vc = oracle.append_kv(pb.k_new, pb.v_new, slots, pb.k_cache, pb.v_cache, in_place=True)
    return dict(b=pb, tables=tables, lens=lens, plants=plants, kc=kc, vc=vc)


def _decode_rows(d, seq, table_row, L):
    b = d["b"]
    return oracle.paged_decode(b.q[seq:seq + 1], d["kc"], d["vc"], table_row[None, :],
                               np.array([L], np.int32), b.scale)[0]


def _without_slabs(d, seq, slabs):
    """Table row and length of sequence `seq` with the listed 16-token slabs (= blocks at
    Bs = 16) cut out, as a decode that skipped them would see it."""
    Bs = d["b"].block_size
    assert Bs == pl.SLAB
    L = int(d["lens"][seq])
    nb = -(-L // Bs)
    keep = [j for j in range(nb) if j not in set(slabs)]
    assert nb - 1 in keep   # the partial last block stays last
    row = np.full(d["tables"].shape[1], -1, np.int32)
    row[:len(keep)] = d["tables"][seq, keep]
    return row, L - Bs * (nb - len(keep))


def test_planted_output_is_the_mean_of_the_planted_values(c4):
    d, b = c4, c4["b"]
    seq = 0
    out = _decode_rows(d, seq, d["tables"][seq], int(d["lens"][seq]))
    G, Bs = b.num_q_heads // b.num_kv_heads, b.block_size
    for h in range(b.num_q_heads):
        rows = []
        for p in d["plants"][(seq, h)]:
            blk = d["tables"][seq, p // Bs]
            rows.append((d["vc"][blk, h // G, p % Bs].astype(np.uint32) << 16).view(np.float32))
        want = np.mean(np.array(rows, dtype=np.float64), axis=0)
        np.testing.assert_allclose(out[h], want, rtol=0, atol=1e-3)


@pytest.mark.parametrize("which", ["first", "last", "mid"])
def test_dropping_one_slab_leaves_the_tolerance(c4, which):
    d = c4
    seq = 0
    L = int(d["lens"][seq])
    full = _decode_rows(d, seq, d["tables"][seq], L)
    # a slice boundary inside sequence 0: the slab on either side of it, or a middle one
    pieces = pl.stream_pieces(d["lens"], d["b"].num_kv_heads, B200_SMS)[(0, seq)]
    assert len(pieces) > 4
    j0, j1 = pieces[2]
    slab = {"first": j0, "last": j1 - 1, "mid": (j0 + j1 - 1) // 2}[which]
    row, L2 = _without_slabs(d, seq, [slab])
    ok, excess = oracle.within_tolerance(_decode_rows(d, seq, row, L2), full)
    assert not ok, "a dropped %s slab stays within tolerance" % which
    assert excess > 0.1


# The merge kernel folds piece k of a sequence into piece group k % PG: for C4 (contexts of 8K
# tokens and more, 256 CTAs of one query head each) PG = 16.
C4_MERGE_GROUPS = 16


@pytest.mark.parametrize("group", [0, 9, 15])
def test_dropping_one_merge_piece_group_leaves_the_tolerance(c4, group):
    d = c4
    seq = 3            # the longest context: cut into about 60 pieces
    L = int(d["lens"][seq])
    pieces = pl.stream_pieces(d["lens"], d["b"].num_kv_heads, B200_SMS)[(0, seq)]
    assert len(pieces) >= 32
    slabs = [j for k, (j0, j1) in enumerate(pieces) if k % C4_MERGE_GROUPS == group
             for j in range(j0, j1)]
    nb = -(-L // pl.SLAB)
    slabs = [j for j in slabs if j != nb - 1]
    full = _decode_rows(d, seq, d["tables"][seq], L)
    row, L2 = _without_slabs(d, seq, slabs)
    ok, excess = oracle.within_tolerance(_decode_rows(d, seq, row, L2), full)
    assert not ok, "a dropped piece group stays within tolerance"
    assert excess > 0.1


def test_every_piece_carries_a_planted_key(c4):
    # every piece a cut sequence leaves holds the first or the last slab of its slice, and a
    # planted key for at least one query head of each kv head
    d, b = c4, c4["b"]
    G = b.num_q_heads // b.num_kv_heads
    for (gi, seq), pieces in pl.stream_pieces(d["lens"], b.num_kv_heads, B200_SMS).items():
        for j0, j1 in pieces:
            for kvh in range(b.num_kv_heads):
                ps = [p for g in range(G) for p in d["plants"].get((seq, kvh * G + g), [])]
                assert any(j0 * pl.SLAB <= p < j1 * pl.SLAB for p in ps), (seq, j0, j1, kvh)


def test_c5_batch_slab_drop_leaves_the_tolerance():
    # the C5 shapes (D = 64, two CTAs per SM): a cut sequence loses one slab at a slice edge
    t = wl.Trace5()
    b = wl.make_batch("C5-batch", t.seed, t.initial_lens, num_q_heads=t.num_q_heads,
                      num_kv_heads=t.num_kv_heads, head_dim=t.head_dim, block_size=t.block_size)
    tables, lens, slots = _after_append(b)
    plants = pl.assign(pl.stream_positions(lens, b.num_kv_heads, 2 * B200_SMS), b.batch,
                       b.num_q_heads, b.num_kv_heads, lens)
    pb = pl.plant(b, tables, lens, plants, copy=False)
    kc, vc = oracle.append_kv(pb.k_new, pb.v_new, slots, pb.k_cache, pb.v_cache, in_place=True)
    d = dict(b=pb, tables=tables, lens=lens, kc=kc, vc=vc)
    pieces = pl.stream_pieces(lens, b.num_kv_heads, 2 * B200_SMS)
    seq, ps = max(pieces.items(), key=lambda kv: len(kv[1]))
    seq = seq[1]
    assert len(ps) >= 3
    L = int(lens[seq])
    full = _decode_rows(d, seq, tables[seq], L)
    for slab in (ps[1][0], ps[1][1] - 1):
        row, L2 = _without_slabs(d, seq, [slab])
        ok, _ = oracle.within_tolerance(_decode_rows(d, seq, row, L2), full)
        assert not ok


@pytest.mark.parametrize("slab", [16, 32])
def test_stream_partition_mirror_tiles_every_sequence(slab):
    """The host mirror of the stream partition (16-token slabs, 32 for E4M3 pools at D=64):
    every (kv group, sequence) is covered by its pieces exactly once and in order, and the
    slices cut the concatenated slabs into runs that differ by at most one slab."""
    rng = np.random.default_rng(11 + slab)
    for trial in range(20):
        B = int(rng.integers(1, 40))
        lens = rng.integers(0, 3000, size=B)
        Hkv = int(rng.choice([8, 16]))
        grid = int(rng.integers(1, 400))
        slices, _ = pl.stream_partition(lens, Hkv, grid, slab)
        sizes = [hi - lo for lo, hi in slices]
        assert max(sizes) - min(sizes) <= 1
        assert slices[0][0] == 0 and all(a[1] == b[0] for a, b in zip(slices, slices[1:]))
        pieces = pl.stream_pieces(lens, Hkv, grid, slab)
        assert len(pieces) == B * (Hkv // 8)
        for (gi, b), ps in pieces.items():
            nb = max(1, -(-int(lens[b]) // slab))
            assert ps[0][0] == 0 and ps[-1][1] == nb
            assert all(p[1] == q[0] for p, q in zip(ps, ps[1:]))
