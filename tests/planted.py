"""Planted-key decode inputs: long contexts whose answer moves by O(1) when any piece of the
work is lost.

With N(0,1) keys a decode over tens of thousands of tokens averages so many V rows that
dropping a sixteenth of them moves the output by less than the parity tolerance.  Here each
query head's attention is pinned to a few planted keys instead:

* query head h = kvh * G + g is ALPHA along one head dimension d(g) and zero elsewhere;
* every K row of the pool (and every new K row) is zero along the G planted dimensions, so an
  ordinary key scores exactly 0 for every query head;
* a planted key of head h carries BETA along d(g): it scores ALPHA * BETA * scale (> 22 in
  natural-log units at D = 128), so the ordinary keys' total weight stays below 1e-4 even over
  131072 tokens, and the exact output is the mean of the head's planted V rows;
* planted V rows are V_GAIN times their N(0,1) values (exact: a power of two), so losing one
  of a head's k planted keys moves its output by about V_GAIN / k, far outside the tolerance.

The planted positions are chosen from the decode kernel's own partition of the work: the
first, middle and last 16-token slab of every CTA slice of the stream-partitioned kernel, and
both sides of every split edge for the split kernels.  Every piece a cut sequence leaves for the
merge holds the first or the last slab of its slice, so every piece (and every piece group of
the merge) carries planted keys.  The stream partition below restates the kernel's slicing
rule: the work is the concatenation, over groups of 8 kv heads and sequences, of 16-token slabs
(an empty sequence counts one), cut into `grid` equal slices [i S / grid, (i + 1) S / grid).

This module builds inputs only; the expected values always come from the oracle.
"""
from __future__ import annotations

import dataclasses

import numpy as np

SLAB = 16
ALPHA = 16.0
BETA = 16.0
V_GAIN = 8.0


def _f32_to_bf16_exact(x: float) -> int:
    """bf16 pattern of a float that bf16 holds exactly (the planted constants)."""
    bits = int(np.array([x], dtype=np.float32).view(np.uint32)[0])
    assert bits & 0xFFFF == 0, "not exact in bf16"
    return bits >> 16


def planted_dims(group: int, head_dim: int) -> list:
    """Head dimension d(g) of query head g of a group: spread evenly over the head."""
    step = head_dim // group
    return [g * step for g in range(group)]


def stream_partition(lens, num_kv_heads: int, grid: int, slab: int = SLAB):
    """The stream kernel's slices (slabs of `slab` tokens).  Returns (slices, locate) where
    slices = [(lo, hi)] in slab indices and locate(s) = (kv group, sequence, slab of the
    sequence)."""
    lens = np.asarray(lens, dtype=np.int64)
    n = np.where(lens == 0, 1, -(-lens // slab))
    s_seq = int(n.sum())
    groups = num_kv_heads // 8
    S = s_seq * groups
    gc = min(S, grid)
    starts = np.concatenate([[0], np.cumsum(n)])
    slices = [(i * S // gc, (i + 1) * S // gc) for i in range(gc)]

    def locate(s):
        gi, r = divmod(int(s), s_seq)
        b = int(np.searchsorted(starts, r, side="right") - 1)
        return gi, b, r - int(starts[b])

    return slices, locate


def stream_pieces(lens, num_kv_heads: int, grid: int, slab: int = SLAB):
    """Per (kv group, sequence): the list of its pieces as (first slab, end slab) of the
    sequence, one per slice it meets, in order (one piece = the sequence was not cut)."""
    slices, locate = stream_partition(lens, num_kv_heads, grid, slab)
    pieces = {}
    for lo, hi in slices:
        s = lo
        while s < hi:
            gi, b, j = locate(s)
            n_b = max(1, -(-int(lens[b]) // slab))
            end = min(n_b, j + (hi - s))
            pieces.setdefault((gi, b), []).append((j, end))
            s += end - j
    return pieces


def stream_positions(lens, num_kv_heads: int, grid: int, slab: int = SLAB):
    """(kv group, sequence, token position) of the first token of each slice's first slab,
    the last valid token of its last slab and a middle token of its middle slab."""
    lens = np.asarray(lens, dtype=np.int64)
    slices, locate = stream_partition(lens, num_kv_heads, grid, slab)
    out = []
    for lo, hi in slices:
        for s, where in ((lo, "first"), ((lo + hi - 1) // 2, "mid"), (hi - 1, "last")):
            gi, b, j = locate(s)
            L = int(lens[b])
            if L == 0:
                continue
            t0, t1 = j * slab, min(L, (j + 1) * slab)
            p = t0 if where == "first" else (t1 - 1 if where == "last" else (t0 + t1 - 1) // 2)
            out.append((gi, b, p))
    return out


def split_positions(lens, num_kv_heads: int, split_tokens: int):
    """Both sides of every split edge k * split_tokens of every sequence (all kv groups)."""
    out = []
    for b, L in enumerate(np.asarray(lens, dtype=np.int64)):
        for e in range(split_tokens, int(L), split_tokens):
            for gi in range(max(1, num_kv_heads // 8)):
                out += [(gi, b, e - 1), (gi, b, e)]
    return out


def assign(positions, batch_size: int, num_q_heads: int, num_kv_heads: int, lens, seed: int = 7):
    """Spread the chosen positions over query heads: a position of kv group gi is planted for
    each of the group's kv heads (up to 8), rotating over the G query heads of each; every
    query head of a non-empty sequence gets at least one planted key.
    Returns {(b, h): sorted positions}."""
    G = num_q_heads // num_kv_heads
    per_group = min(8, num_kv_heads)
    plants = {}
    turn = np.zeros((batch_size, num_kv_heads), dtype=np.int64)
    for gi, b, p in positions:
        for kvh in range(gi * per_group, min(num_kv_heads, (gi + 1) * per_group)):
            g = int(turn[b, kvh] % G)
            turn[b, kvh] += 1
            plants.setdefault((b, kvh * G + g), set()).add(int(p))
    rng = np.random.default_rng(seed)
    for b in range(batch_size):
        L = int(lens[b])
        if L == 0:
            continue
        for h in range(num_q_heads):
            if not plants.get((b, h)):
                plants[(b, h)] = {int(rng.integers(0, L))}
    return {k: sorted(v) for k, v in plants.items()}


def plant(batch, tables, lens, plants, copy: bool = True):
    """`batch` (workloads.DecodeBatch, cached state before the append) with the planted q, K
    and V: a copy, or the batch's own arrays changed in place (copy=False).  tables / lens: the
    rows after this step's append (lens count the new token, which sits at position L - 1 and
    comes from k_new / v_new)."""
    Hq, Hkv, D, Bs = batch.num_q_heads, batch.num_kv_heads, batch.head_dim, batch.block_size
    G = Hq // Hkv
    dims = planted_dims(G, D)
    alpha, beta = _f32_to_bf16_exact(ALPHA), _f32_to_bf16_exact(BETA)
    q = np.zeros_like(batch.q)
    for h in range(Hq):
        q[:, h, dims[h % G]] = alpha
    cp = (lambda a: a.copy()) if copy else (lambda a: a)
    k_cache, v_cache = cp(batch.k_cache), cp(batch.v_cache)
    k_new, v_new = cp(batch.k_new), cp(batch.v_new)
    step = D // G                      # dims[g] = g * step: one strided pass clears them all
    k_cache[..., :G * step:step] = 0
    k_new[..., :G * step:step] = 0
    gained = set()

    def gain(row):
        x = (row.astype(np.uint32) << 16).view(np.float32) * np.float32(V_GAIN)
        return (x.view(np.uint32) >> 16).astype(np.uint16)

    for (b, h), ps in plants.items():
        kvh, g = h // G, h % G
        L = int(lens[b])
        for p in ps:
            assert 0 <= p < L
            if p == L - 1:
                k_new[b, kvh, dims[g]] = beta
                where = ("new", b, kvh)
                if where not in gained:
                    v_new[b, kvh] = gain(v_new[b, kvh])
            else:
                blk, off = int(tables[b, p // Bs]), p % Bs
                k_cache[blk, kvh, off, dims[g]] = beta
                where = ("pool", blk, kvh, off)
                if where not in gained:
                    v_cache[blk, kvh, off] = gain(v_cache[blk, kvh, off])
            gained.add(where)
    return dataclasses.replace(batch, q=q, k_cache=k_cache, v_cache=v_cache, k_new=k_new,
                               v_new=v_new, name=batch.name + "-planted")


def tripwire(gpu: np.ndarray, ref: np.ndarray):
    """A bound well inside the parity tolerance: |gpu - ref| <= 2^-7 |ref| + 2e-4 (bf16 output
    rounding is 2^-9 relative).  Returns (ok, worst ratio of error to bound)."""
    err = np.abs(np.asarray(gpu, dtype=np.float64) - ref)
    bound = 2.0 ** -7 * np.abs(ref) + 2e-4
    return bool(np.all(err <= bound)), float(np.max(err / bound)) if err.size else 0.0
