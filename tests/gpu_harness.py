"""Shared plumbing of the GPU parity tests: one decode step through the C ABI
next to the same step through the oracle, on identical seeded inputs.

Step = (a1) the host block manager gives each sequence a block if its last one
is full, (a2) the newest token's slot, (a3) KV append, (a4-a10) paged decode.
The product side uses libpa (C++ block manager + CUDA kernels); the oracle side
uses oracle.BlockManagerModel + the C oracle.  Nothing flows from the product
side into the oracle side.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads as wl
import pagedattention_kv_cache_pa_b200 as pa

DEV = torch.device("cuda:0")


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(DEV)


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def desc_of(b: wl.DecodeBatch, max_blocks_per_seq=None) -> pa.CacheDesc:
    return pa.CacheDesc.make(num_blocks=b.num_blocks, block_size=b.block_size,
                             num_kv_heads=b.num_kv_heads, num_q_heads=b.num_q_heads,
                             head_dim=b.head_dim,
                             max_blocks_per_seq=max_blocks_per_seq or b.max_blocks_per_seq)


def host_step(b: wl.DecodeBatch):
    """(a1, a2) on both sides; returns product (slots, tables, lens) and oracle ones."""
    B, Bs, MB = b.batch, b.block_size, b.max_blocks_per_seq
    bm = pa.BlockManager(b.num_blocks, Bs, B, MB, b.free_order)
    model = oracle.BlockManagerModel(b.num_blocks, Bs, B, MB, b.free_order)
    for s in range(B):
        L = int(b.context_lens[s])
        blocks = b.block_tables[s, : -(-L // Bs)]
        bm.import_seq(s, L, blocks)
        model.import_seq(s, L, blocks)
    slots = bm.append_tokens(np.arange(B, dtype=np.int32))
    tables = bm.block_tables().copy()
    lens = bm.context_lens().copy()
    bm.close()
    o_slots = np.array(model.append_tokens(list(range(B))), dtype=np.int64)
    o_tables = np.array([model.table_array(s) for s in range(B)], dtype=np.int32)
    o_lens = np.array(model.lens, dtype=np.int32)
    return (slots, tables, lens), (o_slots, o_tables, o_lens)


def bf16_ulps(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in units in the last place between bf16 bit patterns (adjacent values: 1)."""
    def ordered(x):
        x = np.asarray(x, dtype=np.uint16).astype(np.int32)
        return np.where(x & 0x8000, -(x & 0x7FFF), x & 0x7FFF)
    return np.abs(ordered(a) - ordered(b))


def widen(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def rope_close(gpu_bits: np.ndarray, x_bits: np.ndarray, positions: np.ndarray, theta: float):
    """RoPE outputs [T, H, D] against the oracle's unrounded rotation of x_bits: each value
    within 2^-8 |exact| (its bf16 rounding) + 2^-20 (|x[i]| + |x[i + D/2]|) (float cos/sin and
    products on the pair's inputs; where the rotation cancels, the second term dominates).
    Returns (ok, worst error / bound)."""
    exact = oracle.rope(x_bits, positions, theta)
    x = widen(x_bits)
    half = x.shape[-1] // 2
    mag = np.abs(x[..., :half]) + np.abs(x[..., half:])
    mag = np.concatenate([mag, mag], axis=-1)
    bound = 2.0 ** -8 * np.abs(exact) + 2.0 ** -20 * mag + 1e-30
    ratio = np.abs(widen(gpu_bits) - exact) / bound
    return bool(np.all(ratio <= 1.0)), float(ratio.max())


def pool_rows(shape, slots) -> np.ndarray:
    """Mask of the pool rows ([N, Hkv, Bs, D] broadcast) that the given slots address."""
    N, Hkv, Bs, D = shape
    rows = np.zeros((N, Bs), dtype=bool)
    for sl in np.asarray(slots):
        if 0 <= sl < N * Bs:
            rows[sl // Bs, sl % Bs] = True
    return np.broadcast_to(rows[:, None, :, None], shape)


def rope_pool_matches(gpu: np.ndarray, initial: np.ndarray, k_new: np.ndarray, slots, positions,
                      theta: float) -> bool:
    """K pool after a RoPE append: bytes outside the slots' rows unchanged from `initial`, and
    each slot's rows the rotation of its token's K within rope_close's bound."""
    mask = pool_rows(initial.shape, slots)
    if not np.array_equal(gpu[~mask], initial[~mask]):
        return False
    Bs = initial.shape[2]
    for t, sl in enumerate(np.asarray(slots)):
        if 0 <= sl < initial.shape[0] * Bs:
            got = gpu[sl // Bs, :, sl % Bs, :][None]
            ok, _ = rope_close(got, k_new[t:t + 1], positions[t:t + 1], theta)
            if not ok:
                return False
    return True


def run_step(b: wl.DecodeBatch, *, kernel=pa.PA_KERNEL_AUTO, split_tokens: int = 0,
             max_ctas: int = 0, check_pool: bool = True, sample=None, fused: bool = False,
             pdl: bool = False, rope_theta: float = 0.0, ref_out=None):
    """Runs one step on both sides; returns a dict of results and checks.

    fused=False: pa_append_kv through the host slot mapping, then pa_decode.
    fused=True: pa_append_decode (append at position L-1 through the table, then decode).
    pdl=True: PA_FLAG_PDL (the decode kernel may start while the append kernel runs).
    rope_theta > 0 (fused only): q and the new K rows turned by RoPE at position L-1; the
    rotated K rows are held to rope_close's bound, every other byte must be identical.
    ref_out: the oracle's decode of this very step, when the caller already has it (it is
    computed here otherwise); returned as res["ref"] either way.
    """
    assert rope_theta == 0.0 or fused
    (slots, tables, lens), (o_slots, o_tables, o_lens) = host_step(b)
    assert np.array_equal(slots, o_slots), "slot mapping differs from the model"
    assert np.array_equal(tables, o_tables), "block tables differ from the model"
    assert np.array_equal(lens, o_lens)
    assert np.array_equal(slots, oracle.slot_mapping(o_tables, o_lens, b.block_size))

    desc = desc_of(b)
    k_cache, v_cache = to_dev(b.k_cache), to_dev(b.v_cache)
    q = to_dev(b.q)
    out = torch.empty_like(q)
    max_len = int(lens.max()) if lens.size else 0
    opts = pa.DecodeOptions(split_tokens=split_tokens, kernel=kernel, max_ctas=max_ctas,
                            flags=pa.PA_FLAG_CHECK | (pa.PA_FLAG_PDL if pdl else 0),
                            rope_theta=rope_theta)
    ws = torch.zeros(pa.pa_decode_workspace_size(b.batch, max_len, desc, opts), dtype=torch.uint8,
                     device=DEV)
    if fused:
        pa.pa_append_decode(q, to_dev(b.k_new), to_dev(b.v_new), k_cache, v_cache,
                            torch.from_numpy(tables).to(DEV), torch.from_numpy(lens).to(DEV),
                            max_len, b.scale, out, ws, desc, opts)
    else:
        pa.pa_append_kv(to_dev(b.k_new), to_dev(b.v_new), torch.from_numpy(slots).to(DEV), k_cache,
                        v_cache, desc)
        pa.pa_decode(q, k_cache, v_cache, torch.from_numpy(tables).to(DEV),
                     torch.from_numpy(lens).to(DEV), max_len, b.scale, out, ws, desc, opts)
    torch.cuda.synchronize()

    if rope_theta > 0:
        _, ref_k, ref_v, q_ref = oracle.rope_append_decode(b.q, b.k_new, b.v_new, o_slots, b.k_cache,
                                                           b.v_cache, o_tables, o_lens, b.scale,
                                                           rope_theta)
    else:
        ref_k, ref_v = oracle.append_kv(b.k_new, b.v_new, o_slots, b.k_cache, b.v_cache)
        q_ref = b.q
    res = {"splits": pa.pa_decode_max_splits(b.batch, max_len, desc, opts)}
    if check_pool:
        if rope_theta > 0:
            pos = np.maximum(o_lens - 1, 0).astype(np.int32)
            res["pool_equal"] = (rope_pool_matches(to_host_bits(k_cache), b.k_cache, b.k_new, o_slots,
                                                   pos, rope_theta) and
                                 np.array_equal(to_host_bits(v_cache), ref_v))
        else:
            res["pool_equal"] = (np.array_equal(to_host_bits(k_cache), ref_k) and
                                 np.array_equal(to_host_bits(v_cache), ref_v))
    got = out.float().cpu().numpy().astype(np.float64)
    if ref_out is not None:
        ref = ref_out
        res["ok"], res["excess"] = oracle.within_tolerance(got, ref)
    elif sample is None:
        ref = oracle.paged_decode(q_ref, ref_k, ref_v, o_tables, o_lens, b.scale)
        res["ok"], res["excess"] = oracle.within_tolerance(got, ref)
    else:
        idx = np.asarray(sample)
        ref = oracle.paged_decode(q_ref[idx], ref_k, ref_v, o_tables[idx], o_lens[idx], b.scale)
        res["ok"], res["excess"] = oracle.within_tolerance(got[idx], ref)
    res["out"] = got
    res["ref"] = ref
    res["finite"] = bool(np.isfinite(got).all())
    return res
