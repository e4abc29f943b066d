"""Seeded synthetic workloads for paged decode attention.

This module only draws random numbers and lays out *initial* state (which
physical blocks a sequence starts with, the bytes already in the pool, the new
token's q/k/v).  It holds none of the method's arithmetic: no slot mapping, no
gather, no softmax.  Both the CUDA path (tests, bench, smoke) and the CPU
oracle receive the same bytes from here.

Configurations (sizes as the workload descriptions state them):

* C1 ``config1``: batch 2, cached lengths 5 and 37, Hq=2, Hkv=1, D=64, Bs=16,
  8 physical blocks in a seeded random order, scale 1/sqrt(64).
* C2 ``config2``: Llama-3.2-1B-shaped layer, Hq=32, Hkv=8, D=64, Bs=16,
  batch 64, cached lengths uniform in [128, 2048], pool = needed blocks + 10 %.
* C3 ``config3``: Hq=32, Hkv=8, D=64, Bs=256, batch 32, a 1024-token prefix
  held in 4 physical blocks shared by every table, suffixes uniform in
  [256, 7168].
* C4 ``config4``: Hq=64, Hkv=8, D=128, Bs=16, batch 4, cached lengths
  32768, 65536, 98304, 131072.
* C5 ``Trace5``: 16 layers, Hq=32, Hkv=8, D=64, Bs=16, 256 live sequences with
  lognormal lengths (median 512, sigma 1, clipped to [1, 16384]), 100 decode
  steps, each live sequence finishing after a step with probability 0.01 and
  replaced by a fresh one.

All values are standard normals rounded to bf16 (see gen.c for the stream).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_SO = os.path.join(_HERE, "libgen.so")
_LIB = None

CONFIG_SEED_BASE = 0xA5E00000
MASK64 = (1 << 64) - 1


def build(force: bool = False) -> str:
    """Compile gen.c into libgen.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _lib():
    global _LIB
    if _LIB is None:
        build()
        lib = ctypes.CDLL(_SO)
        u64, i64, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p
        for name in ("gen_words", "gen_uniform_f64", "gen_normal_f64", "gen_normal_bf16"):
            fn = getattr(lib, name)
            fn.argtypes = [u64, u64, i64, vp]
            fn.restype = None
        lib.gen_num_threads.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def stream_seed(base: int, name: str) -> int:
    """64-bit seed of the named tensor stream under a configuration seed."""
    h = 0xCBF29CE484222325
    for ch in name.encode():
        h = ((h ^ ch) * 0x100000001B3) & MASK64
    z = (base ^ h) & MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def words(seed: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    if n:
        _lib().gen_words(seed, offset, n, out.ctypes.data)
    return out


def uniform(seed: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    if n:
        _lib().gen_uniform_f64(seed, offset, n, out.ctypes.data)
    return out


def normal(seed: int, n: int, offset: int = 0) -> np.ndarray:
    assert offset % 2 == 0
    out = np.empty(n, dtype=np.float64)
    if n:
        _lib().gen_normal_f64(seed, offset, n, out.ctypes.data)
    return out


def normal_bf16(seed: int, shape, offset: int = 0) -> np.ndarray:
    """Standard normals rounded to bf16, returned as uint16 bit patterns."""
    assert offset % 2 == 0
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    if n:
        _lib().gen_normal_bf16(seed, offset, n, out.ctypes.data)
    return out.reshape(shape)


def uniform_ints(seed: int, n: int, lo: int, hi: int, offset: int = 0) -> np.ndarray:
    """n integers uniform in [lo, hi] (inclusive)."""
    u = uniform(seed, n, offset)
    return (lo + np.floor(u * (hi - lo + 1))).astype(np.int64).clip(lo, hi)


def permutation(seed: int, n: int) -> np.ndarray:
    """Seeded uniform random permutation of range(n) (sort by random keys)."""
    return np.argsort(words(seed, n), kind="stable").astype(np.int32)


def lognormal_lengths(seed: int, n: int, median: float, sigma: float, lo: int, hi: int,
                      offset: int = 0) -> np.ndarray:
    z = normal(seed, n, offset)
    return np.clip(np.rint(np.exp(math.log(median) + sigma * z)), lo, hi).astype(np.int64)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32 (test helper)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _ceil_div(a, b):
    return -(-a // b)


@dataclass
class DecodeBatch:
    """One decode step's inputs: cached state before the append plus the new token.

    ``context_lens`` counts the tokens already cached (before this step's
    append).  ``block_tables`` rows list the physical blocks that hold them
    (-1 beyond).  ``free_order`` lists the free physical blocks, first to be
    handed out first.
    """
    name: str
    seed: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    max_blocks_per_seq: int
    context_lens: np.ndarray          # int32 [B]
    block_tables: np.ndarray          # int32 [B, MB]
    free_order: np.ndarray            # int32 [F]
    k_cache: np.ndarray               # uint16 (bf16 bits) [N, Hkv, Bs, D]
    v_cache: np.ndarray               # uint16 [N, Hkv, Bs, D]
    q: np.ndarray                     # uint16 [B, Hq, D]
    k_new: np.ndarray                 # uint16 [B, Hkv, D]
    v_new: np.ndarray                 # uint16 [B, Hkv, D]
    scale: float
    shared_prefix_blocks: int = 0
    meta: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return int(self.context_lens.shape[0])


def make_batch(name: str, seed: int, lens, *, num_q_heads: int, num_kv_heads: int, head_dim: int,
               block_size: int, num_blocks: int | None = None, free_fraction: float = 0.10,
               shared_prefix_tokens: int = 0, growth_tokens: int = 1, scale: float | None = None,
               max_blocks_per_seq: int | None = None, with_pool: bool = True) -> DecodeBatch:
    """Lay out a batch of sequences in a pool whose blocks come in seeded random order.

    ``lens`` are the cached lengths.  A shared prefix of ``shared_prefix_tokens``
    (a whole number of blocks) is held by the same physical blocks in every
    table.  The pool holds every block the batch needs after ``growth_tokens``
    more tokens, plus ``free_fraction`` spare, unless ``num_blocks`` is given.
    """
    lens = np.asarray(lens, dtype=np.int64)
    B = int(lens.shape[0])
    Bs = block_size
    assert shared_prefix_tokens % Bs == 0
    P = shared_prefix_tokens // Bs
    assert np.all(lens >= shared_prefix_tokens)
    blocks_now = _ceil_div(lens, Bs)
    blocks_later = _ceil_div(lens + growth_tokens, Bs)
    needed = P + int(np.sum(blocks_later - P))
    if num_blocks is None:
        num_blocks = int(math.ceil(needed * (1.0 + free_fraction)))
    assert num_blocks >= P + int(np.sum(blocks_now - P))
    MB = max_blocks_per_seq or int(blocks_later.max())
    perm = permutation(stream_seed(seed, "block_order"), num_blocks)
    tables = np.full((B, MB), -1, dtype=np.int32)
    cursor = 0
    prefix = perm[cursor:cursor + P]
    cursor += P
    for b in range(B):
        nb = int(blocks_now[b])
        tables[b, :P] = prefix
        own = nb - P
        tables[b, P:nb] = perm[cursor:cursor + own]
        cursor += own
    free_order = perm[cursor:].copy()
    Hq, Hkv, D = num_q_heads, num_kv_heads, head_dim
    if with_pool:
        k_cache = normal_bf16(stream_seed(seed, "k_cache"), (num_blocks, Hkv, Bs, D))
        v_cache = normal_bf16(stream_seed(seed, "v_cache"), (num_blocks, Hkv, Bs, D))
    else:
        k_cache = v_cache = np.empty((0, Hkv, Bs, D), dtype=np.uint16)
    q = normal_bf16(stream_seed(seed, "q"), (B, Hq, D))
    k_new = normal_bf16(stream_seed(seed, "k_new"), (B, Hkv, D))
    v_new = normal_bf16(stream_seed(seed, "v_new"), (B, Hkv, D))
    return DecodeBatch(name=name, seed=seed, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                       block_size=Bs, num_blocks=num_blocks, max_blocks_per_seq=MB,
                       context_lens=lens.astype(np.int32), block_tables=tables,
                       free_order=free_order, k_cache=k_cache, v_cache=v_cache, q=q,
                       k_new=k_new, v_new=v_new,
                       scale=scale if scale is not None else 1.0 / math.sqrt(D),
                       shared_prefix_blocks=P)


def config1(**kw) -> DecodeBatch:
    """Tiny correctness case: lengths 5 and 37, Hq=2, Hkv=1, D=64, Bs=16, 8 blocks."""
    return make_batch("C1", CONFIG_SEED_BASE + 1, [5, 37], num_q_heads=2, num_kv_heads=1,
                      head_dim=64, block_size=16, num_blocks=8, scale=1.0 / 8.0, **kw)


def config2_lens(seed: int = CONFIG_SEED_BASE + 2, batch: int = 64) -> np.ndarray:
    return uniform_ints(stream_seed(seed, "context_lens"), batch, 128, 2048)


def config2(**kw) -> DecodeBatch:
    """Llama-3.2-1B-shaped layer: B=64, Hq=32, Hkv=8, D=64, Bs=16, L ~ U[128, 2048]."""
    seed = CONFIG_SEED_BASE + 2
    return make_batch("C2", seed, config2_lens(seed), num_q_heads=32, num_kv_heads=8,
                      head_dim=64, block_size=16, **kw)


def config3(**kw) -> DecodeBatch:
    """Bs=256 with a 1024-token prefix shared by all 32 tables, suffix ~ U[256, 7168]."""
    seed = CONFIG_SEED_BASE + 3
    suffix = uniform_ints(stream_seed(seed, "suffix_lens"), 32, 256, 7168)
    return make_batch("C3", seed, 1024 + suffix, num_q_heads=32, num_kv_heads=8, head_dim=64,
                      block_size=256, shared_prefix_tokens=1024, **kw)


def config4(**kw) -> DecodeBatch:
    """Long contexts 32k..128k, Hq=64, Hkv=8, D=128, Bs=16 (split-KV + merge)."""
    return make_batch("C4", CONFIG_SEED_BASE + 4, [32768, 65536, 98304, 131072],
                      num_q_heads=64, num_kv_heads=8, head_dim=128, block_size=16, **kw)


def small_batch(seed: int, lens, *, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16,
                **kw) -> DecodeBatch:
    return make_batch("small-%x" % seed, seed, lens, num_q_heads=num_q_heads,
                      num_kv_heads=num_kv_heads, head_dim=head_dim, block_size=block_size, **kw)


CONFIGS = {"c1": config1, "c2": config2, "c3": config3, "c4": config4}


class Trace5:
    """Continuous-batching trace (C5): the per-step events, not the pools.

    Step s (0-based) first retires the sequences whose finish draw for step s
    fired (s >= 1), in increasing slot order, then admits a replacement in each
    retired slot (increasing slot order) with a fresh lognormal length, then
    appends one token to every live sequence.  The trace is pure input:
    which slots finish and how long the newcomers are.
    """

    def __init__(self, *, layers: int = 16, steps: int = 100, batch: int = 256,
                 num_q_heads: int = 32, num_kv_heads: int = 8, head_dim: int = 64,
                 block_size: int = 16, median: float = 512.0, sigma: float = 1.0,
                 max_len: int = 16384, finish_p: float = 0.01,
                 seed: int = CONFIG_SEED_BASE + 5, pool_slack: float = 1.10):
        self.layers, self.steps, self.batch = layers, steps, batch
        self.num_q_heads, self.num_kv_heads, self.head_dim = num_q_heads, num_kv_heads, head_dim
        self.block_size, self.seed = block_size, seed
        self.scale = 1.0 / math.sqrt(head_dim)
        self.initial_lens = lognormal_lengths(stream_seed(seed, "initial_lens"), batch,
                                              median, sigma, 1, max_len)
        u = uniform(stream_seed(seed, "finish"), steps * batch).reshape(steps, batch)
        self.finish = u < finish_p
        self.finish[0, :] = False
        n_new = int(self.finish.sum())
        self.new_lens = lognormal_lengths(stream_seed(seed, "new_lens"), max(n_new + (n_new & 1), 2),
                                          median, sigma, 1, max_len)[:n_new]
        # Pool: the most blocks the trace ever holds at once (counted per step after the
        # newcomers arrive and every live sequence has its new token), plus slack.
        Bs = block_size
        lens = self.initial_lens.copy()
        peak, k = 0, 0
        for s in range(steps):
            for slot in np.nonzero(self.finish[s])[0]:
                lens[slot] = self.new_lens[k]
                k += 1
            lens = lens + 1
            peak = max(peak, int(np.sum(_ceil_div(lens, Bs))))
        self.num_blocks = int(math.ceil(pool_slack * peak))
        self.max_blocks_per_seq = _ceil_div(max_len + steps, Bs)
        self.free_order = permutation(stream_seed(seed, "block_order"), self.num_blocks)

    def events(self):
        """Yield (step, retired_slots, [(slot, new_len), ...]) for every step."""
        k = 0
        for s in range(self.steps):
            retired = np.nonzero(self.finish[s])[0].tolist()
            admitted = []
            for slot in retired:
                admitted.append((slot, int(self.new_lens[k])))
                k += 1
            yield s, retired, admitted

    def pool(self, layer: int):
        """(k_cache, v_cache) bf16 bits for one layer, [N, Hkv, Bs, D]."""
        shape = (self.num_blocks, self.num_kv_heads, self.block_size, self.head_dim)
        return (normal_bf16(stream_seed(self.seed, "k_cache/%d" % layer), shape),
                normal_bf16(stream_seed(self.seed, "v_cache/%d" % layer), shape))

    def token_inputs(self, layer: int, step: int):
        """(q [B,Hq,D], k [B,Hkv,D], v [B,Hkv,D]) bf16 bits of the step's new token."""
        B, Hq, Hkv, D = self.batch, self.num_q_heads, self.num_kv_heads, self.head_dim
        tag = "%d/%d" % (layer, step)
        return (normal_bf16(stream_seed(self.seed, "q/" + tag), (B, Hq, D)),
                normal_bf16(stream_seed(self.seed, "k_new/" + tag), (B, Hkv, D)),
                normal_bf16(stream_seed(self.seed, "v_new/" + tag), (B, Hkv, D)))
