"""fp64 CPU oracle for paged KV append and paged decode attention.

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and bench.py's
CPU-baseline leg are the only callers.  The product path never imports this
package.  The arithmetic lives in ``pa_oracle.c`` (plain C, fp64); this module
only marshals numpy arrays into it.  ``block_manager.py`` holds the reference
model of the host block manager.

Array conventions (bf16 values travel as uint16 bit patterns):
    q            uint16 [B, Hq, D]
    k/v_cache    uint16 [N, Hkv, Bs, D]     (physical blocks)
    block_tables int32  [B, MB]             (physical block of logical block i)
    context_lens int32  [B]                 (tokens attended)
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .block_manager import BlockManagerModel, BlockPoolModel, OutOfBlocks, SharedBlockWrite  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")
_LIB = None


def build(force: bool = False) -> str:
    """Compile pa_oracle.c into liboracle.so next to it (gcc, fp64, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _lib():
    global _LIB
    if _LIB is None:
        build()
        lib = ctypes.CDLL(_SO)
        i64, vp, dbl = ctypes.c_int64, ctypes.c_void_p, ctypes.c_double
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_double.restype = dbl
        lib.oracle_kv_bytes.argtypes = [i64] * 5
        lib.oracle_kv_bytes.restype = i64
        lib.oracle_slot.argtypes = [vp, i64, i64]
        lib.oracle_slot.restype = i64
        lib.oracle_slot_mapping.argtypes = [vp, i64, vp, i64, i64, vp]
        lib.oracle_slot_mapping.restype = None
        lib.oracle_append_kv.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, vp, vp]
        lib.oracle_append_kv.restype = None
        lib.oracle_paged_decode.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64,
                                            dbl, vp, vp]
        lib.oracle_paged_decode.restype = ctypes.c_int
        lib.oracle_paged_decode_partial.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64,
                                                    i64, dbl, i64, i64, vp, vp]
        lib.oracle_paged_decode_partial.restype = ctypes.c_int
        lib.oracle_merge_partials.argtypes = [vp, vp, i64, i64, vp]
        lib.oracle_merge_partials.restype = None
        lib.oracle_rope.argtypes = [vp, i64, i64, i64, vp, dbl, vp]
        lib.oracle_rope.restype = None
        lib.oracle_round_bf16.argtypes = [vp, i64, vp]
        lib.oracle_round_bf16.restype = None
        lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_double.restype = dbl
        lib.oracle_e4m3_from_float.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_from_float.restype = ctypes.c_uint8
        lib.oracle_quantize_e4m3.argtypes = [vp, i64, ctypes.c_float, vp]
        lib.oracle_quantize_e4m3.restype = None
        lib.oracle_append_kv_e4m3.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, vp, vp]
        lib.oracle_append_kv_e4m3.restype = None
        lib.oracle_paged_decode_e4m3.argtypes = [vp, vp, vp, dbl, dbl, vp, vp, i64, i64, i64, i64, i64,
                                                 i64, dbl, vp]
        lib.oracle_paged_decode_e4m3.restype = ctypes.c_int
        lib.oracle_paged_prefill.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, dbl, vp]
        lib.oracle_paged_prefill.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_num_threads.restype = None
        lib.oracle_num_threads.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError("expected %s, got %s" % (np.dtype(dtype), a.dtype))
    return a


def set_num_threads(n: int) -> None:
    """OpenMP threads used by the decode oracle (0 = OpenMP default)."""
    _lib().oracle_set_num_threads(int(n))


def num_threads() -> int:
    return int(_lib().oracle_num_threads())


def bf16_to_double(bits: int) -> float:
    return float(_lib().oracle_bf16_to_double(int(bits)))


def kv_bytes(layers: int, kv_heads: int, head_dim: int, tokens: int, bytes_per_element: int) -> int:
    return int(_lib().oracle_kv_bytes(layers, kv_heads, head_dim, tokens, bytes_per_element))


def slot(table_row: np.ndarray, position: int, block_size: int) -> int:
    row = _c(table_row, np.int32)
    return int(_lib().oracle_slot(row.ctypes.data, int(position), int(block_size)))


def slot_mapping(block_tables: np.ndarray, lengths_after_append: np.ndarray, block_size: int) -> np.ndarray:
    """Slot of each sequence's newest token (position length-1); -1 for empty sequences."""
    bt = _c(block_tables, np.int32)
    lens = _c(lengths_after_append, np.int32)
    out = np.empty(lens.shape[0], dtype=np.int64)
    _lib().oracle_slot_mapping(bt.ctypes.data, bt.shape[1], lens.ctypes.data, lens.shape[0],
                               int(block_size), out.ctypes.data)
    return out


def append_kv(k: np.ndarray, v: np.ndarray, slot_mapping_: np.ndarray, k_cache: np.ndarray,
              v_cache: np.ndarray, *, in_place: bool = False):
    """Write each token's K/V rows into its slot; returns the (new) caches."""
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    sm = _c(slot_mapping_, np.int64)
    if not in_place:
        k_cache = k_cache.copy()
        v_cache = v_cache.copy()
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    assert k_cache.dtype == np.uint16 and v_cache.dtype == np.uint16
    N, Hkv, Bs, D = k_cache.shape
    T = sm.shape[0]
    assert k.shape == (T, Hkv, D) and v.shape == (T, Hkv, D)
    _lib().oracle_append_kv(k.ctypes.data, v.ctypes.data, sm.ctypes.data, T, Hkv, D, Bs, N,
                            k_cache.ctypes.data, v_cache.ctypes.data)
    return k_cache, v_cache


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale: float,
                 return_weight_sums: bool = False):
    """fp64 [B, Hq, D] attention output (and optionally the softmax weight sums)."""
    q = _c(q, np.uint16)
    k_cache = _c(k_cache, np.uint16)
    v_cache = _c(v_cache, np.uint16)
    bt = _c(block_tables, np.int32)
    lens = _c(context_lens, np.int32)
    B, Hq, D = q.shape
    N, Hkv, Bs, D2 = k_cache.shape
    assert D2 == D and v_cache.shape == k_cache.shape and bt.shape[0] == B and lens.shape == (B,)
    out = np.empty((B, Hq, D), dtype=np.float64)
    wsum = np.empty((B, Hq), dtype=np.float64) if return_weight_sums else None
    rc = _lib().oracle_paged_decode(q.ctypes.data, k_cache.ctypes.data, v_cache.ctypes.data,
                                    bt.ctypes.data, lens.ctypes.data, B, Hq, Hkv, D, Bs,
                                    bt.shape[1], float(scale), out.ctypes.data,
                                    wsum.ctypes.data if wsum is not None else None)
    if rc != 0:
        raise RuntimeError("oracle_paged_decode failed (%d)" % rc)
    return (out, wsum) if return_weight_sums else out


def paged_decode_partial(q, k_cache, v_cache, block_tables, context_lens, scale: float,
                         t0: int, t1: int):
    """Normalised partial output [B, Hq, D] and natural-log LSE [B, Hq] over tokens [t0, t1)."""
    q = _c(q, np.uint16)
    k_cache = _c(k_cache, np.uint16)
    v_cache = _c(v_cache, np.uint16)
    bt = _c(block_tables, np.int32)
    lens = _c(context_lens, np.int32)
    B, Hq, D = q.shape
    N, Hkv, Bs, _ = k_cache.shape
    o = np.empty((B, Hq, D), dtype=np.float64)
    lse = np.empty((B, Hq), dtype=np.float64)
    rc = _lib().oracle_paged_decode_partial(q.ctypes.data, k_cache.ctypes.data,
                                            v_cache.ctypes.data, bt.ctypes.data,
                                            lens.ctypes.data, B, Hq, Hkv, D, Bs, bt.shape[1],
                                            float(scale), int(t0), int(t1), o.ctypes.data,
                                            lse.ctypes.data)
    if rc != 0:
        raise RuntimeError("oracle_paged_decode_partial failed (%d)" % rc)
    return o, lse


def merge_partials(o: np.ndarray, lse: np.ndarray) -> np.ndarray:
    """Merge S partial states of one query: o [S, D], lse [S] -> [D]."""
    o = _c(o, np.float64)
    lse = _c(lse, np.float64)
    S, D = o.shape
    out = np.empty(D, dtype=np.float64)
    _lib().oracle_merge_partials(o.ctypes.data, lse.ctypes.data, S, D, out.ctypes.data)
    return out


def within_tolerance(gpu: np.ndarray, ref: np.ndarray, atol: float = 1e-2, rtol: float = 1e-2):
    """Elementwise |gpu - ref| <= atol + rtol * |ref|; returns (ok, worst excess)."""
    err = np.abs(np.asarray(gpu, dtype=np.float64) - ref)
    bound = atol + rtol * np.abs(ref)
    excess = float(np.max(err - bound)) if err.size else 0.0
    return bool(np.all(err <= bound)), excess


def rope(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """fp64 rotary embedding of bf16 rows x [T, H, D] at positions [T] (unrounded).

    Pair (x[i], x[i + D/2]) turns by positions[t] * theta^(-2i/D) (rotate-half pairing)."""
    x = _c(x, np.uint16)
    pos = _c(positions, np.int32)
    T, H, D = x.shape
    assert pos.shape == (T,) and D % 2 == 0
    out = np.empty((T, H, D), dtype=np.float64)
    _lib().oracle_rope(x.ctypes.data, T, H, D, pos.ctypes.data, float(theta), out.ctypes.data)
    return out


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Nearest bf16 (ties to even) of each double, as uint16 bit patterns."""
    x = _c(x, np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _lib().oracle_round_bf16(x.ctypes.data, x.size, out.ctypes.data)
    return out


def rope_bf16(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotary embedding rounded to bf16, as the rotated rows are stored."""
    return round_bf16(rope(x, positions, theta))


def rope_append_decode(q, k_new, v_new, slots, k_cache, v_cache, block_tables, context_lens,
                       scale: float, theta: float):
    """One decode step with RoPE at each sequence's newest position (context_lens[b] - 1):
    q and the new K rows are rotated and rounded to bf16, K (rotated) and V go into their
    slots, and the rotated q attends over the cache.  Returns (out fp64, k_cache, v_cache, q_rot)."""
    lens = _c(context_lens, np.int32)
    pos = np.maximum(lens - 1, 0).astype(np.int32)
    q_rot = rope_bf16(q, pos, theta)
    k_rot = rope_bf16(k_new, pos, theta)
    kc, vc = append_kv(k_rot, v_new, slots, k_cache, v_cache)
    return paged_decode(q_rot, kc, vc, block_tables, lens, scale), kc, vc, q_rot


def e4m3_to_double(codes) -> np.ndarray:
    """Value of each E4M3 code (NaN for the NaN codes)."""
    c = np.asarray(codes, dtype=np.uint8)
    lib = _lib()
    return np.array([lib.oracle_e4m3_to_double(int(x)) for x in c.ravel()], dtype=np.float64).reshape(c.shape)


def e4m3_from_float(y) -> np.ndarray:
    """E4M3 code of each float32 value: nearest, ties to even, saturating at +-448."""
    y = np.asarray(y, dtype=np.float32)
    lib = _lib()
    return np.array([lib.oracle_e4m3_from_float(float(v)) for v in y.ravel()], dtype=np.uint8).reshape(y.shape)


def inv_scale(scale: float) -> np.float32:
    """float(1 / scale), the multiplier that quantization applies (both sides form it in float)."""
    return np.float32(1.0) / np.float32(scale)


def quantize_e4m3(x: np.ndarray, scale: float) -> np.ndarray:
    """E4M3 codes of bf16 values x: e4m3(float(x) * float(1/scale))."""
    x = _c(x, np.uint16)
    out = np.empty(x.shape, dtype=np.uint8)
    _lib().oracle_quantize_e4m3(x.ctypes.data, x.size, float(inv_scale(scale)), out.ctypes.data)
    return out


def append_kv_e4m3(k_codes, v_codes, slot_mapping_, k_cache, v_cache):
    """Write each token's (already quantized) K/V codes into its slot of u8 pools (copies)."""
    k = _c(k_codes, np.uint8)
    v = _c(v_codes, np.uint8)
    sm = _c(slot_mapping_, np.int64)
    kc, vc = k_cache.copy(), v_cache.copy()
    N, Hkv, Bs, D = kc.shape
    _lib().oracle_append_kv_e4m3(k.ctypes.data, v.ctypes.data, sm.ctypes.data, sm.shape[0], Hkv, D, Bs, N,
                                 kc.ctypes.data, vc.ctypes.data)
    return kc, vc


def paged_decode_e4m3(q, k_cache, v_cache, k_scale: float, v_scale: float, block_tables, context_lens,
                      scale: float):
    """fp64 [B, Hq, D] attention over E4M3 pools (values = code value x scale)."""
    q = _c(q, np.uint16)
    kc = _c(k_cache, np.uint8)
    vc = _c(v_cache, np.uint8)
    bt = _c(block_tables, np.int32)
    lens = _c(context_lens, np.int32)
    B, Hq, D = q.shape
    N, Hkv, Bs, _ = kc.shape
    out = np.empty((B, Hq, D), dtype=np.float64)
    rc = _lib().oracle_paged_decode_e4m3(q.ctypes.data, kc.ctypes.data, vc.ctypes.data, float(k_scale),
                                         float(v_scale), bt.ctypes.data, lens.ctypes.data, B, Hq, Hkv, D,
                                         Bs, bt.shape[1], float(scale), out.ctypes.data)
    if rc != 0:
        raise RuntimeError("oracle_paged_decode_e4m3 failed (%d)" % rc)
    return out


def paged_prefill(q, k_cache, v_cache, block_tables, cu_q, context_lens, scale: float) -> np.ndarray:
    """fp64 causal attention of each sequence's last Tq = cu_q[b+1]-cu_q[b] tokens (queries,
    rows of q [total_q, Hq, D]) over its paged cache of context_lens[b] tokens."""
    q = _c(q, np.uint16)
    kc = _c(k_cache, np.uint16)
    vc = _c(v_cache, np.uint16)
    bt = _c(block_tables, np.int32)
    cq = _c(cu_q, np.int32)
    lens = _c(context_lens, np.int32)
    T, Hq, D = q.shape
    N, Hkv, Bs, _ = kc.shape
    B = lens.shape[0]
    assert cq.shape == (B + 1,) and cq[-1] == T
    out = np.zeros((T, Hq, D), dtype=np.float64)
    rc = _lib().oracle_paged_prefill(q.ctypes.data, kc.ctypes.data, vc.ctypes.data, bt.ctypes.data, cq.ctypes.data,
                                     lens.ctypes.data, B, Hq, Hkv, D, Bs, bt.shape[1], float(scale), out.ctypes.data)
    if rc != 0:
        raise RuntimeError("oracle_paged_prefill failed (%d)" % rc)
    return out
