"""The C-ABI library loads, exports what include/pa.h declares, and rejects bad
arguments before touching a GPU (CPU only: no compute call runs here)."""
import ctypes
import subprocess

import numpy as np
import pytest

import pagedattention_kv_cache_pa_b200 as pa
from pagedattention_kv_cache_pa_b200 import binding


def test_every_declared_symbol_is_exported():
    declared = pa.declared_symbols()
    assert len(declared) >= 20
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    for s in declared:
        assert hasattr(binding.lib, s)
    # nothing beyond the declared ABI leaks out
    assert exported == set(declared), sorted(exported - set(declared))


def test_status_strings():
    for code in range(-9, 1):
        assert binding.STATUS[code] in pa.pa_status_string(code)
    assert "unknown" in pa.pa_status_string(-1234)


def _desc(**kw):
    base = dict(num_blocks=8, block_size=16, num_kv_heads=1, num_q_heads=2, head_dim=64,
                max_blocks_per_seq=4)
    base.update(kw)
    return pa.CacheDesc.make(**base)


def test_append_rejects_bad_arguments_without_a_gpu():
    lib = binding.lib
    d = _desc()
    fake = ctypes.c_void_p(0x10000)          # never dereferenced: validation fails first
    assert lib.pa_append_kv(None, fake, fake, 1, fake, fake, ctypes.byref(d), None) == -1
    assert lib.pa_append_kv(fake, fake, fake, -1, fake, fake, ctypes.byref(d), None) == -1
    assert lib.pa_append_kv(fake, fake, fake, 0, fake, fake, ctypes.byref(d), None) == 0  # no-op
    assert lib.pa_append_kv(fake, fake, fake, 1, fake, fake, None, None) == -1
    bad = _desc(num_q_heads=3, num_kv_heads=2)
    assert lib.pa_append_kv(fake, fake, fake, 1, fake, fake, ctypes.byref(bad), None) == -1
    odd = _desc(head_dim=60)
    assert lib.pa_append_kv(fake, fake, fake, 1, fake, fake, ctypes.byref(odd), None) == -1
    mis = ctypes.c_void_p(0x10002)
    assert lib.pa_append_kv(mis, fake, fake, 1, fake, fake, ctypes.byref(d), None) == -1


def test_decode_rejects_unsupported_shapes_without_a_gpu():
    lib = binding.lib
    fake = ctypes.c_void_p(0x10000)
    for kw, want in ((dict(head_dim=96), -2), (dict(block_size=12), -2),
                     (dict(num_q_heads=34, num_kv_heads=2), -2), (dict(num_q_heads=3, num_kv_heads=2), -1)):
        d = _desc(**kw)
        rc = lib.pa_decode(fake, fake, fake, fake, fake, 1, 16, ctypes.c_float(0.1), fake, fake, 1 << 20,
                           ctypes.byref(d), None)
        assert rc == want, (kw, rc)
    d = _desc()
    assert lib.pa_decode(fake, fake, fake, fake, fake, -1, 16, ctypes.c_float(0.1), fake, fake, 0,
                         ctypes.byref(d), None) == -1
    assert lib.pa_decode(fake, fake, fake, fake, fake, 0, 16, ctypes.c_float(0.1), fake, fake, 0,
                         ctypes.byref(d), None) == 0   # empty batch: nothing to do
    opts = pa.DecodeOptions(split_tokens=100)          # not a multiple of 64
    assert lib.pa_decode_max_splits(1, 16, ctypes.byref(d), ctypes.byref(opts)) == -1
    opts = pa.DecodeOptions(split_tokens=128, kernel=pa.PA_KERNEL_SIMT)  # no device query needed
    assert lib.pa_decode_max_splits(1, 1000, ctypes.byref(d), ctypes.byref(opts)) == 8
    assert pa.pa_decode_workspace_size(2, 1000, d, opts) > 0
    for bad in (8, 1 << 30, -1):                       # flag bits outside CHECK | PDL | SELFTEST_STALL
        o = pa.DecodeOptions(flags=bad)
        assert lib.pa_decode_ex(fake, fake, fake, fake, fake, 1, 16, ctypes.c_float(0.1), fake, fake,
                                1 << 20, ctypes.byref(d), ctypes.byref(o), None) == -1, bad


def test_decode_describe_without_a_gpu():
    d = _desc()
    opts = pa.DecodeOptions(split_tokens=128, kernel=pa.PA_KERNEL_SIMT)   # no device query needed
    info = pa.pa_decode_describe(2, 1000, d, opts)
    assert (info.kernel, info.ctas, info.split_tokens, info.max_splits) == (pa.PA_KERNEL_SIMT, 0, 128, 8)
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_describe(2, 1000, _desc(head_dim=96), opts)
    assert e.value.status == -2
    assert binding.lib.pa_decode_describe(2, 1000, ctypes.byref(d), ctypes.byref(opts), None) == -1


def test_noalloc_returns_pa_decode_errors_without_a_gpu():
    # refused before any device work: the same codes pa_decode_ex gives
    lib = binding.lib
    fake = ctypes.c_void_p(0x10000)
    cases = [(_desc(head_dim=96), None, -2),                                   # head_dim not built
             (_desc(num_q_heads=34, num_kv_heads=2), None, -2),                # group of 17
             (_desc(), pa.DecodeOptions(kernel=pa.PA_KERNEL_SIMT, kv_dtype=pa.PA_KV_E4M3,
                                        k_scale=1.0, v_scale=1.0), -2),        # E4M3 needs the tensor kernel
             (_desc(), pa.DecodeOptions(split_tokens=100, kernel=pa.PA_KERNEL_SIMT), -1),
             (_desc(), pa.DecodeOptions(flags=8), -1)]
    for d, o, want in cases:
        ob = ctypes.byref(o) if o is not None else None
        got = lib.pa_decode_noalloc(fake, fake, fake, fake, fake, 1, 16, ctypes.c_float(0.1), fake,
                                    ctypes.byref(d), ob, None)
        ref = lib.pa_decode_ex(fake, fake, fake, fake, fake, 1, 16, ctypes.c_float(0.1), fake, fake,
                               1 << 20, ctypes.byref(d), ob, None)
        assert got == ref == want, (want, got, ref)


def test_rope_append_rejects_bad_arguments_without_a_gpu():
    lib = binding.lib
    fake = ctypes.c_void_p(0x10000)
    d = _desc()
    args = lambda n, theta, dd: (fake, fake, fake, fake, fake, fake, n, ctypes.c_float(theta), fake, fake,
                                 ctypes.byref(dd), None)
    assert lib.pa_rope_append_kv(*args(1, 0.0, d)) == -1            # theta must be > 0
    assert lib.pa_rope_append_kv(*args(1, -5.0, d)) == -1
    assert lib.pa_rope_append_kv(*args(1, float("nan"), d)) == -1
    assert lib.pa_rope_append_kv(*args(1, float("inf"), d)) == -1
    assert lib.pa_rope_append_kv(*args(-1, 10000.0, d)) == -1
    assert lib.pa_rope_append_kv(*args(1, 10000.0, _desc(head_dim=96))) == -2
    assert lib.pa_rope_append_kv(*args(0, 10000.0, d)) == 0          # nothing to do
    mis = ctypes.c_void_p(0x10002)                                  # q not 16-byte aligned
    assert lib.pa_rope_append_kv(mis, fake, fake, fake, fake, fake, 1, ctypes.c_float(1e4), fake, fake,
                                 ctypes.byref(d), None) == -1
    for bad in (-1.0, float("nan")):                                 # decode options too
        o = pa.DecodeOptions(rope_theta=bad)
        assert lib.pa_decode_ex(fake, fake, fake, fake, fake, 1, 16, ctypes.c_float(0.1), fake, fake,
                                1 << 20, ctypes.byref(d), ctypes.byref(o), None) == -1, bad


def test_binding_refuses_caches_smaller_than_the_pool():
    import torch
    d = _desc()                                         # 8 blocks x 1 head x 16 x 64
    small = torch.zeros(8 * 16 * 64 - 1, dtype=torch.bfloat16)
    pairs = torch.zeros((1, 2), dtype=torch.int32)
    with pytest.raises(ValueError):
        pa.pa_copy_blocks(small, small, pairs, d)
    with pytest.raises(ValueError):
        pa.pa_append_kv(small, small, torch.zeros(1, dtype=torch.int64), small, small, d)


def test_e4m3_arguments_rejected_without_a_gpu():
    lib = binding.lib
    fake = ctypes.c_void_p(0x10000)
    d = _desc()
    for ks, vs in ((0.0, 1.0), (1.0, -1.0), (float("nan"), 1.0), (1.0, float("inf"))):
        assert lib.pa_append_kv_e4m3(fake, fake, fake, 1, ctypes.c_float(ks), ctypes.c_float(vs), fake, fake,
                                     ctypes.byref(d), None) == -1, (ks, vs)
    assert lib.pa_append_kv_e4m3(fake, fake, fake, 0, ctypes.c_float(1.0), ctypes.c_float(1.0), fake, fake,
                                 ctypes.byref(d), None) == 0
    call = lambda o: lib.pa_decode_ex(fake, fake, fake, fake, fake, 1, 16, ctypes.c_float(0.1), fake, fake,
                                      1 << 20, ctypes.byref(d), ctypes.byref(o), None)
    assert call(pa.DecodeOptions(kv_dtype=2)) == -1                            # unknown dtype
    assert call(pa.DecodeOptions(kv_dtype=pa.PA_KV_E4M3, k_scale=0.0, v_scale=1.0)) == -1
    # E4M3 pools are served by the whole-group tensor kernel only
    assert call(pa.DecodeOptions(kv_dtype=pa.PA_KV_E4M3, k_scale=1.0, v_scale=1.0,
                                 kernel=pa.PA_KERNEL_SIMT)) == -2


def test_prefill_rejects_bad_arguments_without_a_gpu():
    lib = binding.lib
    fake = ctypes.c_void_p(0x10000)
    d = _desc()
    call = lambda n, mq, scale, dd, ws=fake, wsb=256, kernel=0: lib.pa_prefill(
        fake, fake, fake, fake, fake, fake, n, mq, ctypes.c_float(scale), fake, ws, wsb, ctypes.byref(dd), kernel,
        None)
    assert call(-1, 4, 0.1, d) == -1
    assert call(2, 4, 0.1, d, kernel=4) == -1            # unknown kernel
    assert call(2, 4, 0.1, _desc(block_size=24), kernel=pa.PA_PREFILL_TCGEN05_WS) == -2   # off the 64-key tile
    assert call(2, 4, 0.1, d, kernel=-1) == -1
    assert call(0, 4, 0.1, d, kernel=pa.PA_PREFILL_MMA) == 0
    # the binding refuses an unknown kernel name before it touches any buffer
    with pytest.raises(ValueError):
        pa.pa_prefill(None, None, None, None, None, np.zeros(2, np.int32), 4, 0.1, None, None, d,
                      kernel="wgmma")
    assert call(2, -1, 0.1, d) == -1
    assert call(2, 4, 0.0, d) == -1                      # scale must be > 0
    assert call(2, 4, 0.1, _desc(head_dim=96)) == -2
    assert call(0, 4, 0.1, d) == 0                        # nothing to do
    assert call(2, 0, 0.1, d) == 0
    assert call(2, 4, 0.1, d, ws=None) == -4              # workspace (status word) missing
    assert call(2, 4, 0.1, d, wsb=16) == -4


def test_slot_mapping_entry_matches_oracle():
    import oracle
    rng = np.random.default_rng(0)
    tables = rng.integers(0, 1000, size=(50, 20)).astype(np.int32)
    lens = rng.integers(0, 20 * 16 + 1, size=50).astype(np.int32)
    np.testing.assert_array_equal(pa.pa_slot_mapping(tables, lens, 16),
                                  oracle.slot_mapping(tables, lens, 16))
