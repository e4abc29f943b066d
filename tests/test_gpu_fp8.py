"""FP8 (E4M3) KV cache through the C ABI against the fp64 oracle (needs a B200).

Quantized appends must produce the oracle's codes bit for bit (the code is an
integer decided by one float product and a nearest-even rounding, which both
sides take in float), and touch no other byte.  Decodes over E4M3 pools are
compared with the oracle's fp64 attention over the same codes (values = code
value * scale) within 1e-2 + 1e-2 * |oracle|.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
import pagedattention_kv_cache_pa_b200 as pa

pytestmark = pytest.mark.gpu

SCALES = [(5.0 / 448, 5.0 / 448), (1.0 / 64, 0.37), (0.37, 1.0 / 64)]


@pytest.fixture(scope="module")
def h():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests import gpu_harness
    return gpu_harness


def _u8(a, h):
    return torch.from_numpy(np.ascontiguousarray(a)).to(h.DEV)


def _pools(b, ks, vs):
    return oracle.quantize_e4m3(b.k_cache, ks), oracle.quantize_e4m3(b.v_cache, vs)


@pytest.mark.parametrize("ks,vs", SCALES)
@pytest.mark.parametrize("cfg", ["c2", "c4"])
def test_append_e4m3_codes_bit_exact(h, cfg, ks, vs):
    b = wl.CONFIGS[cfg]()
    (slots, _, _), (o_slots, _, _) = h.host_step(b)
    kq, vq = _pools(b, ks, vs)
    kc, vc = _u8(kq, h), _u8(vq, h)
    pa.pa_append_kv_e4m3(h.to_dev(b.k_new), h.to_dev(b.v_new), torch.from_numpy(slots).to(h.DEV), ks, vs,
                         kc, vc, h.desc_of(b))
    torch.cuda.synchronize()
    want_k, want_v = oracle.append_kv_e4m3(oracle.quantize_e4m3(b.k_new, ks), oracle.quantize_e4m3(b.v_new, vs),
                                           o_slots, kq, vq)
    np.testing.assert_array_equal(kc.cpu().numpy(), want_k)
    np.testing.assert_array_equal(vc.cpu().numpy(), want_v)


def test_append_e4m3_extremes(h):
    # saturation, subnormals, signed zero, ties: rows built from chosen bf16 values
    b = wl.small_batch(81, [5], num_q_heads=8, num_kv_heads=8, head_dim=64, block_size=16)
    vals = np.array([0.0, -0.0, 1.0, -1.0, 448.0, 449.0, 1e6, -1e6, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -10,
                     1.0625, 1.1875, 0.3, -7.5, 300.0], dtype=np.float32)
    bits = (np.resize(vals, b.k_new.size).view(np.uint32) >> 16).astype(np.uint16).reshape(b.k_new.shape)
    kq, vq = np.zeros_like(b.k_cache, dtype=np.uint8), np.zeros_like(b.v_cache, dtype=np.uint8)
    kc, vc = _u8(kq, h), _u8(vq, h)
    slots = np.array([7], dtype=np.int64)
    pa.pa_append_kv_e4m3(h.to_dev(bits), h.to_dev(bits), torch.from_numpy(slots).to(h.DEV), 1.0, 0.5,
                         kc, vc, h.desc_of(b))
    torch.cuda.synchronize()
    want_k, want_v = oracle.append_kv_e4m3(oracle.quantize_e4m3(bits, 1.0), oracle.quantize_e4m3(bits, 0.5),
                                           slots, kq, vq)
    np.testing.assert_array_equal(kc.cpu().numpy(), want_k)
    np.testing.assert_array_equal(vc.cpu().numpy(), want_v)


def _decode_case(h, b, ks, vs, *, max_ctas=0, pdl=False, fused=False):
    (slots, tables, lens), (o_slots, o_tables, o_lens) = h.host_step(b)
    kq, vq = _pools(b, ks, vs)
    desc = h.desc_of(b)
    kc, vc = _u8(kq, h), _u8(vq, h)
    q = h.to_dev(b.q)
    out = torch.empty_like(q)
    max_len = int(lens.max())
    opts = pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR, kv_dtype=pa.PA_KV_E4M3, k_scale=ks, v_scale=vs,
                            max_ctas=max_ctas, flags=pa.PA_FLAG_CHECK | (pa.PA_FLAG_PDL if pdl else 0))
    ws = torch.zeros(pa.pa_decode_workspace_size(b.batch, max_len, desc, opts), dtype=torch.uint8,
                     device=h.DEV)
    tb, lb = torch.from_numpy(tables).to(h.DEV), torch.from_numpy(lens).to(h.DEV)
    if fused:
        pa.pa_append_decode(q, h.to_dev(b.k_new), h.to_dev(b.v_new), kc, vc, tb, lb, max_len, b.scale, out,
                            ws, desc, opts)
    else:
        pa.pa_append_kv_e4m3(h.to_dev(b.k_new), h.to_dev(b.v_new), torch.from_numpy(slots).to(h.DEV), ks, vs,
                             kc, vc, desc)
        pa.pa_decode(q, kc, vc, tb, lb, max_len, b.scale, out, ws, desc, opts)
    torch.cuda.synchronize()
    rk, rv = oracle.append_kv_e4m3(oracle.quantize_e4m3(b.k_new, ks), oracle.quantize_e4m3(b.v_new, vs),
                                   o_slots, kq, vq)
    np.testing.assert_array_equal(kc.cpu().numpy(), rk)
    np.testing.assert_array_equal(vc.cpu().numpy(), rv)
    ref = oracle.paged_decode_e4m3(b.q, rk, rv, ks, vs, o_tables, o_lens, b.scale)
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    ok, ex = oracle.within_tolerance(got, ref)
    assert ok, "decode outside tolerance by %g" % ex


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
@pytest.mark.parametrize("cfg", ["c2", "c3", "c4"])
def test_decode_e4m3(h, cfg, fused):
    ks, vs = SCALES[0]
    _decode_case(h, wl.CONFIGS[cfg](), ks, vs, fused=fused)


@pytest.mark.parametrize("ks,vs", SCALES[1:])
@pytest.mark.parametrize("ctas,pdl", [(1, False), (5, True), (64, False)])
def test_decode_e4m3_partitions_and_scales(h, ks, vs, ctas, pdl):
    _decode_case(h, wl.config2(), ks, vs, max_ctas=ctas, pdl=pdl, fused=True)


FP8_SHAPES = [(8, 8, 64, 8), (16, 8, 128, 16), (64, 8, 128, 16), (128, 8, 64, 16), (32, 16, 64, 32),
              (24, 8, 64, 256), (96, 8, 128, 32)]


@pytest.mark.parametrize("shape", FP8_SHAPES, ids=lambda s: "Hq%d-Hkv%d-D%d-Bs%d" % s)
def test_decode_e4m3_shapes(h, shape):
    Hq, Hkv, D, Bs = shape
    lens = sorted({0, 1, Bs - 1, Bs, 62, 63, 64, 65, 127, 128, 129, 300, 777})
    b = wl.small_batch(5000 + Bs + D + Hq, lens, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, block_size=Bs)
    for ctas, fused in ((0, False), (3, True), (17, False)):
        _decode_case(h, b, 5.0 / 448, 0.02, max_ctas=ctas, fused=fused)


# lengths on both sides of every 32-token stage boundary up to a few stages, and past 1024
SLAB_LENS = sorted({0, 1, 2, 31, 32, 33, 63, 64, 65, 95, 96, 97, 159, 160, 161, 255, 256, 257, 1023,
                    1024, 1025})


@pytest.mark.parametrize("Bs", [8, 16, 32, 64])
@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_decode_e4m3_32_token_stages(h, Bs, G):
    """E4M3 pools at head_dim 64 stream K/V in 32-token stages (two bf16-sized 16-token slabs
    per stage): block sizes below, at and above the stage size, every GQA group the kernel
    takes, lengths on both sides of each stage boundary; direct, partitioned and fused."""
    Hkv = 8
    b = wl.small_batch(7100 + Bs * 32 + G, SLAB_LENS, num_q_heads=Hkv * G, num_kv_heads=Hkv, head_dim=64,
                       block_size=Bs)
    opts = pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR, kv_dtype=pa.PA_KV_E4M3, k_scale=0.02, v_scale=0.02)
    plan = pa.pa_decode_describe(b.batch, int(b.context_lens.max()) + 1, h.desc_of(b), opts)
    assert plan.split_tokens == 32
    for ctas, fused, pdl in ((0, True, True), (7, False, False), (40, True, False)):
        _decode_case(h, b, 5.0 / 448, 0.03, max_ctas=ctas, pdl=pdl, fused=fused)


@pytest.mark.parametrize("D,want", [(64, 32), (128, 16)])
def test_e4m3_stage_size_reported(h, D, want):
    """pa_decode_describe reports the stream kernel's stage: 32 tokens for E4M3 at head_dim 64,
    16 otherwise (and 16 for bf16 pools at either head_dim)."""
    b = wl.small_batch(7300 + D, [100, 200], num_q_heads=32, num_kv_heads=8, head_dim=D, block_size=16)
    f8 = pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR, kv_dtype=pa.PA_KV_E4M3, k_scale=0.02, v_scale=0.02)
    bf = pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR)
    assert pa.pa_decode_describe(2, 201, h.desc_of(b), f8).split_tokens == want
    assert pa.pa_decode_describe(2, 201, h.desc_of(b), bf).split_tokens == 16


def test_e4m3_unsupported_combinations(h):
    b = wl.config1()                                     # Hkv = 1: no whole-group kernel
    desc = h.desc_of(b)
    q = h.to_dev(b.q)
    kc = torch.zeros(b.k_cache.size, dtype=torch.uint8, device=h.DEV)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device=h.DEV)
    opts = pa.DecodeOptions(kv_dtype=pa.PA_KV_E4M3, k_scale=1.0, v_scale=1.0)
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode(q, kc, kc, torch.from_numpy(b.block_tables).to(h.DEV),
                     torch.from_numpy(b.context_lens).to(h.DEV), 40, b.scale, torch.empty_like(q), ws, desc,
                     opts)
    assert e.value.status == -2
    opts = pa.DecodeOptions(kernel=pa.PA_KERNEL_SIMT, kv_dtype=pa.PA_KV_E4M3, k_scale=1.0, v_scale=1.0)
    b2 = wl.config2()                                    # the CUDA-core kernel reads bf16 pools only
    kc2 = torch.zeros(b2.k_cache.size, dtype=torch.uint8, device=h.DEV)
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode(h.to_dev(b2.q), kc2, kc2, torch.from_numpy(b2.block_tables).to(h.DEV),
                     torch.from_numpy(b2.context_lens).to(h.DEV), 2048, b2.scale,
                     torch.empty_like(h.to_dev(b2.q)), ws, h.desc_of(b2), opts)
    assert e.value.status == -2


def _bf16_neighbours(bits):
    """The bf16 patterns one unit in the last place below and above each pattern."""
    x = np.asarray(bits, dtype=np.uint16).astype(np.int32)
    o = np.where(x & 0x8000, -(x & 0x7FFF), x & 0x7FFF)          # ordered integer line
    back = lambda v: np.where(v < 0, 0x8000 | (-v), v).astype(np.uint16)
    return back(o - 1), back(o + 1)


def _rope_codes_allowed(gpu_rows, k_new, positions, theta, ks):
    """Each E4M3 code of a rotated K row must be the code of a bf16 value within RoPE's bar
    (2^-8 |exact| + 2^-20 (|x_i| + |x_i+D/2|)) of the exact rotation: the rounded value or a
    neighbour inside the bar.  Returns the fraction of codes that differ from the oracle's."""
    exact = oracle.rope(k_new, positions, theta)
    x = (k_new.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    half = x.shape[-1] // 2
    mag = np.abs(x[..., :half]) + np.abs(x[..., half:])
    bound = 2.0 ** -8 * np.abs(exact) + 2.0 ** -20 * np.concatenate([mag, mag], axis=-1)
    r0 = oracle.round_bf16(exact)
    lo, hi = _bf16_neighbours(r0)
    widen = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    allowed = gpu_rows == oracle.quantize_e4m3(r0, ks)
    for c in (lo, hi):
        allowed |= (np.abs(widen(c) - exact) <= bound) & (gpu_rows == oracle.quantize_e4m3(c, ks))
    assert allowed.all(), "a rotated K code no bf16 value within the bar quantizes to"
    return float(np.mean(gpu_rows != oracle.quantize_e4m3(r0, ks)))


@pytest.mark.parametrize("cfg,ctas,pdl", [("c2", 0, True), ("c3", 0, False), ("c4", 0, True),
                                          ("c2", 7, False)])
def test_rope_append_decode_e4m3(h, cfg, ctas, pdl):
    """RoPE on E4M3 pools: q and the new K turned at position L-1 and rounded to bf16, the K row
    quantized from that bf16 row; against oracle.rope_bf16 then oracle.quantize_e4m3."""
    theta, ks, vs = 500000.0, 5.0 / 448, 5.0 / 448
    b = wl.CONFIGS[cfg]()
    (slots, tables, lens), (o_slots, o_tables, o_lens) = h.host_step(b)
    kq, vq = _pools(b, ks, vs)
    desc = h.desc_of(b)
    kc, vc = _u8(kq, h), _u8(vq, h)
    q = h.to_dev(b.q)
    out = torch.empty_like(q)
    max_len = int(lens.max())
    opts = pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR, kv_dtype=pa.PA_KV_E4M3, k_scale=ks, v_scale=vs,
                            max_ctas=ctas, rope_theta=theta,
                            flags=pa.PA_FLAG_CHECK | (pa.PA_FLAG_PDL if pdl else 0))
    ws = torch.zeros(pa.pa_decode_workspace_size(b.batch, max_len, desc, opts), dtype=torch.uint8,
                     device=h.DEV)
    pa.pa_append_decode(q, h.to_dev(b.k_new), h.to_dev(b.v_new), kc, vc, torch.from_numpy(tables).to(h.DEV),
                        torch.from_numpy(lens).to(h.DEV), max_len, b.scale, out, ws, desc, opts)
    torch.cuda.synchronize()
    pos = np.maximum(o_lens - 1, 0).astype(np.int32)
    q_rot = oracle.rope_bf16(b.q, pos, theta)
    k_rot = oracle.rope_bf16(b.k_new, pos, theta)
    rk, rv = oracle.append_kv_e4m3(oracle.quantize_e4m3(k_rot, ks), oracle.quantize_e4m3(b.v_new, vs),
                                   o_slots, kq, vq)
    got_k, got_v = kc.cpu().numpy(), vc.cpu().numpy()
    np.testing.assert_array_equal(got_v, rv)
    # K: every byte outside the new rows identical; the new rows within the rounding bar
    mask = h.pool_rows(kq.shape, o_slots)
    np.testing.assert_array_equal(got_k[~mask], rk[~mask])
    Bs = b.block_size
    rows = np.stack([got_k[s // Bs, :, s % Bs, :] for s in o_slots])
    differ = _rope_codes_allowed(rows, b.k_new, pos, theta, ks)
    assert differ < 0.01
    ref = oracle.paged_decode_e4m3(q_rot, rk, rv, ks, vs, o_tables, o_lens, b.scale)
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    ok, ex = oracle.within_tolerance(got, ref)
    assert ok, "decode outside tolerance by %g" % ex
