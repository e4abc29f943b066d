"""RoPE fused with the KV append, through the C ABI, against the fp64 oracle (needs a B200).

Rotated rows (q and the cached K) are compared with the oracle's unrounded
fp64 rotation: each value within 2^-8 of its magnitude (its bf16 rounding,
with one ulp of slack) plus 2^-20 of the pair's input magnitude.  The kernels
take cos/sin in float of an angle reduced in double and rotate in float, so
where the rotation cancels (a tiny result from large inputs) the absolute term
dominates; a relative-only bar would not be met there by any float kernel.
Every other byte of the pool must be identical, V rows included.  Decode
outputs on the rotated cache follow the attention tolerance 1e-2 + 1e-2 * |oracle|.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
import pagedattention_kv_cache_pa_b200 as pa

pytestmark = pytest.mark.gpu

KERNELS = [pa.PA_KERNEL_SIMT, pa.PA_KERNEL_TENSOR, pa.PA_KERNEL_TENSOR_SPLIT]
KNAMES = {pa.PA_KERNEL_SIMT: "simt", pa.PA_KERNEL_TENSOR: "tensor",
          pa.PA_KERNEL_TENSOR_SPLIT: "split"}
THETAS = [10000.0, 500000.0]


@pytest.fixture(scope="module")
def h():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests import gpu_harness
    return gpu_harness


def _rope_append_case(h, b, theta, in_place):
    (slots, tables, lens), (o_slots, o_tables, o_lens) = h.host_step(b)
    positions = np.maximum(lens - 1, 0).astype(np.int32)
    desc = h.desc_of(b)
    kc, vc = h.to_dev(b.k_cache), h.to_dev(b.v_cache)
    q = h.to_dev(b.q)
    q_out = q if in_place else torch.empty_like(q)
    pa.pa_rope_append_kv(q, q_out, h.to_dev(b.k_new), h.to_dev(b.v_new),
                         torch.from_numpy(positions).to(h.DEV), torch.from_numpy(slots).to(h.DEV),
                         theta, kc, vc, desc)
    torch.cuda.synchronize()
    q_ref = oracle.rope_bf16(b.q, positions, theta)
    got_q = h.to_host_bits(q_out)
    ok, worst = h.rope_close(got_q, b.q, positions, theta)
    assert ok, "rotated q outside the bound (worst %.3g of it)" % worst
    assert h.rope_pool_matches(h.to_host_bits(kc), b.k_cache, b.k_new, o_slots, positions, theta), \
        "rotated K rows outside the bound, or another byte changed"
    _, ref_v = oracle.append_kv(b.k_new, b.v_new, o_slots, b.k_cache, b.v_cache)
    np.testing.assert_array_equal(h.to_host_bits(vc), ref_v)
    return float((got_q == q_ref).mean())


@pytest.mark.parametrize("theta", THETAS)
@pytest.mark.parametrize("cfg", ["c1", "c2", "c4"])
def test_rope_append_kv_matches_oracle(h, cfg, theta):
    exact = _rope_append_case(h, wl.CONFIGS[cfg](), theta, in_place=False)
    assert exact > 0.95, "only %.3f of rotated q values bit-identical" % exact


def test_rope_append_kv_in_place(h):
    _rope_append_case(h, wl.config2(), 10000.0, in_place=True)


def test_rope_append_kv_skips_negative_slots_but_rotates_q(h):
    b = wl.small_batch(61, [40, 9, 100], num_q_heads=8, num_kv_heads=2, head_dim=128)
    desc = h.desc_of(b)
    kc, vc = h.to_dev(b.k_cache), h.to_dev(b.v_cache)
    q = h.to_dev(b.q)
    q_out = torch.empty_like(q)
    slots = np.array([-1, 5, b.num_blocks * b.block_size], dtype=np.int64)   # skip, write, past pool
    positions = np.array([40, 9, 100], dtype=np.int32)
    pa.pa_rope_append_kv(q, q_out, h.to_dev(b.k_new), h.to_dev(b.v_new),
                         torch.from_numpy(positions).to(h.DEV), torch.from_numpy(slots).to(h.DEV),
                         10000.0, kc, vc, desc)
    torch.cuda.synchronize()
    assert h.rope_close(h.to_host_bits(q_out), b.q, positions, 10000.0)[0]
    assert h.rope_pool_matches(h.to_host_bits(kc), b.k_cache, b.k_new, slots, positions, 10000.0)
    _, ref_v = oracle.append_kv(b.k_new, b.v_new, slots, b.k_cache, b.v_cache)
    np.testing.assert_array_equal(h.to_host_bits(vc), ref_v)


@pytest.mark.parametrize("kernel", KERNELS, ids=KNAMES.get)
@pytest.mark.parametrize("cfg", ["c1", "c2", "c3", "c4"])
def test_rope_append_decode(h, kernel, cfg):
    res = h.run_step(wl.CONFIGS[cfg](), kernel=kernel, fused=True, rope_theta=500000.0)
    assert res["pool_equal"], "rotated append outside the bound, or another byte changed"
    assert res["finite"]
    assert res["ok"], "decode outside tolerance by %g" % res["excess"]


ROPE_SHAPES = [(32, 8, 64, 16), (16, 8, 128, 8), (128, 8, 64, 256), (64, 8, 128, 32), (8, 1, 128, 16),
               (6, 3, 64, 64)]


@pytest.mark.parametrize("kernel", KERNELS, ids=KNAMES.get)
@pytest.mark.parametrize("shape", ROPE_SHAPES, ids=lambda s: "Hq%d-Hkv%d-D%d-Bs%d" % s)
def test_rope_append_decode_shapes(h, kernel, shape):
    Hq, Hkv, D, Bs = shape
    lens = sorted({0, 1, Bs - 1, Bs, 63, 64, 65, 300, 777, 5000})
    b = wl.small_batch(3000 + Bs + D + Hq, lens, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                       block_size=Bs)
    for ctas, pdl in ((0, False), (7, True)):
        res = h.run_step(b, kernel=kernel, fused=True, max_ctas=ctas, pdl=pdl, rope_theta=10000.0)
        assert res["pool_equal"] and res["finite"]
        assert res["ok"], "decode outside tolerance by %g" % res["excess"]


def test_rope_rejected_without_new_token(h):
    b = wl.config1()
    desc = h.desc_of(b)
    q = h.to_dev(b.q)
    opts = pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR, rope_theta=10000.0)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device=h.DEV)
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode(q, h.to_dev(b.k_cache), h.to_dev(b.v_cache),
                     torch.from_numpy(b.block_tables).to(h.DEV),
                     torch.from_numpy(b.context_lens).to(h.DEV), int(b.context_lens.max()), b.scale,
                     torch.empty_like(q), ws, desc, opts)
    assert e.value.status == -1
