"""Long-context parity on planted keys, through the C ABI (needs a B200).

On N(0,1) inputs a decode that loses a whole slab of a 32K+ context, or one of the merge's
piece groups, still meets the parity tolerance.  These cases plant dominant keys
(tests/planted.py) at the first, middle and last slab of every CTA slice of the decode's own
partition (read back with pa_decode_describe), and at both sides of every split edge for the
split kernels, so the exact answer of every query head moves by O(1) when any piece of the
work is lost.  tests/test_planted_oracle.py shows, on the CPU, that these inputs fail the
tolerance with one slab or one merge piece group cut out.

Bar: the parity tolerance (|gpu - oracle| <= 1e-2 + 1e-2 |oracle|) and, next to it, a tripwire
well inside it: |gpu - oracle| <= 2^-7 |oracle| + 2e-4.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
import pagedattention_kv_cache_pa_b200 as pa
from tests import planted as pl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests import gpu_harness
    return gpu_harness


def _planted(h, b, opts, max_len, split_tokens=0):
    """Plant keys for the partition this call will run; returns (planted batch, plan)."""
    (slots, tables, lens), _ = h.host_step(b)
    info = pa.pa_decode_describe(b.batch, max_len, h.desc_of(b), opts)
    if info.kernel == pa.PA_KERNEL_TENSOR:
        assert info.ctas > 0
        assert info.split_tokens in (16, 32)             # the stream kernel's slab
        pos = pl.stream_positions(lens, b.num_kv_heads, info.ctas, info.split_tokens)
    else:
        assert info.split_tokens == split_tokens and info.max_splits > 1
        pos = pl.split_positions(lens, b.num_kv_heads, info.split_tokens)
    plants = pl.assign(pos, b.batch, b.num_q_heads, b.num_kv_heads, lens)
    assert min(len(v) for v in plants.values()) >= 1
    return pl.plant(b, tables, lens, plants, copy=False), info


def _check(res):
    assert res["pool_equal"], "append is not bit-exact"
    assert res["finite"]
    assert res["ok"], "decode outside the parity tolerance by %g" % res["excess"]
    ok, worst = pl.tripwire(res["out"], res["ref"])
    assert ok, "decode outside the tripwire: worst error / bound = %g" % worst


@pytest.fixture(scope="module")
def c4_stream(h):
    b = wl.config4()
    opts = pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR)
    max_len = int(b.context_lens.max()) + 1
    pb, info = _planted(h, b, opts, max_len)
    return pb, info


@pytest.mark.parametrize("fused", [False, True], ids=["append+decode", "append_decode"])
def test_c4_planted_stream_kernel(h, c4_stream, fused):
    pb, info = c4_stream
    res = h.run_step(pb, kernel=pa.PA_KERNEL_TENSOR, fused=fused, pdl=fused)
    _check(res)


def test_c4_planted_stream_kernel_odd_grid(h):
    # a grid that is no multiple of the SM count (max_ctas caps the resident grid): slices
    # start mid-block everywhere and every sequence is cut into more, longer pieces
    b = wl.config4()
    max_len = int(b.context_lens.max()) + 1
    opts = pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR, max_ctas=97)
    pb, info = _planted(h, b, opts, max_len)
    assert info.ctas == 97
    _check(h.run_step(pb, kernel=pa.PA_KERNEL_TENSOR, max_ctas=97))


@pytest.mark.parametrize("kernel", [pa.PA_KERNEL_TENSOR_SPLIT, pa.PA_KERNEL_SIMT], ids=["split", "simt"])
def test_c4_planted_split_kernels(h, kernel):
    b = wl.config4()
    max_len = int(b.context_lens.max()) + 1
    opts = pa.DecodeOptions(kernel=kernel, split_tokens=1024)
    pb, _ = _planted(h, b, opts, max_len, split_tokens=1024)
    _check(h.run_step(pb, kernel=kernel, split_tokens=1024, fused=True))


KS = VS = 1.0 / 8   # planted K along its dim: 16 = code 128; planted V: 8 x N(0,1) stays < 448 / 8


def _e4m3_case(h, pb, fused, max_ctas=0):
    (slots, tables, lens), (o_slots, o_tables, o_lens) = h.host_step(pb)
    kq, vq = oracle.quantize_e4m3(pb.k_cache, KS), oracle.quantize_e4m3(pb.v_cache, VS)
    desc = h.desc_of(pb)
    kc, vc = torch.from_numpy(kq).to(h.DEV), torch.from_numpy(vq).to(h.DEV)
    q = h.to_dev(pb.q)
    out = torch.empty_like(q)
    max_len = int(lens.max())
    opts = pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR, kv_dtype=pa.PA_KV_E4M3, k_scale=KS, v_scale=VS,
                            max_ctas=max_ctas, flags=pa.PA_FLAG_CHECK)
    ws = torch.zeros(pa.pa_decode_workspace_size(pb.batch, max_len, desc, opts), dtype=torch.uint8,
                     device=h.DEV)
    tb, lb = torch.from_numpy(tables).to(h.DEV), torch.from_numpy(lens).to(h.DEV)
    if fused:
        pa.pa_append_decode(q, h.to_dev(pb.k_new), h.to_dev(pb.v_new), kc, vc, tb, lb, max_len, pb.scale,
                            out, ws, desc, opts)
    else:
        pa.pa_append_kv_e4m3(h.to_dev(pb.k_new), h.to_dev(pb.v_new), torch.from_numpy(slots).to(h.DEV),
                             KS, VS, kc, vc, desc)
        pa.pa_decode(q, kc, vc, tb, lb, max_len, pb.scale, out, ws, desc, opts)
    torch.cuda.synchronize()
    rk, rv = oracle.append_kv_e4m3(oracle.quantize_e4m3(pb.k_new, KS), oracle.quantize_e4m3(pb.v_new, VS),
                                   o_slots, kq, vq)
    pool_equal = np.array_equal(kc.cpu().numpy(), rk) and np.array_equal(vc.cpu().numpy(), rv)
    ref = oracle.paged_decode_e4m3(pb.q, rk, rv, KS, VS, o_tables, o_lens, pb.scale)
    got = out.float().cpu().numpy().astype(np.float64)
    ok, excess = oracle.within_tolerance(got, ref)
    return dict(pool_equal=pool_equal, finite=bool(np.isfinite(got).all()), ok=ok, excess=excess,
                out=got, ref=ref)


@pytest.mark.parametrize("fused", [False, True], ids=["append+decode", "append_decode"])
def test_c4_planted_e4m3(h, fused):
    b = wl.config4()
    max_len = int(b.context_lens.max()) + 1
    opts = pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR, kv_dtype=pa.PA_KV_E4M3, k_scale=KS, v_scale=VS)
    pb, _ = _planted(h, b, opts, max_len)
    _check(_e4m3_case(h, pb, fused))


def _c5_batch():
    t = wl.Trace5()
    return wl.make_batch("C5-batch", t.seed, t.initial_lens, num_q_heads=t.num_q_heads,
                         num_kv_heads=t.num_kv_heads, head_dim=t.head_dim, block_size=t.block_size)


@pytest.mark.parametrize("fused", [False, True], ids=["append+decode", "append_decode"])
def test_c5_batch_planted(h, fused):
    # 256 sequences of the trace's lognormal lengths (up to 16384): short sequences inside one
    # slice, long ones cut into many pieces and merged in 16 groups
    b = _c5_batch()
    max_len = int(b.context_lens.max()) + 1
    pb, info = _planted(h, b, pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR), max_len)
    _check(h.run_step(pb, kernel=pa.PA_KERNEL_TENSOR, fused=fused, pdl=fused))


def test_c5_batch_planted_e4m3(h):
    b = _c5_batch()
    max_len = int(b.context_lens.max()) + 1
    opts = pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR, kv_dtype=pa.PA_KV_E4M3, k_scale=KS, v_scale=VS)
    pb, _ = _planted(h, b, opts, max_len)
    _check(_e4m3_case(h, pb, True))
