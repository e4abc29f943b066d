"""Warp-specialized tcgen05 prefill (PA_PREFILL_TCGEN05_WS) against the fp64 oracle, and the
chunked-prefill workload the bench times at its full size, for every tensor-core kernel
(needs a B200).

The same cases as tests/test_gpu_prefill.py for the block sizes this kernel serves (8, 16,
32, 64 or multiples of 64), within 1e-2 + 1e-2 * |oracle|; the full-size workload (4
sequences, 2048 new tokens each after 0/512/1024/1536 cached ones, Llama-3.2-1B attention
shape) is compared on windows of 64 consecutive queries at the start, middle and end of every
chunk, which the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
import pagedattention_kv_cache_pa_b200 as pa
from tests.test_gpu_prefill import SHAPES, _poison_unused_rows, _run

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests import gpu_harness
    return gpu_harness


WS_SHAPES = [s for s in SHAPES if s[3] % 64 == 0 or (s[3] >= 8 and 64 % s[3] == 0)]


@pytest.mark.parametrize("shape", WS_SHAPES, ids=lambda s: "Hq%d-Hkv%d-D%d-Bs%d" % s)
def test_ws_prefill_shapes(h, shape):
    Hq, Hkv, D, Bs = shape
    _run(h, 7000 + Hq + D + Bs, [1, 64, 65, 200, 333, 130], [1, 64, 17, 200, 40, 1], kernel="tcgen05_ws",
         num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, block_size=Bs)


def test_ws_prefill_llama_1b_prompt_and_chunk(h):
    _run(h, 7100, [2048, 1500], [2048, 700], kernel="tcgen05_ws", num_q_heads=32, num_kv_heads=8, head_dim=64,
         block_size=16)


def test_ws_prefill_head_dim_128_long_chunk(h):
    _run(h, 7150, [1000, 777], [600, 777], kernel="tcgen05_ws", num_q_heads=16, num_kv_heads=4, head_dim=128,
         block_size=32)


def test_ws_prefill_large_scores_rescale(h):
    # q scaled by 8: scores spread over tens of log2 units, so rows raise their running max
    # by more than the rescale threshold many times
    b = wl.small_batch(7170, [900, 300], num_q_heads=8, num_kv_heads=2, head_dim=64, block_size=16)
    rng = np.random.default_rng(7170)
    cu = np.array([0, 500, 800], dtype=np.int32)
    qf = rng.standard_normal((800, 8, 64)).astype(np.float32) * 8
    q = (qf.view(np.uint32) >> 16).astype(np.uint16)
    out = torch.zeros((800, 8, 64), dtype=torch.bfloat16, device=h.DEV)
    ws = torch.zeros(256, dtype=torch.uint8, device=h.DEV)
    pa.pa_prefill(h.to_dev(q), h.to_dev(b.k_cache), h.to_dev(b.v_cache), torch.from_numpy(b.block_tables).to(h.DEV),
                  torch.from_numpy(cu).to(h.DEV), torch.from_numpy(b.context_lens).to(h.DEV), 500, b.scale, out, ws,
                  h.desc_of(b), kernel="tcgen05_ws")
    torch.cuda.synchronize()
    assert pa.pa_decode_status(ws) == 0
    ref = oracle.paged_prefill(q, b.k_cache, b.v_cache, b.block_tables, cu, b.context_lens, b.scale)
    ok, ex = oracle.within_tolerance(out.float().cpu().numpy(), ref)
    assert ok, ex


@pytest.mark.parametrize("Bs", [16, 128])
def test_ws_prefill_ignores_pool_rows_past_each_sequence(h, Bs):
    _run(h, 7300 + Bs, [37, 130, 64, 201], [37, 9, 64, 100], kernel="tcgen05_ws", mutate=_poison_unused_rows,
         num_q_heads=8, num_kv_heads=2, head_dim=64, block_size=Bs)


def test_ws_prefill_reports_bad_lengths_and_blocks(h):
    b = wl.small_batch(7200, [40, 20], num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16)
    desc = h.desc_of(b)
    q = torch.zeros((10, 4, 64), dtype=torch.bfloat16, device=h.DEV)
    out = torch.zeros_like(q)
    ws = torch.zeros(256, dtype=torch.uint8, device=h.DEV)
    cu = torch.tensor([0, 5, 10], dtype=torch.int32, device=h.DEV)
    kc, vc = h.to_dev(b.k_cache), h.to_dev(b.v_cache)
    pa.pa_prefill(q, kc, vc, torch.from_numpy(b.block_tables).to(h.DEV), cu,
                  torch.tensor([40, 3], dtype=torch.int32, device=h.DEV), 5, b.scale, out, ws, desc,
                  kernel="tcgen05_ws")
    torch.cuda.synchronize()
    assert pa.pa_decode_status(ws) == -8
    bad = b.block_tables.copy()
    bad[0, 1] = b.num_blocks + 5
    pa.pa_prefill(q, kc, vc, torch.from_numpy(bad).to(h.DEV), cu, torch.tensor([40, 20], dtype=torch.int32,
                  device=h.DEV), 5, b.scale, out, ws, desc, kernel="tcgen05_ws")
    torch.cuda.synchronize()
    assert pa.pa_decode_status(ws) == -7


def test_ws_prefill_refuses_block_sizes_off_the_tile(h):
    b = wl.small_batch(7210, [40], num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=24)
    q = torch.zeros((4, 4, 64), dtype=torch.bfloat16, device=h.DEV)
    with pytest.raises(pa.PaError) as e:
        pa.pa_prefill(q, h.to_dev(b.k_cache), h.to_dev(b.v_cache), torch.from_numpy(b.block_tables).to(h.DEV),
                      torch.tensor([0, 4], dtype=torch.int32, device=h.DEV),
                      torch.from_numpy(b.context_lens).to(h.DEV), 4, b.scale, torch.zeros_like(q),
                      torch.zeros(256, dtype=torch.uint8, device=h.DEV), h.desc_of(b), kernel="tcgen05_ws")
    assert e.value.status == -2


PF_CACHED, PF_NEW = [0, 512, 1024, 1536], 2048


@pytest.fixture(scope="module")
def pf(h):
    """The chunked-prefill workload the bench times: the chunk's K/V appended through the
    library (checked bit-exact against the oracle's append), then attention."""
    lens = [c + PF_NEW for c in PF_CACHED]
    b = wl.make_batch("PF", wl.CONFIG_SEED_BASE + 41, [L - 1 for L in lens], num_q_heads=32, num_kv_heads=8,
                      head_dim=64, block_size=16)
    rng = np.random.default_rng(wl.CONFIG_SEED_BASE + 42)
    T = PF_NEW * len(lens)
    bits = lambda shape: (rng.standard_normal(shape).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    q, k, v = bits((T, 32, 64)), bits((T, 8, 64)), bits((T, 8, 64))
    Bs = b.block_size
    slots = np.concatenate([[int(b.block_tables[s][p // Bs]) * Bs + p % Bs for p in range(L - PF_NEW, L)]
                            for s, L in enumerate(lens)]).astype(np.int64)
    cu = np.arange(0, T + 1, PF_NEW, dtype=np.int32)
    kc, vc = h.to_dev(b.k_cache), h.to_dev(b.v_cache)
    pa.pa_append_kv(h.to_dev(k), h.to_dev(v), torch.from_numpy(slots).to(h.DEV), kc, vc, h.desc_of(b))
    torch.cuda.synchronize()
    rk, rv = oracle.append_kv(k, v, slots, b.k_cache, b.v_cache)
    assert np.array_equal(h.to_host_bits(kc), rk) and np.array_equal(h.to_host_bits(vc), rv)
    return dict(b=b, lens=np.array(lens, np.int32), q=q, cu=cu, kc=kc, vc=vc, rk=rk, rv=rv)


@pytest.mark.parametrize("kernel", ["tcgen05_ws", "tcgen05", "mma"])
def test_pf_workload_full_size(h, pf, kernel):
    b = pf["b"]
    out = torch.full((pf["q"].shape[0], 32, 64), 9.0, dtype=torch.bfloat16, device=h.DEV)
    ws = torch.zeros(256, dtype=torch.uint8, device=h.DEV)
    pa.pa_prefill(h.to_dev(pf["q"]), pf["kc"], pf["vc"], torch.from_numpy(b.block_tables).to(h.DEV),
                  torch.from_numpy(pf["cu"]).to(h.DEV), torch.from_numpy(pf["lens"]).to(h.DEV), PF_NEW, b.scale,
                  out, ws, h.desc_of(b), kernel=kernel)
    torch.cuda.synchronize()
    assert pa.pa_decode_status(ws) == 0
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    for s, L in enumerate(pf["lens"]):
        for w in (0, PF_NEW // 128 - 1, PF_NEW // 64 - 1):     # first, middle and last 64 queries
            rows = slice(int(pf["cu"][s]) + 64 * w, int(pf["cu"][s]) + 64 * (w + 1))
            end = int(L) - PF_NEW + 64 * (w + 1)                 # the window's queries end at position end - 1
            ref = oracle.paged_prefill(pf["q"][rows], pf["rk"], pf["rv"], b.block_tables[s:s + 1],
                                       np.array([0, 64], np.int32), np.array([end], np.int32), b.scale)
            ok, ex = oracle.within_tolerance(got[rows], ref)
            assert ok, "sequence %d window %d outside tolerance by %g" % (s, w, ex)
