"""Paged (chunked) prefill through the C ABI against the fp64 oracle (needs a B200).

The automatic choice and the single-issuer kernels (tcgen05 with tensor-memory accumulators,
warp-level mma.sync), each within 1e-2 + 1e-2 * |oracle|; cases: whole prompts (Tq = L), chunks after a cached
prefix (Tq < L), one-token chunks, lengths off the 64-key and 64/128-row tiles, GQA
groups 1..16, head dims 64 and 128, block sizes 8..256; errors reported through the
status word without a fault.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
import pagedattention_kv_cache_pa_b200 as pa

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests import gpu_harness
    return gpu_harness


KERNELS = ["auto", "tcgen05", "mma"]   # auto: the warp-specialized kernel where it serves the block size


def _run(h, seed, lens, q_lens, kernel="auto", mutate=None, **kw):
    b = wl.small_batch(seed, lens, **kw)
    if mutate is not None:
        mutate(b)
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q = (rng.standard_normal((int(cu[-1]), b.num_q_heads, b.head_dim)).astype(np.float32)
         .view(np.uint32) >> 16).astype(np.uint16)
    desc = h.desc_of(b)
    out = torch.full((int(cu[-1]), b.num_q_heads, b.head_dim), 9.0, dtype=torch.bfloat16, device=h.DEV)
    ws = torch.zeros(256, dtype=torch.uint8, device=h.DEV)
    pa.pa_prefill(h.to_dev(q), h.to_dev(b.k_cache), h.to_dev(b.v_cache), torch.from_numpy(b.block_tables).to(h.DEV),
                  torch.from_numpy(cu).to(h.DEV), torch.from_numpy(b.context_lens).to(h.DEV), max(q_lens),
                  b.scale, out, ws, desc, kernel=kernel)
    torch.cuda.synchronize()
    assert pa.pa_decode_status(ws) == 0
    ref = oracle.paged_prefill(q, b.k_cache, b.v_cache, b.block_tables, cu, b.context_lens, b.scale)
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    ok, ex = oracle.within_tolerance(got, ref)
    assert ok, "prefill outside tolerance by %g" % ex


# block sizes 8..256 that tile 64 keys (copied by TMA in the tcgen05 kernel) and 24, 4
# that do not (gathered with cp.async)
SHAPES = [(32, 8, 64, 16), (8, 8, 64, 8), (16, 1, 128, 16), (64, 8, 128, 32), (6, 3, 64, 256), (2, 2, 128, 64),
          (24, 8, 64, 16), (8, 2, 64, 24), (4, 4, 128, 4), (8, 1, 64, 128)]


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "Hq%d-Hkv%d-D%d-Bs%d" % s)
def test_prefill_shapes(h, shape, kernel):
    Hq, Hkv, D, Bs = shape
    lens = [1, 64, 65, 200, 333, 130]
    q_lens = [1, 64, 17, 200, 40, 1]                   # whole prompts, chunks, single tokens
    _run(h, 7000 + Hq + D + Bs, lens, q_lens, kernel=kernel, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
         block_size=Bs)


@pytest.mark.parametrize("kernel", KERNELS)
def test_prefill_llama_1b_prompt_and_chunk(h, kernel):
    _run(h, 7100, [2048, 1500], [2048, 700], kernel=kernel, num_q_heads=32, num_kv_heads=8, head_dim=64,
         block_size=16)


@pytest.mark.parametrize("kernel", KERNELS)
def test_prefill_head_dim_128_long_chunk(h, kernel):
    # several 128-row tiles and 64-key tiles with ragged ends, G = 4, blocks of 32
    _run(h, 7150, [1000, 777], [600, 777], kernel=kernel, num_q_heads=16, num_kv_heads=4, head_dim=128,
         block_size=32)


def _poison_unused_rows(b):
    """NaN (bf16 0x7FC0) in every pool row no sequence holds: free blocks and the tail of
    each sequence's last block.  The attention must not read them into the output."""
    used = np.zeros(b.k_cache.shape[0], dtype=bool)
    for s, L in enumerate(b.context_lens):
        nb = (int(L) + b.block_size - 1) // b.block_size
        used[b.block_tables[s, :nb]] = True
    for cache in (b.k_cache, b.v_cache):
        cache[~used] = 0x7FC0
        for s, L in enumerate(b.context_lens):
            L = int(L)
            if L % b.block_size:
                cache[b.block_tables[s, (L - 1) // b.block_size], :, L % b.block_size:, :] = 0x7FC0


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("Bs", [16, 24, 128])
def test_prefill_ignores_pool_rows_past_each_sequence(h, kernel, Bs):
    _run(h, 7300 + Bs, [37, 130, 64, 201], [37, 9, 64, 100], kernel=kernel, mutate=_poison_unused_rows,
         num_q_heads=8, num_kv_heads=2, head_dim=64, block_size=Bs)


@pytest.mark.parametrize("kernel", KERNELS)
def test_prefill_reports_bad_lengths_and_blocks(h, kernel):
    b = wl.small_batch(7200, [40, 20], num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16)
    desc = h.desc_of(b)
    q = torch.zeros((10, 4, 64), dtype=torch.bfloat16, device=h.DEV)
    out = torch.zeros_like(q)
    ws = torch.zeros(256, dtype=torch.uint8, device=h.DEV)
    cu = torch.tensor([0, 5, 10], dtype=torch.int32, device=h.DEV)
    lens = torch.tensor([40, 3], dtype=torch.int32, device=h.DEV)      # second: fewer tokens than queries
    kc, vc = h.to_dev(b.k_cache), h.to_dev(b.v_cache)
    tables = torch.from_numpy(b.block_tables).to(h.DEV)
    pa.pa_prefill(q, kc, vc, tables, cu, lens, 5, b.scale, out, ws, desc, kernel=kernel)
    torch.cuda.synchronize()
    assert pa.pa_decode_status(ws) == -8
    bad = b.block_tables.copy()
    bad[0, 1] = b.num_blocks + 5
    lens = torch.tensor([40, 20], dtype=torch.int32, device=h.DEV)
    pa.pa_prefill(q, kc, vc, torch.from_numpy(bad).to(h.DEV), cu, lens, 5, b.scale, out, ws, desc, kernel=kernel)
    torch.cuda.synchronize()
    assert pa.pa_decode_status(ws) == -7


@pytest.mark.parametrize("kernel", KERNELS)
def test_prefill_many_sequences_mixed_lengths(h, kernel):
    # more than 32 sequences (the work-item search walks them 32 at a time), with empty
    # chunks, single tokens, whole prompts and chunks after long caches mixed
    rng = np.random.default_rng(7400)
    q_lens = [int(x) for x in rng.choice([0, 1, 3, 64, 129, 300], size=70)]
    lens = [t + int(rng.choice([0, 5, 200, 900])) for t in q_lens]
    lens = [max(L, 1) for L in lens]
    _run(h, 7401, lens, q_lens, kernel=kernel, num_q_heads=16, num_kv_heads=4, head_dim=64, block_size=16)


@pytest.mark.parametrize("kernel", KERNELS)
def test_prefill_reports_more_queries_than_max_q_len(h, kernel):
    b = wl.small_batch(7500, [40, 30], num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16)
    desc = h.desc_of(b)
    q = torch.zeros((30, 4, 64), dtype=torch.bfloat16, device=h.DEV)
    out = torch.zeros_like(q)
    ws = torch.zeros(256, dtype=torch.uint8, device=h.DEV)
    cu = torch.tensor([0, 10, 30], dtype=torch.int32, device=h.DEV)       # second: 20 queries
    lens = torch.tensor([40, 30], dtype=torch.int32, device=h.DEV)
    pa.pa_prefill(q, h.to_dev(b.k_cache), h.to_dev(b.v_cache), torch.from_numpy(b.block_tables).to(h.DEV), cu,
                  lens, 10, b.scale, out, ws, desc, kernel=kernel)
    torch.cuda.synchronize()
    assert pa.pa_decode_status(ws) == -8
