"""CUDA path vs fp64 oracle through the C ABI (needs a B200).

Append: bit-exact, everywhere in the pool.  Decode: |gpu - oracle| <= 1e-2 +
1e-2 * |oracle| elementwise (the tolerance the workload statement fixes).
Both decode kernels (CUDA-core and tensor-core) are checked on every case.
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


@pytest.fixture(scope="module")
def h():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests import gpu_harness
    return gpu_harness


def _assert(res):
    assert res["pool_equal"], "append is not bit-exact"
    assert res["finite"]
    assert res["ok"], "decode outside tolerance by %g" % res["excess"]


@pytest.mark.parametrize("kernel", KERNELS, ids=KNAMES.get)
def test_c1_tiny(h, kernel):
    _assert(h.run_step(wl.config1(), kernel=kernel))


@pytest.mark.parametrize("kernel", KERNELS, ids=KNAMES.get)
@pytest.mark.parametrize("split", [0, 64, 256])
def test_c2_llama_1b_layer(h, kernel, split):
    res = h.run_step(wl.config2(), kernel=kernel, split_tokens=split)
    _assert(res)


@pytest.mark.parametrize("kernel", KERNELS, ids=KNAMES.get)
@pytest.mark.parametrize("cfg", ["c1", "c2", "c3", "c4"])
def test_fused_append_decode(h, kernel, cfg):
    # pa_append_decode: the append through the table inside the decode call
    _assert(h.run_step(wl.CONFIGS[cfg](), kernel=kernel, fused=True))


@pytest.mark.parametrize("ctas", [1, 2, 5, 64, 1000])
def test_c2_stream_partitions(h, ctas):
    # the tensor kernel's slices of the token stream: one CTA (no merge), a few (long
    # merges), many (every sequence cut several times)
    _assert(h.run_step(wl.config2(), kernel=pa.PA_KERNEL_TENSOR, max_ctas=ctas))


@pytest.mark.parametrize("kernel", KERNELS, ids=KNAMES.get)
def test_c3_shared_prefix_bs256(h, kernel):
    _assert(h.run_step(wl.config3(), kernel=kernel))


@pytest.mark.parametrize("kernel", KERNELS, ids=KNAMES.get)
def test_c4_long_context_split(h, kernel):
    res = h.run_step(wl.config4(), kernel=kernel)
    if kernel != pa.PA_KERNEL_TENSOR:        # the stream kernel has no fixed split grid
        assert res["splits"] > 1
    _assert(res)


EDGE_SHAPES = [
    # (Hq, Hkv, D, Bs)
    (4, 2, 64, 16), (8, 1, 128, 16), (3, 1, 64, 8), (16, 1, 64, 32), (6, 3, 128, 64),
    (32, 8, 64, 128), (2, 2, 64, 256), (16, 2, 128, 8),
    # kv heads in groups of 8 (the tensor kernel's whole-group path)
    (8, 8, 64, 8), (16, 8, 128, 16), (64, 8, 128, 16), (128, 8, 64, 16), (32, 16, 64, 32),
    (24, 8, 64, 256), (96, 8, 128, 32),
]


@pytest.mark.parametrize("kernel", KERNELS, ids=KNAMES.get)
@pytest.mark.parametrize("shape", EDGE_SHAPES, ids=lambda s: "Hq%d-Hkv%d-D%d-Bs%d" % s)
def test_edge_lengths(h, kernel, shape):
    Hq, Hkv, D, Bs = shape
    # cached lengths around block and split edges (appended token makes +1)
    lens = sorted({0, 1, Bs - 2, Bs - 1, Bs, 62, 63, 64, 65, 127, 128, 129, 300, 511, 777})
    lens = [x for x in lens if x >= 0]
    b = wl.small_batch(1000 + Bs + D + Hq, lens, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                       block_size=Bs)
    for split, ctas, fused in ((64, 3, False), (128, 17, True), (0, 0, False), (0, 1, True)):
        _assert(h.run_step(b, kernel=kernel, split_tokens=split, max_ctas=ctas, fused=fused))


@pytest.mark.parametrize("kernel", KERNELS, ids=KNAMES.get)
def test_empty_context_outputs_zero(h, kernel):
    # a sequence with no cached tokens and a negative slot (nothing appended)
    b = wl.small_batch(77, [40, 3], num_q_heads=4, num_kv_heads=2)
    desc = h.desc_of(b)
    q = h.to_dev(b.q)
    out = torch.full_like(q, 7.0)
    lens = torch.tensor([40, 0], dtype=torch.int32, device=h.DEV)
    tables = torch.from_numpy(b.block_tables).to(h.DEV)
    opts = pa.DecodeOptions(split_tokens=64, kernel=kernel, flags=pa.PA_FLAG_CHECK)
    ws = torch.zeros(pa.pa_decode_workspace_size(2, 40, desc, opts), dtype=torch.uint8, device=h.DEV)
    pa.pa_decode(q, h.to_dev(b.k_cache), h.to_dev(b.v_cache), tables, lens, 40, b.scale, out, ws,
                 desc, opts)
    torch.cuda.synchronize()
    assert torch.all(out[1] == 0)
    ref = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables,
                              np.array([40, 0], np.int32), b.scale)
    ok, ex = oracle.within_tolerance(out.float().cpu().numpy(), ref)
    assert ok, ex


@pytest.mark.parametrize("kernel", KERNELS, ids=KNAMES.get)
def test_physical_permutation_is_bitwise_invisible(h, kernel):
    b = wl.small_batch(88, [100, 17, 640, 33], num_q_heads=8, num_kv_heads=2)
    desc = h.desc_of(b)
    lens = torch.from_numpy(b.context_lens).to(h.DEV)
    opts = pa.DecodeOptions(split_tokens=128, kernel=kernel)
    wsb = pa.pa_decode_workspace_size(b.batch, 640, desc, opts)

    def run(kc, vc, tables):
        out = torch.empty_like(h.to_dev(b.q))
        ws = torch.zeros(wsb, dtype=torch.uint8, device=h.DEV)
        pa.pa_decode(h.to_dev(b.q), h.to_dev(kc), h.to_dev(vc), torch.from_numpy(tables).to(h.DEV),
                     lens, 640, b.scale, out, ws, desc, opts)
        torch.cuda.synchronize()
        return h.to_host_bits(out)

    ref = run(b.k_cache, b.v_cache, b.block_tables)
    perm = np.random.default_rng(5).permutation(b.num_blocks).astype(np.int32)
    kc = np.empty_like(b.k_cache); vc = np.empty_like(b.v_cache)
    kc[perm] = b.k_cache; vc[perm] = b.v_cache
    tables = np.where(b.block_tables >= 0, perm[np.maximum(b.block_tables, 0)], -1).astype(np.int32)
    np.testing.assert_array_equal(run(kc, vc, tables), ref)


@pytest.mark.parametrize("kernel", KERNELS, ids=KNAMES.get)
def test_workspace_reused_without_clearing(h, kernel):
    b = wl.small_batch(99, [1000, 513, 64], num_q_heads=4, num_kv_heads=1)
    desc = h.desc_of(b)
    lens = torch.from_numpy(b.context_lens).to(h.DEV)
    tables = torch.from_numpy(b.block_tables).to(h.DEV)
    opts = pa.DecodeOptions(split_tokens=64, kernel=kernel, flags=pa.PA_FLAG_CHECK)
    ws = torch.zeros(pa.pa_decode_workspace_size(b.batch, 1000, desc, opts), dtype=torch.uint8,
                     device=h.DEV)
    ref = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale)
    kc, vc, q = h.to_dev(b.k_cache), h.to_dev(b.v_cache), h.to_dev(b.q)
    outs = []
    for _ in range(3):
        out = torch.empty_like(q)
        pa.pa_decode(q, kc, vc, tables, lens, 1000, b.scale, out, ws, desc, opts)
        torch.cuda.synchronize()
        outs.append(h.to_host_bits(out))
        ok, ex = oracle.within_tolerance(out.float().cpu().numpy(), ref)
        assert ok, ex
    np.testing.assert_array_equal(outs[0], outs[1])
    np.testing.assert_array_equal(outs[0], outs[2])


def _decode_into(h, b, ws, opts):
    desc = h.desc_of(b)
    q = h.to_dev(b.q)
    out = torch.full_like(q, 5.0)
    max_len = int(b.context_lens.max())
    assert ws.numel() >= pa.pa_decode_workspace_size(b.batch, max_len, desc, opts)
    pa.pa_decode(q, h.to_dev(b.k_cache), h.to_dev(b.v_cache), torch.from_numpy(b.block_tables).to(h.DEV),
                 torch.from_numpy(b.context_lens).to(h.DEV), max_len, b.scale, out, ws, desc, opts)
    torch.cuda.synchronize()
    ref = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale)
    return oracle.within_tolerance(out.float().cpu().numpy(), ref)


def test_stream_workspace_shared_across_shapes_and_kernels(h):
    # one workspace, never cleared, through calls of different shapes, partitions and
    # kernels: nothing a call leaves behind may leak into the next one
    rng = np.random.default_rng(31)
    ws = torch.zeros(64 << 20, dtype=torch.uint8, device=h.DEV)
    a = wl.small_batch(501, list(rng.integers(1, 3000, 12)), num_q_heads=32, num_kv_heads=8)
    mixed = wl.small_batch(502, [5000] + list(rng.integers(1, 200, 30)), num_q_heads=16,
                           num_kv_heads=8, head_dim=128)
    wide = wl.small_batch(503, list(rng.integers(1, 400, 300)), num_q_heads=8, num_kv_heads=8)
    steps = [
        (a, dict(kernel=pa.PA_KERNEL_TENSOR, max_ctas=7)),             # a few pieces per sequence
        (wide, dict(kernel=pa.PA_KERNEL_TENSOR_SPLIT, split_tokens=64)),  # partials over the region
        (wide, dict(kernel=pa.PA_KERNEL_TENSOR)),
        (a, dict(kernel=pa.PA_KERNEL_TENSOR)),                         # > 16 pieces per sequence
        (mixed, dict(kernel=pa.PA_KERNEL_TENSOR, max_ctas=40)),        # one long + many short
        (wide, dict(kernel=pa.PA_KERNEL_SIMT, split_tokens=64)),
        (a, dict(kernel=pa.PA_KERNEL_TENSOR, max_ctas=7)),
        (mixed, dict(kernel=pa.PA_KERNEL_TENSOR, max_ctas=40)),
    ]
    for i, (b, o) in enumerate(steps):
        ok, ex = _decode_into(h, b, ws, pa.DecodeOptions(flags=pa.PA_FLAG_CHECK, **o))
        assert ok, "call %d outside tolerance by %g" % (i, ex)


def test_stream_many_short_sequences(h):
    # 8200 short sequences (65600 (sequence, kv head) pairs), cut by a 50-CTA grid and by
    # the full one
    rng = np.random.default_rng(32)
    b = wl.small_batch(504, list(rng.integers(1, 48, 8200)), num_q_heads=8, num_kv_heads=8)
    for ctas in (50, 0):
        opts = pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR, flags=pa.PA_FLAG_CHECK, max_ctas=ctas)
        ws = torch.zeros(pa.pa_decode_workspace_size(b.batch, int(b.context_lens.max()), h.desc_of(b),
                                                     opts), dtype=torch.uint8, device=h.DEV)
        ok, ex = _decode_into(h, b, ws, opts)
        assert ok, ex


@pytest.mark.parametrize("cfg", ["c1", "c2", "c3", "c4"])
@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
def test_pdl_early_start(h, cfg, fused):
    # PA_FLAG_PDL: the decode kernel may start while the append kernel before it runs;
    # the new token's K/V (written by that kernel) must still be seen
    _assert(h.run_step(wl.CONFIGS[cfg](), kernel=pa.PA_KERNEL_TENSOR, fused=fused, pdl=True))


def test_pdl_chain_matches_plain_launches(h):
    # calls chained through their outputs (each call's q is the previous call's out, written
    # by the previous merge kernel): with PA_FLAG_PDL every call starts early and must
    # still read the finished q; the chain is bitwise the chain of plain launches
    b = wl.config2()
    desc = h.desc_of(b)
    kc, vc = h.to_dev(b.k_cache), h.to_dev(b.v_cache)
    tables = torch.from_numpy(b.block_tables).to(h.DEV)
    lens = torch.from_numpy(b.context_lens).to(h.DEV)
    max_len = int(b.context_lens.max())

    def chain(flags, ctas):
        opts = pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR, flags=flags, max_ctas=ctas)
        ws = torch.zeros(pa.pa_decode_workspace_size(b.batch, max_len, desc, opts), dtype=torch.uint8,
                         device=h.DEV)
        bufs = [h.to_dev(b.q)] + [torch.empty_like(h.to_dev(b.q)) for _ in range(6)]
        for i in range(6):
            pa.pa_decode(bufs[i], kc, vc, tables, lens, max_len, b.scale, bufs[i + 1], ws, desc, opts)
        torch.cuda.synchronize()
        assert pa.pa_decode_status(ws) == 0
        return [h.to_host_bits(x) for x in bufs[1:]]

    ref = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale)
    for ctas in (0, 37):
        plain = chain(0, ctas)
        early = chain(pa.PA_FLAG_PDL, ctas)
        first = plain[0].view(np.int16)
        got = torch.from_numpy(first.copy()).view(torch.bfloat16).float().numpy()
        ok, ex = oracle.within_tolerance(got, ref)
        assert ok, ex
        for i, (x, y) in enumerate(zip(plain, early)):
            np.testing.assert_array_equal(x, y, err_msg="call %d of the chain" % i)


@pytest.mark.parametrize("kernel", KERNELS, ids=KNAMES.get)
def test_bad_block_id_reported_not_faulted(h, kernel):
    b = wl.small_batch(111, [50, 20], num_q_heads=4, num_kv_heads=2)
    desc = h.desc_of(b)
    tables = b.block_tables.copy()
    tables[0, 1] = b.num_blocks + 5      # outside the pool
    opts = pa.DecodeOptions(split_tokens=64, kernel=kernel, flags=pa.PA_FLAG_CHECK)
    ws = torch.zeros(pa.pa_decode_workspace_size(2, 50, desc, opts), dtype=torch.uint8, device=h.DEV)
    out = torch.empty_like(h.to_dev(b.q))
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode(h.to_dev(b.q), h.to_dev(b.k_cache), h.to_dev(b.v_cache),
                     torch.from_numpy(tables).to(h.DEV), torch.from_numpy(b.context_lens).to(h.DEV),
                     50, b.scale, out, ws, desc, opts)
    assert e.value.status == -7
    # the untouched sequence is still right, and the status word was cleared
    ref = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale)
    ok, ex = oracle.within_tolerance(out.float().cpu().numpy()[1], ref[1])
    assert ok, ex
    assert pa.pa_decode_status(ws) == 0


@pytest.mark.parametrize("kernel", KERNELS, ids=KNAMES.get)
def test_length_beyond_bound_reported(h, kernel):
    b = wl.small_batch(112, [50, 20], num_q_heads=4, num_kv_heads=2)
    desc = h.desc_of(b)
    opts = pa.DecodeOptions(split_tokens=64, kernel=kernel, flags=pa.PA_FLAG_CHECK)
    ws = torch.zeros(pa.pa_decode_workspace_size(2, 40, desc, opts), dtype=torch.uint8, device=h.DEV)
    out = torch.empty_like(h.to_dev(b.q))
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode(h.to_dev(b.q), h.to_dev(b.k_cache), h.to_dev(b.v_cache),
                     torch.from_numpy(b.block_tables).to(h.DEV),
                     torch.from_numpy(b.context_lens).to(h.DEV), 40, b.scale, out, ws, desc, opts)
    assert e.value.status == -8


def test_argument_errors(h):
    b = wl.config1()
    desc = h.desc_of(b)
    q = h.to_dev(b.q)
    kc = h.to_dev(b.k_cache)
    tables = torch.from_numpy(b.block_tables).to(h.DEV)
    lens = torch.from_numpy(b.context_lens).to(h.DEV)
    out = torch.empty_like(q)
    ws = torch.zeros(pa.pa_decode_workspace_size(2, 37, desc), dtype=torch.uint8, device=h.DEV)
    with pytest.raises(pa.PaError) as e:   # workspace too small
        pa.pa_decode(q, kc, kc, tables, lens, 37, b.scale, out, ws, desc, workspace_bytes=16)
    assert e.value.status == -4
    bad = pa.CacheDesc.make(num_blocks=8, block_size=16, num_kv_heads=1, num_q_heads=2, head_dim=96,
                            max_blocks_per_seq=3)
    with pytest.raises(pa.PaError) as e:   # head_dim 96 not built (raw pointers: the C check, not
        # the binding's pool-size check, answers; the shape is refused before any access)
        pa.pa_decode(q, kc.data_ptr(), kc.data_ptr(), tables, lens, 37, b.scale, out, ws, bad)
    assert e.value.status == -2
    with pytest.raises(pa.PaError) as e:   # misaligned output pointer
        pa.pa_decode(q, kc, kc, tables, lens, 37, b.scale, out.data_ptr() + 2, ws, desc)
    assert e.value.status == -1


@pytest.mark.parametrize("kernel", [pa.PA_KERNEL_TENSOR, pa.PA_KERNEL_SIMT], ids=["tensor", "simt"])
def test_c5_continuous_batching_trace(h, kernel):
    """Full-size C5 batch (256 sequences) through 12 trace steps on layers 0 and 15.

    Each step: retire finished sequences, admit newcomers, append one token per
    sequence (host block manager vs its model, bit-exact), then the fused
    append + decode per layer; the oracle keeps its own pools, appending at the
    model's slots.  Outputs compared in full at steps 0, 5 and 11 (step 11 is
    past the trace's first retirements).
    """
    t = wl.Trace5()
    B, Bs, MB, N = t.batch, t.block_size, t.max_blocks_per_seq, t.num_blocks
    layers, steps, check = (0, 15), 12, {0, 5, 11}
    assert t.finish[1:steps].any()
    bm = pa.BlockManager(N, Bs, B, MB, t.free_order)
    model = oracle.BlockManagerModel(N, Bs, B, MB, t.free_order)
    for s in range(B):
        bm.add_seq(s, int(t.initial_lens[s]))
        model.add_seq(s, int(t.initial_lens[s]))
    host = {l: [a.copy() for a in t.pool(l)] for l in layers}
    devp = {l: [h.to_dev(a) for a in host[l]] for l in layers}
    desc = pa.CacheDesc.make(num_blocks=N, block_size=Bs, num_kv_heads=t.num_kv_heads,
                             num_q_heads=t.num_q_heads, head_dim=t.head_dim, max_blocks_per_seq=MB)
    opts = pa.DecodeOptions(kernel=kernel, flags=pa.PA_FLAG_CHECK)
    ws = torch.zeros(pa.pa_decode_workspace_size(B, 16384 + 200, desc, opts), dtype=torch.uint8,
                     device=h.DEV)
    seqs = np.arange(B, dtype=np.int32)
    for step, retired, admitted in t.events():
        if step >= steps:
            break
        for s in retired:
            bm.free_seq(s)
            model.free_seq(s)
        for s, n in admitted:
            bm.add_seq(s, n)
            model.add_seq(s, n)
        slots = bm.append_tokens(seqs)
        m_slots = np.array(model.append_tokens(list(range(B))), dtype=np.int64)
        assert np.array_equal(slots, m_slots)
        tables = bm.block_tables().copy()
        lens = bm.context_lens().copy()
        m_tables = np.array([model.table_array(s) for s in range(B)], dtype=np.int32)
        assert np.array_equal(tables, m_tables) and list(lens) == model.lens
        td, ld = torch.from_numpy(tables).to(h.DEV), torch.from_numpy(lens).to(h.DEV)
        for l in layers:
            q, k, v = t.token_inputs(l, step)
            out = torch.empty_like(h.to_dev(q))
            pa.pa_append_decode(h.to_dev(q), h.to_dev(k), h.to_dev(v), devp[l][0], devp[l][1], td, ld,
                                int(lens.max()), t.scale, out, ws, desc, opts)
            oracle.append_kv(k, v, m_slots, host[l][0], host[l][1], in_place=True)
            if step in check:
                torch.cuda.synchronize()
                ref = oracle.paged_decode(q, host[l][0], host[l][1], m_tables, lens, t.scale)
                ok, ex = oracle.within_tolerance(out.float().cpu().numpy(), ref)
                assert ok, "layer %d step %d: excess %g" % (l, step, ex)
    torch.cuda.synchronize()
    for l in layers:   # the pools the GPU appended into equal the oracle's, byte for byte
        assert np.array_equal(h.to_host_bits(devp[l][0]), host[l][0])
        assert np.array_equal(h.to_host_bits(devp[l][1]), host[l][1])
    bm.close()
