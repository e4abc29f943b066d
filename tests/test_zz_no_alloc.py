"""pa_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a runtime's memory planner that owns every allocation, a
latency-bound loop where cudaMalloc could stall, a C caller without an
allocator) cannot provide pa_decode's workspace; pa_decode_noalloc takes its
scratch from a fixed array in the library instead.  This file checks, through
the C ABI, that two calls in a row match the fp64 oracle within the parity
tolerance (with and without the status read-back), that a call which reported
an error leaves nothing behind for the next call of another kernel or shape,
that unsupported shapes get pa_decode's own error, and that a shape needing
more scratch than the array holds is refused without a launch.  It is
collected last on purpose.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
import pagedattention_kv_cache_pa_b200 as pa

pytestmark = pytest.mark.gpu


def _dev(a, device):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


@pytest.fixture(scope="module")
def c2():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    b = wl.config2()
    lens = (b.context_lens + 1).astype(np.int32)          # attend over the cached tokens + 1 slot
    tables = b.block_tables.copy()
    for s in range(b.batch):                               # give full last blocks a next block
        L = int(b.context_lens[s])
        if L % b.block_size == 0:
            tables[s, L // b.block_size] = b.free_order[s]
    desc = pa.CacheDesc.make(num_blocks=b.num_blocks, block_size=b.block_size,
                             num_kv_heads=b.num_kv_heads, num_q_heads=b.num_q_heads,
                             head_dim=b.head_dim, max_blocks_per_seq=b.max_blocks_per_seq)
    return dict(b=b, desc=desc, dev=dev, q=_dev(b.q, dev), k=_dev(b.k_cache, dev),
                v=_dev(b.v_cache, dev), tables=torch.from_numpy(tables).to(dev),
                lens=torch.from_numpy(lens).to(dev), max_len=int(lens.max()))


@pytest.fixture(scope="module")
def c2_ref(c2):
    d = c2
    return oracle.paged_decode(d["b"].q, d["b"].k_cache, d["b"].v_cache, d["tables"].cpu().numpy(),
                               d["lens"].cpu().numpy(), d["b"].scale)


@pytest.mark.parametrize("opts", [
    dict(),                                                # automatic (tensor kernel, full grid)
    dict(kernel=pa.PA_KERNEL_TENSOR, max_ctas=5),          # most sequences cut: partials in the array
    dict(kernel=pa.PA_KERNEL_TENSOR_SPLIT, split_tokens=128),
    dict(kernel=pa.PA_KERNEL_SIMT, split_tokens=256),
], ids=["auto", "tensor-5ctas", "split128", "simt256"])
def test_matches_the_oracle_on_two_calls_in_a_row(c2, c2_ref, opts):
    d = c2
    for flags in (pa.PA_FLAG_CHECK, 0):                    # with and without the status read-back
        o = pa.DecodeOptions(flags=flags, **opts)
        for _ in range(2):
            out = torch.full_like(d["q"], 3.0)
            pa.pa_decode_noalloc(d["q"], d["k"], d["v"], d["tables"], d["lens"], d["max_len"],
                                 d["b"].scale, out, d["desc"], o)
            torch.cuda.synchronize()
            ok, excess = oracle.within_tolerance(out.float().cpu().numpy(), c2_ref)
            assert ok, "pa_decode_noalloc outside the tolerance of the oracle by %g" % excess


def test_a_failed_call_leaves_nothing_behind(c2, c2_ref):
    # a call that reports a bad block id, then a clean call of the same shape, then one of
    # another kernel and shape: the shared array's leftovers must not leak into the next call
    d = c2
    o = pa.DecodeOptions(flags=pa.PA_FLAG_CHECK)
    bad = d["tables"].clone()
    bad[3, 2] = d["b"].num_blocks + 7
    out = torch.empty_like(d["q"])
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_noalloc(d["q"], d["k"], d["v"], bad, d["lens"], d["max_len"], d["b"].scale, out,
                             d["desc"], o)
    assert e.value.status == -7
    out = torch.full_like(d["q"], 3.0)
    pa.pa_decode_noalloc(d["q"], d["k"], d["v"], d["tables"], d["lens"], d["max_len"], d["b"].scale,
                         out, d["desc"], o)
    torch.cuda.synchronize()
    ok, excess = oracle.within_tolerance(out.float().cpu().numpy(), c2_ref)
    assert ok, excess
    # another shape (D = 128, 16 query heads per kv head) on the CUDA-core kernel, then on the
    # tensor-core split kernel
    b = wl.small_batch(611, [3000, 17, 900, 1], num_q_heads=32, num_kv_heads=2, head_dim=128)
    desc = pa.CacheDesc.make(num_blocks=b.num_blocks, block_size=b.block_size, num_kv_heads=2,
                             num_q_heads=32, head_dim=128, max_blocks_per_seq=b.max_blocks_per_seq)
    ref = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale)
    args = [_dev(b.q, d["dev"]), _dev(b.k_cache, d["dev"]), _dev(b.v_cache, d["dev"]),
            torch.from_numpy(b.block_tables).to(d["dev"]), torch.from_numpy(b.context_lens).to(d["dev"]),
            3000, b.scale]
    for o2 in (pa.DecodeOptions(kernel=pa.PA_KERNEL_SIMT, split_tokens=64, flags=pa.PA_FLAG_CHECK),
               pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR, flags=pa.PA_FLAG_CHECK)):
        out2 = torch.full_like(args[0], 3.0)
        pa.pa_decode_noalloc(*args, out2, desc, o2)
        torch.cuda.synchronize()
        ok, excess = oracle.within_tolerance(out2.float().cpu().numpy(), ref)
        assert ok, excess


def test_unsupported_shape_gets_the_same_error_as_pa_decode(c2):
    d = c2
    # head_dim 96 is not built: PA_ERR_UNSUPPORTED from both entry points, nothing launched
    bad = pa.CacheDesc.make(num_blocks=d["b"].num_blocks, block_size=16, num_kv_heads=8, num_q_heads=32,
                            head_dim=96, max_blocks_per_seq=d["b"].max_blocks_per_seq)
    out = torch.empty_like(d["q"])
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device=d["dev"])
    for call in (lambda: pa.pa_decode(d["q"], d["k"].data_ptr(), d["v"].data_ptr(), d["tables"], d["lens"],
                                      d["max_len"], 0.1, out, ws, bad),
                 lambda: pa.pa_decode_noalloc(d["q"], d["k"].data_ptr(), d["v"].data_ptr(), d["tables"],
                                              d["lens"], d["max_len"], 0.1, out, bad)):
        with pytest.raises(pa.PaError) as e:
            call()
        assert e.value.status == -2


def test_shape_beyond_the_array_is_refused(c2):
    d = c2
    # 2049 splits of 64 tokens x 32 kv heads x 16 query heads x D=128: far beyond 16 MiB
    big = pa.CacheDesc.make(num_blocks=64, block_size=16, num_kv_heads=32, num_q_heads=512,
                            head_dim=128, max_blocks_per_seq=8193)
    o = pa.DecodeOptions(kernel=pa.PA_KERNEL_SIMT, split_tokens=64)
    assert pa.pa_decode_workspace_size(4, 131073, big, o) > (16 << 20)
    out = torch.zeros(4 * 512 * 128, dtype=torch.bfloat16, device=d["dev"])
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_noalloc(out, d["k"], d["v"], d["tables"], d["lens"][:4], 131073, 0.1, out,
                             big, o, num_seqs=4)
    assert e.value.status == -4
