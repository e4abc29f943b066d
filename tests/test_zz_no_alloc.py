"""pa_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a runtime's memory planner that owns every allocation, a
latency-bound loop where cudaMalloc could stall, a C caller without an
allocator) cannot provide pa_decode's workspace; pa_decode_noalloc takes its
scratch from a fixed array in the library instead.  This file checks, through
the C ABI, that two calls in a row give the existing entry point's result
within the parity tolerance, and that a shape needing more scratch than the
array holds is refused without a launch.  It is collected last on purpose.
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


@pytest.mark.parametrize("opts", [
    dict(),                                                # automatic (tensor kernel, full grid)
    dict(kernel=pa.PA_KERNEL_TENSOR, max_ctas=5),          # most sequences cut: partials in the array
    dict(kernel=pa.PA_KERNEL_TENSOR_SPLIT, split_tokens=128),
    dict(kernel=pa.PA_KERNEL_SIMT, split_tokens=256),
], ids=["auto", "tensor-5ctas", "split128", "simt256"])
def test_matches_pa_decode_on_two_calls_in_a_row(c2, opts):
    o = pa.DecodeOptions(flags=pa.PA_FLAG_CHECK, **opts)
    d = c2
    ref = torch.empty_like(d["q"])
    ws = torch.zeros(pa.pa_decode_workspace_size(d["b"].batch, d["max_len"], d["desc"], o),
                     dtype=torch.uint8, device=d["dev"])
    pa.pa_decode(d["q"], d["k"], d["v"], d["tables"], d["lens"], d["max_len"], d["b"].scale, ref,
                 ws, d["desc"], o)
    torch.cuda.synchronize()
    want = ref.float().cpu().numpy().astype(np.float64)
    for _ in range(2):
        out = torch.full_like(d["q"], 3.0)
        pa.pa_decode_noalloc(d["q"], d["k"], d["v"], d["tables"], d["lens"], d["max_len"],
                             d["b"].scale, out, d["desc"], o)
        torch.cuda.synchronize()
        ok, excess = oracle.within_tolerance(out.float().cpu().numpy(), want)
        assert ok, "pa_decode_noalloc differs from pa_decode by %g beyond tolerance" % excess


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
