"""The decode's bounded waits give up cleanly (needs a B200).

PA_FLAG_SELFTEST_STALL makes the stream kernel's CTA 0 skip every copy and signal, so its
consumer warps wait on a barrier nothing will complete: no copy is ever issued for it, so none
is in flight when the wait gives up.  The waits must run out (10 ms in this mode), raise the
timeout bit, and leave the context and the workspace fit for the next call, whose result must
match the oracle.  No fault, trap or hang is involved: the only failure is an unanswered wait.
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


@pytest.mark.parametrize("fused", [False, True], ids=["decode", "append_decode"])
@pytest.mark.parametrize("pdl", [False, True], ids=["plain", "pdl"])
def test_timed_out_wait_is_reported_and_the_next_call_is_clean(h, fused, pdl):
    b = wl.config2()
    (slots, tables, lens), (o_slots, o_tables, o_lens) = h.host_step(b)
    desc = h.desc_of(b)
    kc, vc = h.to_dev(b.k_cache), h.to_dev(b.v_cache)
    q, kn, vn = h.to_dev(b.q), h.to_dev(b.k_new), h.to_dev(b.v_new)
    td, ld = torch.from_numpy(tables).to(h.DEV), torch.from_numpy(lens).to(h.DEV)
    max_len = int(lens.max())
    extra = pa.PA_FLAG_PDL if pdl else 0
    opts = pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR, flags=pa.PA_FLAG_CHECK | extra)
    stall = pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR,
                             flags=pa.PA_FLAG_CHECK | pa.PA_FLAG_SELFTEST_STALL | extra)
    ws = torch.zeros(pa.pa_decode_workspace_size(b.batch, max_len, desc, opts), dtype=torch.uint8,
                     device=h.DEV)
    out = torch.empty_like(q)

    def call(o):
        if fused:
            pa.pa_append_decode(q, kn, vn, kc, vc, td, ld, max_len, b.scale, out, ws, desc, o)
        else:
            pa.pa_decode(q, kc, vc, td, ld, max_len, b.scale, out, ws, desc, o)

    if not fused:
        pa.pa_append_kv(kn, vn, torch.from_numpy(slots).to(h.DEV), kc, vc, desc)
    with pytest.raises(pa.PaError) as e:
        call(stall)
    assert e.value.status == -9                        # PA_ERR_TIMEOUT
    torch.cuda.synchronize()                           # the context is still usable
    assert pa.pa_decode_status(ws) == 0                # PA_FLAG_CHECK cleared the status word
    for _ in range(2):                                 # the same workspace, as it was left
        out.fill_(7.0)
        call(opts)
        torch.cuda.synchronize()
        ref_k, ref_v = oracle.append_kv(b.k_new, b.v_new, o_slots, b.k_cache, b.v_cache)
        ref = oracle.paged_decode(b.q, ref_k, ref_v, o_tables, o_lens, b.scale)
        ok, excess = oracle.within_tolerance(out.float().cpu().numpy(), ref)
        assert ok, "call after the timeout outside tolerance by %g" % excess
    assert np.array_equal(h.to_host_bits(kc), ref_k) and np.array_equal(h.to_host_bits(vc), ref_v)


def test_selftest_flag_needs_the_stream_kernel(h):
    b = wl.small_batch(5, [40, 3], num_q_heads=4, num_kv_heads=2)
    desc = h.desc_of(b)
    o = pa.DecodeOptions(kernel=pa.PA_KERNEL_TENSOR, flags=pa.PA_FLAG_SELFTEST_STALL)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device=h.DEV)
    out = torch.empty_like(h.to_dev(b.q))
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode(h.to_dev(b.q), h.to_dev(b.k_cache), h.to_dev(b.v_cache),
                     torch.from_numpy(b.block_tables).to(h.DEV), torch.from_numpy(b.context_lens).to(h.DEV),
                     40, b.scale, out, ws, desc, o)
    assert e.value.status == -2
