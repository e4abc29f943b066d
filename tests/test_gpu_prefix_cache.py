"""Device side of prefix caching and copy-on-write, through the C ABI (needs a B200).

pa_copy_blocks must copy blocks bit-exactly and touch nothing else.  End to end:
sequences forked whole from one prompt append a token each; the manager reports
the copy-on-write pairs, pa_copy_blocks runs them, pa_append_kv writes the new
rows and pa_decode reads every sequence.  The oracle side replays the same
steps with the model and numpy copies: the pool must match byte for byte and
the outputs within 1e-2 + 1e-2 * |oracle|.
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


@pytest.mark.parametrize("shape", [(8, 16, 64), (8, 256, 64), (1, 16, 128), (16, 8, 128)],
                         ids=lambda s: "Hkv%d-Bs%d-D%d" % s)
def test_copy_blocks_bit_exact(h, shape):
    Hkv, Bs, D = shape
    b = wl.small_batch(71 + Bs, [Bs * 30], num_q_heads=Hkv, num_kv_heads=Hkv, head_dim=D, block_size=Bs)
    N = b.num_blocks
    rng = np.random.default_rng(Bs + D)
    perm = rng.permutation(N)
    src, dst = perm[: N // 3], perm[N // 3: 2 * (N // 3)]
    pairs = np.stack([src, dst], axis=1).astype(np.int32)
    pairs = np.concatenate([pairs, [[-1, 0], [0, N]]]).astype(np.int32)   # skipped pairs
    kc, vc = h.to_dev(b.k_cache), h.to_dev(b.v_cache)
    pa.pa_copy_blocks(kc, vc, torch.from_numpy(pairs).to(h.DEV), h.desc_of(b))
    torch.cuda.synchronize()
    want_k, want_v = b.k_cache.copy(), b.v_cache.copy()
    want_k[dst], want_v[dst] = b.k_cache[src], b.v_cache[src]
    np.testing.assert_array_equal(h.to_host_bits(kc), want_k)
    np.testing.assert_array_equal(h.to_host_bits(vc), want_v)


@pytest.mark.parametrize("Bs,prompt", [(16, 37), (16, 32), (8, 5), (64, 100)])
def test_fork_copy_on_write_then_decode(h, Bs, prompt):
    Hq, Hkv, D, S = 16, 8, 64, 4
    base = wl.small_batch(900 + Bs + prompt, [prompt] * S, num_q_heads=Hq, num_kv_heads=Hkv,
                          head_dim=D, block_size=Bs)
    N, MB = base.num_blocks + 8, base.max_blocks_per_seq + 2
    # a pool with spare blocks: random contents stand for the prompt's prefilled K/V
    rng = np.random.default_rng(Bs)
    extra = np.arange(8) % base.num_blocks                # exactly 8 more blocks
    kpool = np.concatenate([base.k_cache, base.k_cache[extra]])
    vpool = np.concatenate([base.v_cache, base.v_cache[extra]])
    assert kpool.shape[0] == N and vpool.shape[0] == N
    order = rng.permutation(N).astype(np.int32)
    bm = pa.BlockManager(N, Bs, S, MB, order)
    m = oracle.BlockManagerModel(N, Bs, S, MB, order)
    ids = [int(t) for t in rng.integers(0, 1000, prompt)]
    bm.add_seq_tokens(0, ids)
    m.add_seq_tokens(0, ids)
    for s in range(1, S):
        bm.fork_all(s, 0)
        m.fork_all(s, 0)
    seqs = list(range(S))
    new_ids = [int(t) for t in rng.integers(0, 1000, S)]
    slots, copies = bm.append_token_ids(seqs, new_ids)
    want_slots, want_copies = m.append_token_ids(seqs, new_ids)
    assert list(slots) == want_slots and [tuple(c) for c in copies.tolist()] == want_copies
    if prompt % Bs:
        assert len(want_copies) == S - 1          # every holder but the last writer copies
    # device: copies, append, decode
    desc = pa.CacheDesc.make(num_blocks=N, block_size=Bs, num_kv_heads=Hkv, num_q_heads=Hq,
                             head_dim=D, max_blocks_per_seq=MB)
    kc, vc = h.to_dev(kpool), h.to_dev(vpool)
    if len(copies):
        pa.pa_copy_blocks(kc, vc, torch.from_numpy(np.ascontiguousarray(copies)).to(h.DEV), desc)
    pa.pa_append_kv(h.to_dev(base.k_new), h.to_dev(base.v_new), torch.from_numpy(slots).to(h.DEV),
                    kc, vc, desc)
    tables = bm.block_tables().copy()
    lens = bm.context_lens().copy()
    q = h.to_dev(base.q)
    out = torch.empty_like(q)
    for kernel in (pa.PA_KERNEL_TENSOR, pa.PA_KERNEL_SIMT):
        opts = pa.DecodeOptions(kernel=kernel, flags=pa.PA_FLAG_CHECK)
        ws = torch.zeros(pa.pa_decode_workspace_size(S, int(lens.max()), desc, opts),
                         dtype=torch.uint8, device=h.DEV)
        pa.pa_decode(q, kc, vc, torch.from_numpy(tables).to(h.DEV), torch.from_numpy(lens).to(h.DEV),
                     int(lens.max()), base.scale, out, ws, desc, opts)
        torch.cuda.synchronize()
        # oracle: the same copies and append on host pools, then the fp64 decode
        rk, rv = kpool.copy(), vpool.copy()
        for a, b_ in want_copies:
            rk[b_], rv[b_] = kpool[a], vpool[a]
        rk, rv = oracle.append_kv(base.k_new, base.v_new, np.array(want_slots, dtype=np.int64), rk, rv)
        np.testing.assert_array_equal(h.to_host_bits(kc), rk)
        np.testing.assert_array_equal(h.to_host_bits(vc), rv)
        o_tables = np.array([m.table_array(s) for s in range(S)], dtype=np.int32)
        ref = oracle.paged_decode(base.q, rk, rv, o_tables, np.array(m.lens, dtype=np.int32), base.scale)
        ok, ex = oracle.within_tolerance(out.float().cpu().numpy(), ref)
        assert ok, ex
    bm.close()
