"""Host-side pieces of bench.py that need no GPU: the chunked-prefill CPU baseline (the
oracle on query windows spread over the chunks) reports a positive rate and says what it
sampled."""
import numpy as np

import bench
import workloads as wl


def test_pf_cpu_baseline_samples_every_part_of_the_chunks():
    lens = [c + bench.PF_NEW for c in bench.PF_CACHED]
    b = wl.make_batch("PF", wl.CONFIG_SEED_BASE + 41, [L - 1 for L in lens], num_q_heads=32, num_kv_heads=8,
                      head_dim=64, block_size=16)
    B = len(lens)
    cu = np.concatenate([[0], np.cumsum([bench.PF_NEW] * B)]).astype(np.int32)
    q_h = np.zeros((int(cu[-1]), 32, 64), dtype=np.uint16)
    res = bench.pf_cpu_baseline(b, q_h, cu, lens, B, 0.0)       # runs for at least a second
    assert res["kind"] == "oracle" and res["unit"] == "tokens/s" and res["value"] > 0
    assert res["cores"] >= 1 and "windows of 64 query tokens" in res["sample"]
    # the visiting order reaches every window of every sequence
    windows = bench.PF_NEW // 64
    seen = {(n % B, (13 * (n // B)) % windows) for n in range(B * windows)}
    assert len(seen) == B * windows


def test_unique_kv_bytes_counts_shared_blocks_once():
    """The roofline's bytes for a shared prefix: a block held by several tables counts once
    (with the most tokens any sequence uses in it); without sharing they equal the logical
    K+V bytes."""
    Bs, Hkv, D = 4, 2, 8
    # three sequences over one shared 2-block prefix (8 tokens), then private blocks
    tables = np.array([[0, 1, 2, 3], [0, 1, 4, 0], [0, 1, 5, 6]], dtype=np.int32)
    lens = np.array([15, 9, 13], dtype=np.int32)
    row = 2 * Hkv * D * 2                                  # K+V bytes of one token, bf16
    # prefix 8 tokens once; suffixes 7, 1 and 5 tokens
    assert bench.unique_kv_bytes(tables, lens, Bs, Hkv, D) == (8 + 7 + 1 + 5) * row
    assert bench.kv_read_bytes(lens, Hkv, D) == int(lens.sum()) * row
    # private tables: unique == logical, and E4M3 halves both
    private = np.array([[0, 1, 2, 3], [4, 5, 6, 7], [8, 9, 10, 11]], dtype=np.int32)
    assert bench.unique_kv_bytes(private, lens, Bs, Hkv, D) == bench.kv_read_bytes(lens, Hkv, D)
    assert bench.unique_kv_bytes(private, lens, Bs, Hkv, D, 1) * 2 == bench.kv_read_bytes(lens, Hkv, D)
    # a partly used shared block counts the longest use: two sequences of 2 and 3 tokens in block 7
    assert bench.unique_kv_bytes(np.array([[7], [7]]), np.array([2, 3]), Bs, Hkv, D) == 3 * row


def test_profiled_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    """A DRAM figure from a profile summary is used only while the kernel sources still hash
    to the build that was captured; any other hash (an edited kernel) gives null."""
    import os
    pkg = tmp_path / "pagedattention_kv_cache_pa_b200"
    pkg.mkdir()
    os.symlink(os.path.join(bench.ROOT, "pagedattention_kv_cache_pa_b200", "csrc"), pkg / "csrc")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    good = bench.kernel_source_hash("tensor")
    (tmp_path / "profiles" / "a.md").write_text(
        "traffic[c9,tensor]: 12345 bytes/launch source=%s\n"
        "traffic[c8,tensor]: 999 bytes/launch source=%s\n" % (good, "0" * 16))
    assert bench.profiled_traffic("c9", "tensor") == 12345
    assert bench.profiled_traffic("c8", "tensor") is None     # captured on other sources
    assert bench.profiled_traffic("c7", "tensor") is None     # never captured
    assert bench.kernel_source_hash("prefill_ws") != good     # each kernel hashes its own files


def test_decode_cpu_baseline_reports_parallel_and_single_thread():
    """The decode CPU baseline times the oracle on the host's threads and again on one thread,
    and leaves the oracle's thread count as it found it."""
    import oracle
    b = wl.small_batch(77, [5, 40, 300], num_q_heads=8, num_kv_heads=2)
    B, Bs = b.batch, b.block_size
    lens = b.context_lens.astype(np.int32) + 1
    slots = np.array([int(b.block_tables[s, (L - 1) // Bs]) * Bs + (L - 1) % Bs for s, L in enumerate(lens)],
                     dtype=np.int64)
    before = oracle.num_threads()
    res = bench.cpu_baseline(b, slots, b.block_tables, lens, 0.05)
    assert oracle.num_threads() == before
    assert res["kind"] == "oracle" and res["value"] > 0 and res["cores"] == before
    st = res["single_thread"]
    assert st["cores"] == 1 and st["value"] > 0 and st["unit"] == res["unit"]
