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
