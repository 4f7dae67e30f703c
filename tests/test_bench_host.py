"""Host-side parts of the benchmark that need no GPU: the oracle timing legs."""
import bench
from paged_kv_cache_432_b200 import workload as wl


def test_cpu_baseline_times_the_oracle_on_one_and_on_all_cores():
    w = wl.make("tiny", device="cpu")
    cb = bench.cpu_baseline(w, budget_s=0.05)
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] > 0
    assert cb["unit"] == "GB/s"
    ac = cb["all_cores"]
    assert ac["cores"] >= 1 and ac["value"] > 0 and ac["unit"] == "GB/s"


def test_sample_bytes_adds_up_over_sequences():
    w = wl.make("tiny", device="cpu")
    one = [bench.sample_bytes(w, [s]) for s in range(w.num_seqs)]
    assert sum(one) == bench.sample_bytes(w, list(range(w.num_seqs)))
    # KV of every attended token once per kv head, plus q, out, table entries and the cache write
    e, D, Hkv, Hq = w.elem_bytes, w.head_dim, w.num_kv_heads, w.num_q_heads
    s = 0
    assert one[s] == (2 * w.lens_host[s] * Hkv * D * e + 2 * Hq * D * e + 4 * len(w.tables_host[s])
                      + 2 * 2 * Hkv * D * e)
