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


def test_reference_arm_reports_the_same_config_as_the_gpu_arm(capsys):
    """The oracle arm times bounded samples of the same workload and prints
    the config dict the GPU arm prints for the same arguments."""
    import argparse
    import json

    args = argparse.Namespace(config="tiny", seed=0, max_seqs=None, warmup=3, steps=3, ref_budget_s=0.2,
                              partition_blocks=None, kv="bf16")
    bench.run_reference(args)
    line = json.loads(capsys.readouterr().out)
    w = wl.make("tiny", device="cpu")
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "GB/s"
    assert line["config"] == bench.workload_config(w, bench.resolve_partition_blocks(w.partition_blocks), "bf16")
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["step_ms"]["min"] <= line["step_ms"]["median"]
