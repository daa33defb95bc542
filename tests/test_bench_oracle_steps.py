"""bench.py's CPU baseline and reference arm: whole oracle steps on worker
processes, reporting exactly the steps that ran and the worker count (CPU only)."""
import bench
import synth


def test_oracle_steps_report_what_ran():
    r = bench.oracle_timed("tiny", 2, 1)
    w = synth.WORKLOADS["tiny"]
    assert r["steps"] == 2 and r["warmup"] == 1
    assert 1 <= r["cores"] <= w.batch * w.n_kv_heads
    assert r["timed_misses"] == 0          # inputs were built in the untimed step
    assert r["ms_per_step"] > 0 and abs(r["total_s"] - 2 * r["ms_per_step"] / 1e3) < 1e-6
    assert abs(r["value"] - w.batch * w.q_tokens / (r["ms_per_step"] / 1e3)) < 1e-9 * r["value"]
    assert "2 whole decode steps" in bench.oracle_sample_text(r, w)


def test_both_arms_print_the_same_config():
    w = synth.WORKLOADS[bench.WORKLOAD]
    for n in (1, 2, 8):
        assert bench.base_config(w, n) == bench.base_config(synth.WORKLOADS[bench.WORKLOAD], n)
        assert bench.base_config(w, n)["parallelism"] == f"replicas x{n}"
