"""bench.py's host side without a GPU: the reference arm (the oracle) prints
one JSON line with the contract's keys, and the step's byte accounting."""
import json

import numpy as np

import bench
from paged_kv_cache_456_b200.workloads import build_workload


def test_reference_arm_prints_one_contract_line(capsys):
    bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1"])
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["config"]["workload"] == "tiny"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_step_bytes_fused_and_separate():
    w = build_workload("tiny")
    row = w.num_kv_heads * w.head_dim * w.elem_bytes
    live = int((w.context_lens > 0).sum())
    assert bench.step_bytes(w, fused=False) == w.decode_bytes() + 4 * live * row + 8 * live
    assert bench.step_bytes(w, fused=True) == w.decode_bytes() + 2 * live * row


def test_new_rows_per_sequence_layout():
    w = build_workload("tiny")
    k, v = w.new_rows_per_sequence()
    assert k.shape == (w.num_seqs, w.num_kv_heads, w.head_dim)
    live = np.nonzero(w.context_lens > 0)[0]
    assert np.array_equal(k[live].view(np.uint8), w.new_key.view(np.uint8))
    assert np.array_equal(v[live].view(np.uint8), w.new_value.view(np.uint8))


def test_dedup_flag_and_its_counters(capsys):
    # the reference arm names a deduplicated run in its config (same attention)
    bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "1",
                "--dedup"])
    d = json.loads([ln for ln in capsys.readouterr().out.splitlines() if ln.strip()][0])
    assert d["config"]["dedup"] is True
    # recorded DRAM counters are keyed per path; a deduplicated run's hash
    # also covers the shared-prefix pass
    assert bench.kernel_source_hash(True) != bench.kernel_source_hash()


def test_recorded_traffic_is_keyed_to_the_path_it_was_taken_on(tmp_path, monkeypatch):
    """A recorded DRAM count is reported only while its kernels' source is
    unchanged: decode entries follow the decode kernel, and the prefill and
    deduplicated entries also follow the tensor-core kernel."""
    rec = {"7b": {"kernel_source_hash": bench.kernel_source_hash(False), "dram_bytes_per_launch": 1},
           "prefill": {"kernel_source_hash": bench.kernel_source_hash(True), "dram_bytes_per_launch": 2},
           "prefix_cow+dedup": {"kernel_source_hash": bench.kernel_source_hash(False),
                                "dram_bytes_per_launch": 3}}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(path))
    assert bench.recorded_traffic("7b") == 1
    assert bench.recorded_traffic("prefill") == 2
    assert bench.recorded_traffic("prefix_cow+dedup") is None   # taken on another source
    assert bench.recorded_traffic("gqa70b") is None              # never taken


def test_default_run_times_the_four_large_workloads_headline_first():
    args = bench.parse_args([])
    names = bench.workload_names(args)
    assert names == ("long", "7b", "gqa70b", "prefix_cow", "prefill")
    # the headline is the largest step by algorithmic bytes
    sizes = {n: bench.step_bytes(build_workload(n), fused=True) for n in ("long", "7b")}
    assert sizes["long"] > 2 * sizes["7b"]
    assert bench.workload_names(bench.parse_args(["--workload", "tiny"])) == ("tiny",)
