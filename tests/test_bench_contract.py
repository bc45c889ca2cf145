"""bench.py on the CPU: its byte and flop counts, the per-sequence lambda of the ragged
batch, and the JSON line of the reference arm (the oracle timed on host cores), which
needs no GPU."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_algorithmic_bytes_counts_each_term_once():
    # two sequences of 300 and 200 cached rows, budgets 100 and 50, window 4, G = 2,
    # one layer, three KV heads, 7 rows moved over the whole launch
    n_tok, budgets, G, w = (300, 200), (100, 50), 2, 4
    per_seq = [256 * (300 + 8) + 8 * 296 + 4 * 100, 256 * (200 + 8) + 8 * 196 + 4 * 50]
    want = 3 * sum(per_seq) + 1024 * 7
    assert bench.algorithmic_bytes(n_tok, budgets, 1, 3, G, w, 7) == want
    # layers and heads scale the per-unit part, not the moved rows (already a launch total)
    assert bench.algorithmic_bytes(n_tok, budgets, 2, 3, G, w, 7) == 2 * 3 * sum(per_seq) + 1024 * 7


def test_gram_executed_flops_counts_the_symmetric_tile_pairs():
    one = 2 * 128 ** 3
    assert bench.gram_executed_flops(1, 8) == one
    assert bench.gram_executed_flops(128, 8) == one
    assert bench.gram_executed_flops(129, 8) == 3 * one          # (0,0), (0,1), (1,1)
    assert bench.gram_executed_flops(2176, 8) == 17 * 18 // 2 * one


def test_ragged_lambda_cycles_over_the_two_ablations_and_the_default():
    w = bench.WORKLOADS["ragged_batch"]
    assert [bench.lambda_of(w, b) for b in range(6)] == [0.0, 0.1, 1.0, 0.0, 0.1, 1.0]
    w8 = bench.WORKLOADS["llama3_8b_step"]
    assert bench.lambda_of(w8, 5) == w8.mix_lambda


def test_reference_arm_prints_one_json_line_with_the_contract_keys():
    env = dict(os.environ)
    env.pop("RANK", None)
    env.pop("WORLD_SIZE", None)
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 0
    assert d["higher_is_better"] is True and d["value"] > 0
    assert d["config"]["workload"] == "ragged_batch"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert isinstance(cb["sample"], str) and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_profiled_traffic_follows_the_kernel_sources(tmp_path, monkeypatch):
    # a committed ncu summary counts only while the kernel's sources hash to its digest
    path = tmp_path / "summary.traffic.txt"
    monkeypatch.setattr(bench, "profile_traffic_path", lambda kernel, workload, variant="": str(path))
    digest = bench.kernel_source_digest("rkv_unit_kernel")
    path.write_text("# dram bytes\nkernel_source_sha256_16: %s\nunits_per_launch: 8\n"
                    "dram_bytes_per_unit: 1000\n" % digest)
    assert bench.profiled_traffic("rkv_unit_kernel", "w", 16) == 16000
    path.write_text("kernel_source_sha256_16: %s\ndram_bytes_per_unit: 1000\n" % ("0" * 16))
    assert bench.profiled_traffic("rkv_unit_kernel", "w", 16) is None
    path.unlink()
    assert bench.profiled_traffic("rkv_unit_kernel", "w", 16) is None


def test_committed_traffic_summaries_name_a_known_kernel_and_their_units():
    # every summary under profiles/ parses, names a timed kernel and gives a per-unit figure
    prof = os.path.join(ROOT, "profiles")
    names = [n for n in os.listdir(prof) if n.endswith(".traffic.txt")]
    assert names
    for n in names:
        kernel = n.split(".")[0]
        assert kernel in bench.KERNEL_SOURCES, n
        kv = {}
        with open(os.path.join(prof, n)) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    kv[k.strip()] = v.strip()
        assert len(kv["kernel_source_sha256_16"]) == 16, n
        assert int(kv["units_per_launch"]) > 0 and int(kv["dram_bytes_per_unit"]) > 0, n
