"""The bench's oracle arm (`bench.py --impl reference`) runs on the host cores
alone, so its JSON line is checked here without a GPU: one line with the
metric, value and unit, the run's parameters, and the cpu_baseline and e2e
objects describing the run."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                         cwd=ROOT, capture_output=True, text=True, timeout=600, check=True)
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    for key in ("metric", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config"):
        assert key in d, key
    assert d["steps"] == 1 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_unknown_extra_workload_is_rejected():
    out = subprocess.run([sys.executable, "bench.py", "--extra", "nonsense"], cwd=ROOT, capture_output=True,
                         text=True, timeout=120)
    assert out.returncode != 0 and "unknown workload" in out.stderr


def _bench_module():
    import importlib.util

    spec = importlib.util.spec_from_file_location("bench_records", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    return bench


def test_roofline_unit_figures():
    """The per-unit figures behind `roofline.achieved`: per token and head at
    dk = dv = 128 in bf16, q, k, g (3 x 256 B), v (256 B), beta (2 B) read and
    o (256 B) written; FLOPs 6 dk dv for the state products, C (3 dk + 2 dv)
    for the intra-chunk ones at C = 64, C^2 / 3 for the inverse."""
    bench = _bench_module()
    assert bench.bytes_per_token_head() == 1282
    assert bench.bytes_per_token_head(esz=4) == 2564
    assert abs(bench.flops_per_token_head() - (98304 + 40960 + 4096 / 3)) < 1e-9


def test_profiled_traffic_matches_sources():
    """Each DRAM-traffic figure the bench reports comes from an ncu capture of
    the kernel source as it stands: the recorded sha1 prefix is the source's,
    and the profile summary it cites names that prefix."""
    import hashlib

    bench = _bench_module()
    assert bench.PROFILED_TRAFFIC
    for src, rec in bench.PROFILED_TRAFFIC.items():
        with open(os.path.join(ROOT, "gated_delta_rule_136_b200", src), "rb") as f:
            assert hashlib.sha1(f.read()).hexdigest()[:12] == rec["sha1"], src
        with open(os.path.join(ROOT, rec["profile"])) as f:
            assert rec["sha1"] in f.read(), rec["profile"]
        assert any(k.startswith("bytes_per_") and v > 0 for k, v in rec.items()), src
