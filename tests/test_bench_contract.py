"""bench.py's output contract, checked on the CPU through its reference arm
(the fp64 oracle timed on the host cores): one JSON line with the metric,
the whole-job value, the timing and workload fields, and the reference arm's
own cpu_baseline and zero-copy e2e block."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, res.stdout
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["n_gpus"] == 1 and d["steps"] == 1
    assert d["warmup"] >= 3  # at least three untimed steps, whatever was asked
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["unit"] == "tokens/s" and d["dtype"] == "f64"
    assert isinstance(d["config"].get("workload"), str) and "model" not in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_attention_sources_follow_the_kernel():
    sys.path.insert(0, ROOT)
    import bench
    # the CTA-pair kernel (128 heads) is built from one more header than the
    # one-CTA kernel, so its committed traffic is keyed by that header too
    for w in ("v2", "v2_fp8", "long", "prefill"):
        assert "tc_attn2.cuh" in bench.attention_sources(w)
    for w in ("lite", "lite_fp8"):
        assert bench.attention_sources(w) == ("common.cuh", "tc_attn.cuh")
    assert bench.kernel_source_hash("v2") == bench.kernel_source_hash("v2_fp8")
    assert bench.kernel_source_hash("v2") != bench.kernel_source_hash("lite")


def test_gpus_flag_must_match_the_launched_ranks():
    # under torch.distributed.run the rank count is WORLD_SIZE; a different
    # --gpus is refused before any work
    env = dict(os.environ, WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "4", "--impl", "reference"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert res.returncode != 0
    assert "--gpus 4 but 2 rank(s)" in res.stderr
    assert res.stdout.strip() == ""


def test_attention_tokens_per_s_is_whole_job_rows_over_the_stage_time():
    sys.path.insert(0, ROOT)
    import bench
    # 64 rows per call in 0.140 ms on each of 2 ranks
    assert bench.attention_tokens_per_s(2, 64, 0.140) == round(2 * 64 / 0.140e-3, 1)
    assert bench.attention_tokens_per_s(1, 64, 0.0) is None
