"""Host-side checks of bench.py's reporting logic (no GPU): the ncu DRAM
traffic figure of the roofline object is reported only while the kernel
sources it was captured on are unchanged, keyed by the MLA form's own sources,
and the peaks come from the measured file when it exists."""
import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_traffic_reported_only_for_matching_sources(bench, monkeypatch):
    good = bench.sources_hash("ffn", "absorbed")
    monkeypatch.setattr(bench, "TRAFFIC", {
        ("ffn", "w_same", "absorbed"): {"bytes": 1.5e7, "sha16": good},
        ("ffn", "w_stale", "absorbed"): {"bytes": 2.5e7, "sha16": "0" * 16},
    })
    assert bench.traffic_of("ffn", "w_same", "absorbed") == 1.5e7
    assert bench.traffic_of("ffn", "w_stale", "absorbed") is None    # sources changed since
    assert bench.traffic_of("ffn", "w_missing", "absorbed") is None  # never captured


def test_source_hash_follows_the_form_kernel(bench, monkeypatch):
    # the per-head form runs its own attention kernel: its figure must not be
    # invalidated by edits to the absorbed-form kernel, and vice versa
    per_head = bench.KERNEL_SOURCES[("attn", "per_head")]
    absorbed = bench.KERNEL_SOURCES["attn"]
    assert "attn_heads_sm100.cu" in per_head and "attn_sm100.cu" not in per_head
    assert "attn_sm100.cu" in absorbed and "attn_heads_sm100.cu" not in absorbed
    assert bench.sources_hash("attn", "per_head") != bench.sources_hash("attn", "absorbed")
    # steps without a form-specific list use the step's own list in both forms
    assert bench.sources_hash("ffn", "per_head") == bench.sources_hash("ffn", "absorbed")
    # every listed source exists (a missing file would make the hash meaningless)
    csrc = os.path.join(ROOT, "latent_attention_jagged_b200", "csrc")
    for names in bench.KERNEL_SOURCES.values():
        for n in names:
            assert os.path.exists(os.path.join(csrc, n)), n


def test_stored_traffic_entries_are_well_formed(bench):
    for (step, workload, form), t in bench.TRAFFIC.items():
        assert form in ("absorbed", "per_head")
        assert step in bench.KERNEL_SOURCES or (step, form) in bench.KERNEL_SOURCES
        assert t["bytes"] > 0 and len(t["sha16"]) == 16


def test_peaks_from_the_measured_file(bench):
    peaks = bench.load_peaks()
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            j = json.load(f)
        assert peaks["source"] == "measured"
        assert peaks["bf16_tflops"] == j["bf16_tflops"] and peaks["hbm_gbs"] == j["hbm_gbs"]
    else:
        assert peaks["source"] == "fallback"
    # the burst figure is the denominator; the sustained one is never above it
    assert peaks["bf16_tflops_sustained"] <= peaks["bf16_tflops"]


def _bench(args, env_extra):
    import subprocess
    import sys
    env = dict(os.environ, LLATTE_REF_STEP_S="0.5", **env_extra)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, env=env, cwd=ROOT,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    return r.stdout


def test_reference_arm_prints_one_line_with_the_contract_keys():
    # the oracle on the host cores, a bounded sample per step, the same metric
    # and workload as the CUDA arm's main line
    out = _bench(["--impl", "reference", "--steps", "1", "--warmup", "3"], {})
    lines = [l for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["metric"] == "user-seqs/s" and j["unit"] == "user-seqs/s"
    assert j["value"] > 0 and j["higher_is_better"] is True and j["steps"] == 1 and j["warmup"] == 3
    assert j["config"]["workload"] == "online"
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == j["value"] and cb["sample"]
    e = j["e2e"]
    assert e["value"] == j["value"] and e["unit"] == j["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_without_work():
    out = _bench(["--impl", "reference", "--steps", "1", "--warmup", "3"],
                 {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert out.strip() == ""
