"""Host logic of bench.py that needs no GPU: the clock record taken during the timed region,
the gate that keeps a stored DRAM-traffic figure only while the kernel code it was
measured on is unchanged, and the peak figures' fallbacks."""

import json
import os
import shutil
import stat
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _fake_smi(tmp_path, rows):
    """An nvidia-smi stand-in on PATH that prints the given CSV rows and then waits."""
    script = tmp_path / "nvidia-smi"
    body = "".join(f"echo '{r}'\n" for r in rows)
    script.write_text("#!/bin/bash\n" + body + "exec sleep 30\n")
    script.chmod(script.stat().st_mode | stat.S_IEXEC)
    return str(tmp_path)


def _sample(monkeypatch, tmp_path, rows):
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, rows) + os.pathsep + os.environ["PATH"])
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.5)
    return s.stop()


IDLE = "Not Active"


def test_clock_record_median_and_no_reason(monkeypatch, tmp_path):
    rows = [f"0, {mhz}, 1965, 700.1, 0x0000000000000000, {IDLE}, {IDLE}, {IDLE}, {IDLE}"
            for mhz in (1965, 1950, 1965, 1800, 1965)]
    rec = _sample(monkeypatch, tmp_path, rows)
    assert rec == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 5}


def test_clock_record_names_active_reasons_and_skips_bad_rows(monkeypatch, tmp_path):
    rows = [f"0, 1300, 1965, 998.0, 0x0000000000000004, {IDLE}, {IDLE}, {IDLE}, Active",
            "0, [N/A], 1965, 998.0, 0x0, [N/A], [N/A], [N/A], [N/A]",
            f"0, 1310, 1965, 999.0, 0x0000000000000044, {IDLE}, Active, {IDLE}, Active",
            "garbage"]
    rec = _sample(monkeypatch, tmp_path, rows)
    assert rec["samples"] == 2 and rec["sm_mhz"] == 1305.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_clock_record_without_nvidia_smi(monkeypatch, tmp_path):
    monkeypatch.setenv("PATH", str(tmp_path))   # nothing to run
    s = bench.ClockSampler(0)
    s.start()
    assert s.stop() is None


def test_code_sha1_ignores_comments_only(tmp_path):
    a = tmp_path / "a.cu"
    a.write_text("int f(int x) {  // doubles\n\n  return 2 * x;\n}\n")
    b = tmp_path / "b.cu"
    b.write_text("// header comment\nint f(int x) {  // twice x\n  return 2 * x;   \n}\n")
    c = tmp_path / "c.cu"
    c.write_text("int f(int x) {\n  return 3 * x;\n}\n")
    assert bench.code_sha1(a) == bench.code_sha1(b)
    assert bench.code_sha1(a) != bench.code_sha1(c)


def _traffic_tree(tmp_path):
    """A copy of the repository's traffic record and kernel source under tmp_path."""
    (tmp_path / "profiles").mkdir()
    (tmp_path / "mha_mla_latent_b200" / "csrc").mkdir(parents=True)
    shutil.copy(os.path.join(ROOT, "mha_mla_latent_b200", "csrc", "chunk_tc.cu"),
                tmp_path / "mha_mla_latent_b200" / "csrc" / "chunk_tc.cu")
    src = tmp_path / "mha_mla_latent_b200" / "csrc" / "chunk_tc.cu"
    record = tmp_path / "profiles" / "attn_tc_traffic.txt"
    record.write_text("# test record\n"
                      f"source_sha1={bench.code_sha1(src)}\n"
                      "traffic_bytes.llama2_7b_bf16=138781952\n"
                      "traffic_bytes.llama2_7b_int4=312934400\n")
    return src


def test_traffic_gated_by_kernel_code_and_workload(monkeypatch, tmp_path):
    src = _traffic_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("llama2_7b_bf16", 3) == 138781952
    assert bench.measured_traffic("llama2_7b_int4", 3) == 312934400
    assert bench.measured_traffic("llama2_7b_ragged_bf16", 3) is None   # not captured
    assert bench.measured_traffic("llama2_7b_bf16", 1) is None          # CUDA-core kernel: none kept
    with open(src, "a") as f:
        f.write("// a comment at the end\n")
    assert bench.measured_traffic("llama2_7b_bf16", 3) == 138781952      # comments keep it
    with open(src, "a") as f:
        f.write("static int changed_code = 1;\n")
    assert bench.measured_traffic("llama2_7b_bf16", 3) is None           # code voids it


def test_committed_traffic_record_is_well_formed():
    """Every line of the committed record is a comment or key=value, with the SHA-1 key and
    integer byte counts per workload."""
    kv = {}
    with open(os.path.join(ROOT, "profiles", "attn_tc_traffic.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split("=", 1)
            kv[k] = v
    assert len(kv["source_sha1"]) == 40
    counts = {k: int(v) for k, v in kv.items() if k.startswith("traffic_bytes.")}
    assert "traffic_bytes.llama2_7b_bf16" in counts and all(v > 0 for v in counts.values())


def test_peak_fallbacks(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))   # no MEASURED_PEAKS.json there
    gbs, source = bench.measured_peak_hbm()
    assert gbs == bench.FALLBACK_HBM_GBS and source.startswith("fallback")
    assert bench.measured_peak_tflops() == bench.FALLBACK_BF16_TFLOPS
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 6551.0, "bf16_tflops": 1600.5}')
    gbs, source = bench.measured_peak_hbm()
    assert gbs == 6551.0 and source.startswith("measured")
    assert bench.measured_peak_tflops() == pytest.approx(1600.5)


def test_reference_arm_prints_one_contract_line(capsys, monkeypatch):
    """The reference arm (the float64 oracle on the host cores) prints exactly one JSON line
    with the bench contract's keys, its own e2e figure and the CPU-baseline description."""
    monkeypatch.setenv("RANK", "0")
    args = type("A", (), {"workload": "tiny_f32", "steps": 3, "warmup": 3, "gpus": 1})()
    assert bench.run_reference(args) == 0
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1
    line = json.loads(out[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 3 and line["warmup"] == 3
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT and line["higher_is_better"] is True
    assert line["value"] > 0 and line["ms_per_step"] > 0 and line["vs_baseline"] is None
    assert line["e2e"] == {"value": line["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["config"]["workload"] == "tiny_f32"
