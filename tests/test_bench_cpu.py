"""bench.py's reference arm on the CPU: the fp64 oracle timed on the host,
printing the one JSON line the measurement contract asks for."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny_fp32", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"].startswith("tiny_fp32")


def test_warmup_below_three_is_rejected():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--warmup", "2"],
                         capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0 and "warmup" in out.stderr


def test_traffic_record_needs_same_gemm_sources_and_launches(tmp_path, monkeypatch):
    """bench.py reports recorded GEMM DRAM traffic only for the workload it was
    captured on, with the same GEMM kernel / dispatch sources and the same GEMM
    launches per step; anything else gives null."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    sig = {"gemm.up_fwd": [12.0, 1855425871872], "gemm.o_fwd": [12.0, 463856467968]}
    rec = {"workload": "gpt2s_bf16", "sources_sha256": bench.gemm_sources_sha(), "gemm_launches": sig,
           "dram_bytes_per_launch": 123.0}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.recorded_traffic("gpt2s_bf16", dict(sig)) == 123.0
    assert bench.recorded_traffic("d32_bf16", dict(sig)) is None
    assert bench.recorded_traffic("gpt2s_bf16", dict(sig, **{"gemm.o_fwd": [24.0, 463856467968]})) is None
    path.write_text(json.dumps(dict(rec, sources_sha256="0" * 64)))
    assert bench.recorded_traffic("gpt2s_bf16", dict(sig)) is None
    # the launch signature: per label, launches and FLOPs per step
    prof = {"gemm.a": {"launches": 30, "flops": 3 * 2.0 * 128 * 256 * 64}, "rmsnorm_bwd": {"launches": 3, "flops": 0}}
    assert bench.gemm_launch_signature(prof, 3) == {"gemm.a": [10.0, 2 * 128 * 256 * 64]}
