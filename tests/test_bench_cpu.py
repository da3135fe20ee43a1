"""bench.py's host-side pieces and its reference arm (the oracle), on CPU."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from synthetic import workloads as W  # noqa: E402


def test_prefill_flops_of_the_35b_layer():
    # 2 * T*k * (H*2I + I*H) = 154.6 GFLOP for 2048 tokens, top-8, H=2048, I=768
    assert bench.prefill_flops(W.PREFILL_35B, 2048) == pytest.approx(154.618822656e9, rel=1e-12)


def test_expert_bytes_of_the_35b_layer():
    assert bench.expert_bytes_alg(W.DECODE_35B) == 3 * (2048 * 768 // 2 + 2048 * 768 // 16)


def test_ffn_launch_bytes_include_the_fused_combine():
    # 8 experts x 2,654,208 B of weights + x (T*H bf16) + y_part (T*k*H fp32) + y (T*H bf16)
    assert bench.ffn_alg_bytes(W.DECODE_35B, 1, 8) == 8 * 2654208 + 4096 + 65536 + 4096 == 21307392
    assert bench.ffn_alg_bytes(W.DECODE_35B, 8, 20) == 20 * 2654208 + 8 * 2048 * (2 + 8 * 4 + 2)


def test_overlap_efficiency_definition():
    assert bench.overlap_efficiency(10.0, 10.0, 4.0) == 1.0        # fully hidden
    assert bench.overlap_efficiency(14.0, 10.0, 4.0) == 0.0        # serialised
    assert bench.overlap_efficiency(12.0, 10.0, 4.0) == pytest.approx(0.5)
    assert bench.overlap_efficiency(12.0, 0.0, 4.0) is None


def test_traffic_ratio_needs_the_profiled_source(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    src = tmp_path / "expert_offload_fp4_b200" / "csrc"
    prof.mkdir()
    src.mkdir(parents=True)
    (src / "k.cu").write_text("kernel v1")
    import hashlib
    h = hashlib.sha256(b"kernel v1").hexdigest()
    (prof / "k.md").write_text(f"# k\n\n- dram_bytes_per_alg_byte: 1.25\n- source_sha256: {h}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic_ratio("k.md", "k.cu") == 1.25
    (src / "k.cu").write_text("kernel v2")            # changed since the capture
    assert bench.profiled_traffic_ratio("k.md", "k.cu") is None


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "2", "--warmup", "3", "--oracle-budget", "0.5"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["config"] == bench.decode_config(W.DECODE_35B, 1, 1)
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
