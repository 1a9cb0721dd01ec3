"""Host-side logic of bench.py that needs no GPU: argument checks and the
lookup of stored DRAM traffic, which must refuse counters taken from a kernel
source other than the current one."""
import hashlib
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("extra", [["--tokens", "0"], ["--workload", "kda_varlen", "--tokens", "128"]])
def test_tokens_override_is_checked_before_any_device_work(extra):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *extra],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 2
    assert "--tokens" in r.stderr


def test_stored_traffic_is_used_only_for_the_source_it_was_taken_from(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel source\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    rec = {"k": {"w": {"bytes": 1234, "source": "kernel.cu", "source_sha256_16": sha}}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("k", "w") == 1234
    assert bench.measured_traffic("k", "other") is None
    assert bench.measured_traffic("other", "w") is None
    src.write_text("// kernel source, changed\n")
    assert bench.measured_traffic("k", "w") is None


def test_gpu_count_must_match_the_ranks():
    """--gpus N without N ranks is refused before any device work (the bench
    never reports a one-GPU number under an N-GPU label)."""
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "8"],
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 2
    assert "WORLD_SIZE" in r.stderr
