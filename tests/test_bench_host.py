"""Host-side logic of bench.py, on the CPU (no GPU).

* The traffic-record key (`_code_sha`) ignores comments and blank lines but
  changes with any code edit, so a committed ncu DRAM figure is reported only
  for the kernel source it was measured on.
* `_traffic` scales a matching record by the units of a launch and returns None
  for a stale or missing one.
* The reference arm (`--impl reference`, the CPU oracle on the host cores)
  prints one JSON line with the fields the benchmark contract names.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

import bench  # noqa: E402  (ROOT is on sys.path via conftest)

CODE = """// header comment
#include <x.h>
/* block
   comment */
__global__ void k(float *p) {   // trailing comment
    p[0] = 1.f;

}
"""


def test_code_sha_ignores_comments_and_blank_lines():
    reworded = CODE.replace("// header comment", "// another header\n// and one more line")
    reworded = reworded.replace("/* block\n   comment */", "/* other */")
    assert bench._code_sha(CODE) == bench._code_sha(reworded)
    assert bench._code_sha(CODE) == bench._code_sha(CODE + "\n\n// tail\n")


def test_code_sha_changes_with_the_code():
    assert bench._code_sha(CODE) != bench._code_sha(CODE.replace("1.f", "2.f"))
    assert bench._code_sha(CODE) != bench._code_sha(CODE.replace("p[0]", "p[1]"))


def _fake_tree(tmp_path, record_sha):
    csrc = tmp_path / "linear_attention_serving_prefill_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text(CODE)
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "dram_traffic.json").write_text(json.dumps({
        "my_kernel": {"source_sha": record_sha, "dram_bytes_per_token_head": 1500.5}}))


def test_traffic_record_used_only_for_its_source(tmp_path, monkeypatch):
    _fake_tree(tmp_path, bench._code_sha(CODE))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic("k.cu", "my_kernel", 1000) == pytest.approx(1500.5 * 1000)
    assert bench._traffic("k.cu", "other_kernel", 1000) is None


def test_traffic_record_is_null_once_the_source_changed(tmp_path, monkeypatch):
    _fake_tree(tmp_path, bench._code_sha(CODE.replace("1.f", "2.f")))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic("k.cu", "my_kernel", 1000) is None


def test_traffic_without_a_record_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic("k.cu", "my_kernel", 1000) is None


def test_single_rank_max_is_the_value():
    assert bench.max_over_ranks(3.25, 1) == 3.25


def test_reference_arm_prints_the_contract_line():
    env = dict(os.environ, RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "tokens/s"
    # At least 3 warm-up steps whatever is asked for (the timing rules).
    assert d["higher_is_better"] is True and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["dtype"] == "f64" and d["data"] == "synthetic"
    assert d["config"]["workload"].startswith("prefill_32k (B=1,H=96,T=32768")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert "token-heads" in cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s",
                        "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_print_nothing():
    env = dict(os.environ, RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert not [l for l in out.stdout.splitlines() if l.startswith("{")]


@pytest.mark.parametrize("extra", [[], ["--impl", "reference", "--prefill-only"]])
def test_varlen_workload_is_prefill_only(extra):
    """The 16-sequence resume workload times the prefill leg alone; asking for the
    other legs (or the reference arm) is refused on the host before any work."""
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "varlen_resume",
                          "--steps", "1"] + extra,
                         cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 2
    assert "varlen_resume workload runs the prefill leg alone" in out.stderr
