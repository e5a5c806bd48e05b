"""bench.py's host logic without a GPU: the comment-insensitive source hash that
decides whether a committed ncu capture still describes the kernel, the reading of
a capture summary, and the reference arm's JSON line (the CPU oracle on a bounded
sample), which the benchmark contract fixes key by key."""
import importlib.util
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_source_hash_ignores_comments_and_blank_space(tmp_path):
    b = _bench()
    a, c, d = tmp_path / "a.cu", tmp_path / "c.cu", tmp_path / "d.cu"
    a.write_text("int f(int x) {\n    return x + 1;  // one\n}\n")
    c.write_text("/* a block\n   comment */\nint f(int x)\n{\n  return x + 1;\n}\n// trailing\n")
    d.write_text("int f(int x) {\n    return x + 2;\n}\n")
    assert b.source_hash([str(a)]) == b.source_hash([str(c)])
    assert b.source_hash([str(a)]) != b.source_hash([str(d)])


def test_profiled_traffic_only_for_the_captured_source(tmp_path, monkeypatch):
    b = _bench()
    src = tmp_path / "k.cu"
    src.write_text("__global__ void k() {}\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    h = b.source_hash([str(src)])
    (prof / "k.md").write_text(f"# k\n\n- source_sha256: `{h}`\n- dram_bytes_per_full_launch: `123456`\n")
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    assert b.profiled_traffic("k.md", [str(src)]) == 123456
    src.write_text("__global__ void k() { int changed; }\n")
    assert b.profiled_traffic("k.md", [str(src)]) is None      # the kernel changed since
    assert b.profiled_traffic("missing.md", [str(src)]) is None


def test_committed_combine_summary_is_readable():
    b = _bench()
    p = os.path.join(ROOT, "profiles", "combine_kernel_normal_4096x7168.md")
    text = open(p).read()
    assert "- source_sha256: `" in text and "- dram_bytes_per_full_launch: `" in text
    assert "--clock-control none" in text


def test_reference_arm_json_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "3",
                          "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["steps"] == 3 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["config"]["workload"].startswith("normal")
    # the same config object as the GPU arm prints for this workload: what the work is,
    # not how this arm samples it
    assert set(line["config"]) == {"workload", "tokens_per_gpu", "hidden", "topk", "experts",
                                   "partitions", "recv_rows", "bytes_per_step", "seed", "l2",
                                   "parallelism"}
    assert line["config"]["tokens_per_gpu"] == 4096 and line["config"]["recv_rows"] == 32768
    assert 1 <= line["sample_tokens"] <= 4096
    assert line["cpu_baseline"]["cores"] >= 1 and line["cpu_baseline"]["host_cores"] >= 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
