"""bench.py's reference arm (the oracle timed on host cores) keeps the JSON-line contract, and
under a multi-rank launch only rank 0 prints.  CPU only."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra, *args):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *args],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_json_line():
    r = _run({}, "--steps", "1", "--warmup", "3")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["steps"] == 1 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "llama3_8b_128k_b4"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_print_nothing():
    r = _run({"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"}, "--gpus", "2", "--steps", "1")
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]


def test_traffic_capture_digest_ignores_comments_and_debug_blocks(tmp_path):
    """A committed ncu capture stays attached to a kernel while only its comments, blank lines or
    #ifdef TQ_DEBUG blocks (compiled out of the timed library) change; any code change detaches it."""
    sys.path.insert(0, ROOT)
    import bench

    base = "int f(int x) {\n  int y = x + 1;\n  return y;\n}\n"
    variants_same = [
        "// header\nint f(int x) {\n  int y = x + 1;  // add\n\n  return y;\n}\n",
        "int f(int x) {\n  /* block\n     comment */\n  int y = x + 1;\n  return y;\n}\n",
        "int f(int x) {\n  int y = x + 1;\n#ifdef TQ_DEBUG\n  if (y < 0) return -1;\n#endif\n  return y;\n}\n",
    ]
    variants_diff = ["int f(int x) {\n  int y = x + 2;\n  return y;\n}\n",
                     "int f(int x) {\n  int y = x + 1;\n#ifdef OTHER\n  y = 0;\n#endif\n  return y;\n}\n"]

    def digest(text, name):
        p = tmp_path / name
        p.write_text(text)
        return bench.source_digest(str(p))

    d0 = digest(base, "base.cu")
    for i, v in enumerate(variants_same):
        assert digest(v, f"same{i}.cu") == d0, i
    for i, v in enumerate(variants_diff):
        assert digest(v, f"diff{i}.cu") != d0, i
