"""The benchmark's reference arm (the oracle, timed on the host cores) keeps
the JSON-line contract on CPU: one line on rank 0 with the contract's keys,
nothing and exit 0 on the other ranks."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--config", "tiny", "--steps", "2", "--warmup", "3"],
                          capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)


def test_reference_arm_prints_one_contract_line():
    r = _run({"RANK": "0", "WORLD_SIZE": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    r = _run({"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_profile_hash_ignores_debug_only_blocks():
    """A committed ncu summary is tied to the product kernel by a hash of the
    kernel sources with every `#ifdef MQA_DEBUG` block removed (code of the
    debug build only), its `#else` branch kept, nested conditionals inside a
    removed block removed with it."""
    sys.path.insert(0, ROOT)
    import bench

    src = ("a\n#ifdef MQA_DEBUG\nx\n#if Y\ny\n#endif\nz\n#endif\nb\n"
           "#ifdef MQA_DEBUG\np\n#else\nq\n#endif\n#ifdef OTHER\nr\n#endif\n")
    assert bench.product_source(src) == "a\nb\nq\n#ifdef OTHER\nr\n#endif\n"
    # the product sources: stripping changes nothing but the debug blocks, so
    # every committed summary's hash still matches its kernel
    for kind, name in (("fp8", "decode"), ("fp4", "fp4"), ("nvfp4", "nvfp4")):
        path = os.path.join(ROOT, "profiles", f"{kind}_logits_{name}.md")
        tag = [ln for ln in open(path) if ln.startswith("<!-- source_hash=")][0]
        assert bench.source_hash(bench.SOURCES_OF_KIND[kind]) == tag.split("=")[1].split()[0], kind
