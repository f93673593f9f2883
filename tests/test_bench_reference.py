"""bench.py's reference arm (the fp64 oracle timed on the host cores) on the CPU: one JSON
line with the contract's keys, the same workload description as the GPU arm, and
nothing from ranks other than 0."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None):
    env = dict(os.environ)
    env.update(extra_env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                           "--steps", "1", "--warmup", "0"], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=600)


def test_reference_line():
    r = _run()
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["higher_is_better"] is True and d["steps"] == 1 and d["warmup"] == 0
    cfg = d["config"]
    # tiny: one 24 x 24 image merged 2 x 2, no tiling
    assert cfg["workload"] == "tiny" and cfg["merged_tokens"] == 144 and cfg["assembled_rows"] == 144
    assert cfg["k"] == 2 and cfg["tiling"] == "none" and cfg["layernorm"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_other_ranks_print_nothing():
    r = _run({"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [x for x in r.stdout.splitlines() if x.startswith("{")]


def test_images_override_scales_the_sequences():
    """--images keeps the workload's shapes and scales its sequences with the image count."""
    import argparse
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    stress = W.WORKLOADS["stress"]
    wl = bench.pick_workload(argparse.Namespace(workload="stress", images=16))
    assert (wl.n_images, wl.B, wl.S, wl.k, wl.C, wl.N1) == (16, 1, stress.S, stress.k, stress.C, stress.N1)
    wl = bench.pick_workload(argparse.Namespace(workload="moonvit", images=4))
    assert (wl.n_images, wl.B) == (4, 4)
    assert bench.pick_workload(argparse.Namespace(workload="vl2", images=0)) is W.WORKLOADS["vl2"]


def test_code_only_ignores_comments_and_blank_lines():
    """The stored DRAM counters stay keyed to the kernels' code: comment edits keep the
    key, code edits change it."""
    sys.path.insert(0, ROOT)
    import bench
    a = "int x = 1;  // one\n\n// a note\nint y = 2;\n"
    b = "int x = 1;  // the first\n// another note\nint y = 2;   \n\n"
    c = "int x = 1;\nint y = 3;\n"
    assert bench.code_only(a) == bench.code_only(b) == "int x = 1;\nint y = 2;"
    assert bench.code_only(c) != bench.code_only(a)
    assert bench.code_only('printf("//");') == 'printf("//");'
