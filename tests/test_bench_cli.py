"""bench.py's reference arm (the fp64 oracle on the host cores) runs without a
GPU, prints one JSON line with the contract's keys, measures the same
workload as the GPU arm, and maps none of the product's native code."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_its_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "2",
                        "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"] == "tiny"
    # the oracle's mask of every head: the tiny workload keeps 0.451171875 of its blocks (462 of 1024
    # pairs), the density the GPU arm measures with its own mask on the same inputs
    assert abs(line["config"]["density"] - 462 / 1024) < 1e-12
    # every timed step ran real work inside the time it reports
    assert line["ms_per_step"] > 0


def test_reference_arm_maps_no_native_code():
    code = ("import sys; sys.argv = ['bench.py', '--impl', 'reference', '--workload', 'tiny', '--steps', '1',"
            " '--warmup', '3']; import bench; bench.main(sys.argv[1:]);"
            " maps = open('/proc/self/maps').read(); print('LIBBSA' if 'libbsa' in maps else 'CLEAN')")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip().splitlines()[-1] == "CLEAN"


def test_package_import_maps_the_library_only_on_first_call():
    code = ("import block_sparse_attention_fractal_b200.synth, block_sparse_attention_fractal_b200 as b;"
            " m0 = 'libbsa' in open('/proc/self/maps').read();"
            " s = b.make_shape(1, 4, 16, 16, 2, 64, 64, 8); ok = b.validate_shape(s) == 0;"
            " m1 = 'libbsa' in open('/proc/self/maps').read(); print(m0, ok, m1)")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.split() == ["False", "True", "True"]


def test_recorded_traffic_follows_the_measured_kernel_source(tmp_path, monkeypatch):
    """The bench line's `traffic` comes from the committed ncu record only while
    the measured kernel's source and the shared headers are those it was taken
    from: a change to that kernel voids it, a change to another kernel does not."""
    import shutil
    sys.path.insert(0, ROOT)
    import bench
    rec = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))
    assert bench.recorded_traffic("attn", "wan480p") == rec["attn"]["bytes_per_launch"]
    assert bench.recorded_traffic("attn", "hunyuan720p") is None      # recorded on another workload
    csrc = tmp_path / "block_sparse_attention_fractal_b200" / "csrc"
    shutil.copytree(os.path.join(ROOT, "block_sparse_attention_fractal_b200", "csrc"), csrc)
    shutil.copytree(os.path.join(ROOT, "profiles"), tmp_path / "profiles")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("attn", "wan480p") == rec["attn"]["bytes_per_launch"]
    with open(csrc / "attn_bwd.cu", "a") as f:
        f.write("\n// another kernel's change\n")
    assert bench.recorded_traffic("attn", "wan480p") == rec["attn"]["bytes_per_launch"]
    with open(csrc / "attn_fwd.cu", "a") as f:
        f.write("\n// the measured kernel's change\n")
    assert bench.recorded_traffic("attn", "wan480p") is None
    assert bench.recorded_traffic("fine", "wan480p") == rec["fine"]["bytes_per_launch"]
    with open(csrc / "sm100.cuh", "a") as f:
        f.write("\n// a shared header's change\n")
    assert bench.recorded_traffic("fine", "wan480p") is None
