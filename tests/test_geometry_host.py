"""Index math of the kernels (multiply-shift division, item decoding, tile rows,
token addressing with the cyclic shift) checked on the host against plain
integer arithmetic, by compiling the same header with g++."""
import os
import subprocess


def test_geometry_host(tmp_path):
    here = os.path.dirname(os.path.abspath(__file__))
    exe = tmp_path / "test_geometry"
    subprocess.run(["g++", "-O2", "-std=c++17", "-o", str(exe), os.path.join(here, "cpp", "test_geometry.cpp")],
                   check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout + r.stderr
