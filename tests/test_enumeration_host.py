"""The library's tile enumeration and mask helpers, compiled for the host and
checked against a brute-force evaluation of the mask (no GPU needed)."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_tile_enumeration_is_exact(tmp_path):
    exe = str(tmp_path / "host_enum_check")
    subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-std=c++17", "-O2",
                           "-Wno-deprecated-gpu-targets", "-x", "cu",
                           os.path.join(ROOT, "tests", "host_enum_check.cu"), "-o", exe])
    r = subprocess.run([exe, "1500"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.startswith("OK"), r.stdout + r.stderr
