"""The plain-C program examples/heta_run.c builds against include/heta.h
and libheta.so, and turns bad arguments and missing inputs into a non-zero
exit before it touches a GPU."""
import subprocess

from uncertainty_routed_heterogeneous_b200 import build as heta_build


def test_c_program_builds_and_refuses_bad_arguments(tmp_path):
    exe = heta_build.build_example()
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 1 and "usage" in r.stderr
    r = subprocess.run([exe, str(tmp_path)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 1 and "meta.txt" in r.stderr
    (tmp_path / "meta.txt").write_text("1 2 64 4 8 8 3 3 3 256 0.25\n")
    r = subprocess.run([exe, str(tmp_path)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 1 and "q.bin" in r.stderr
