"""include/ttt.h from plain C: compile tests/c_abi_check.c as C99 against the header, link it to
libttt.so and run it (host-only calls; no GPU needed)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_is_plain_c_and_host_calls_work(libttt, tmp_path):
    lib_dir = os.path.dirname(libttt.LIB_PATH)
    exe = tmp_path / "c_abi_check"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    os.path.join(HERE, "c_abi_check.c"), "-o", str(exe), "-L", lib_dir, "-lttt",
                    "-Wl,-rpath," + lib_dir], check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True)
    print(res.stdout)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "FAIL" not in res.stdout
