"""The C ABI from plain C: tests/c_abi/check_abi.c is compiled with the system C
compiler against include/ipttt.h, linked to libipttt.so and run (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

from chunk_wise_weight_gate_b200 import ipttt as ip

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_plain_c_program_uses_the_abi(tmp_path):
    ip.lib()  # builds nothing; fails loudly when the library is missing
    lib_dir = os.path.dirname(ip.LIB_PATH)
    exe = tmp_path / "check_abi"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi", "check_abi.c"), "-L", lib_dir, "-lipttt",
                    "-Wl,-rpath," + lib_dir, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert "C ABI checks passed" in r.stdout
