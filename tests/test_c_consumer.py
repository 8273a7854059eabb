"""The C ABI from plain C: tests/c/abi_consumer.c is compiled with gcc against include/w4a16.h and
linked to libw4a16.so (no Python, no PyTorch in that program), then run on the CPU.  It exercises
only what needs no GPU: size queries, argument validation and status strings."""
import os
import shutil
import subprocess

import pytest

from weight_only_int4_06_b200 import w4a16 as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_plain_c_program_uses_the_abi(tmp_path):
    if not os.path.exists(B.LIB_PATH):
        from weight_only_int4_06_b200 import build_lib
        build_lib.build()
    libdir = os.path.dirname(B.LIB_PATH)
    exe = str(tmp_path / "abi_consumer")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_consumer.c"), "-L", libdir, "-lw4a16",
                    f"-Wl,-rpath,{libdir}", "-o", exe], check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip().endswith("0 failed")
