"""include/flexattn.h is plain C: a C99 program compiled with gcc against it
links the library and gets the documented host-side answers (no GPU needed)."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc is not installed")
def test_c_program_uses_the_abi(tmp_path):
    from programmable_block_sparse_b200 import build
    build.build()
    pkg = os.path.join(ROOT, "programmable_block_sparse_b200")
    exe = tmp_path / "abi_consumer"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_consumer.c"), "-L", pkg, "-lflexattn_b200",
                    "-Wl,-rpath," + pkg, "-o", str(exe)], check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip().endswith("ok")
