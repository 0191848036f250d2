"""The C ABI used from plain C: tests/c_abi_check.c is compiled as C99 with every warning
an error against include/vt.h, linked against the in-tree libvt.so, and run.  It makes
host-only calls (configuration checks, error messages, the workspace plan, index maps),
so no GPU is needed."""
import os
import shutil
import subprocess

import pytest

from vision_transformer_encoder_vit_b200 import vt as V

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_program_builds_against_the_header_and_runs(tmp_path):
    lib_dir = os.path.dirname(V.lib._name)
    exe = str(tmp_path / "c_abi_check")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-O1",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_check.c"),
           "-o", exe, "-L", lib_dir, "-l:libvt.so", f"-Wl,-rpath,{lib_dir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c abi ok" in r.stdout
