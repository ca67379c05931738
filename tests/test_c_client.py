"""The C ABI from plain C: tests/kvpop_client.c is compiled as C99 with warnings as errors against
include/kvpop.h, linked to the in-tree libkvpop.so (no Python, no PyTorch) and run; its calls only
exercise host-side validation and workspace sizes, so no GPU is needed."""
import os
import shutil
import subprocess

import pytest

from future_attention_targets_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c99_client_builds_links_and_passes(tmp_path):
    B.lib()   # builds nothing; fails loudly if libkvpop.so is missing
    libdir = os.path.dirname(B.LIB_PATH)
    exe = tmp_path / "kvpop_client"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "kvpop_client.c"), "-L", libdir, "-lkvpop",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "c client ok: abi 3" in out.stdout
