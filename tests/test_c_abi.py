"""The C ABI from plain C: tests/c/abi_check.c includes include/svg.h, links
libsvg_b200.so with gcc and runs the host-side checks (no GPU, no Python
types involved)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sparse_attention_video_svg_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_plain_c_client(tmp_path):
    lib = os.path.join(PKG, "libsvg_b200.so")
    assert os.path.exists(lib), "build the library first"
    exe = tmp_path / "abi_check"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_check.c"), "-o", str(exe),
                    "-L", PKG, "-lsvg_b200", f"-Wl,-rpath,{PKG}", "-lm"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    assert "c abi ok" in out.stdout
