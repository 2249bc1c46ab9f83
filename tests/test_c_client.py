"""include/bbc.h as a plain C99 header: a C program compiled with gcc against it, linked to
libbbc.so, runs the host-side validation paths (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_c99_client_compiles_links_and_validates(tmp_path):
    from blockwise_bit_codebook_b200 import build
    lib = build.build()
    libdir = os.path.dirname(lib)
    exe = tmp_path / "abi_host_check"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi", "abi_host_check.c"), "-o", str(exe),
           "-L", libdir, "-l:" + os.path.basename(lib), "-Wl,-rpath," + libdir]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "c abi ok" in out.stdout
