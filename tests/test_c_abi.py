"""The header is usable from plain C and from C++: tests/abi_check.c is
compiled with gcc (C99, pedantic, warnings as errors) and with g++ (C++17),
linked against libtwotower.so and run.  It checks status names, workspace
sizes and the host-side argument checks; no GPU is needed."""
import os
import shutil
import subprocess

import pytest

from block_wise_diffusion_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "abi_check.c")
INC = os.path.join(ROOT, "include")


@pytest.mark.parametrize("compiler,flags", [
    ("gcc", ["-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror"]),
    ("g++", ["-x", "c++", "-std=c++17", "-Wall", "-Wextra", "-Werror"]),
])
def test_header_compiles_links_and_runs(tmp_path, compiler, flags):
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not found")
    lib = build.build()
    libdir = os.path.dirname(lib)
    exe = str(tmp_path / "abi_check")
    subprocess.run([compiler, *flags, "-I", INC, SRC, "-x", "none", "-L", libdir, "-ltwotower",
                    f"-Wl,-rpath,{libdir}", "-o", exe], check=True, capture_output=True,
                   text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "abi_check: ok" in r.stdout
