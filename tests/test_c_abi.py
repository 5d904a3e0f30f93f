"""The boundary from plain C: `tests/c_abi_demo.c` (C11, -pedantic -Werror) includes
both headers, takes the address of every entry point, links against libpa.so and runs
the calls that need no GPU (version, status strings, a block-manager step, refusals
before any launch)."""
import os
import shutil
import subprocess

import pytest

from paged_kv_cache_441_b200 import build as pa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_program_uses_the_library(tmp_path):
    lib = pa_build.build()
    exe = str(tmp_path / "c_abi_demo")
    libdir = os.path.dirname(lib)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                    os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_demo.c"),
                    "-L", libdir, "-l:libpa.so", f"-Wl,-rpath,{libdir}", "-o", exe],
                   check=True, capture_output=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
