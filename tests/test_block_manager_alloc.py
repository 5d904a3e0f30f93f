"""Failure atomicity of the host block manager under failed host allocations.

`tests/bm_alloc_fault.cpp` replaces operator new so that one chosen allocation inside a
manager call throws, for every allocation a seeded script of calls makes, and checks
that the call returns PA_ERR_HOST_ALLOC with nothing it can observe changed.  Host
only (g++), no GPU.  A copy of the manager with a planted mistake -- reference counts
raised before the allocation that can fail -- must be caught."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HARNESS = os.path.join(ROOT, "tests", "bm_alloc_fault.cpp")
MANAGER = os.path.join(ROOT, "paged_kv_cache_441_b200", "csrc", "pa_block_manager.cpp")

pytestmark = pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")


def _build_and_run(manager_src, out_dir):
    exe = os.path.join(out_dir, "bm_alloc_fault")
    subprocess.run(["g++", "-std=c++17", "-O1", "-Wno-mismatched-new-delete", "-I",
                    os.path.join(ROOT, "include"), HARNESS, manager_src, "-o", exe],
                   check=True, capture_output=True)
    return subprocess.run([exe], capture_output=True, text=True, timeout=300)


def test_every_failed_allocation_leaves_the_manager_unchanged(tmp_path):
    r = _build_and_run(MANAGER, str(tmp_path))
    assert r.returncode == 0, r.stdout + r.stderr
    _, runs, injected = r.stdout.split()
    assert int(injected) > 100  # the script's calls really allocate and really fail


def test_harness_catches_a_change_before_the_failing_allocation(tmp_path):
    src = open(MANAGER).read()
    old = ("        pa_block_manager::Seq &child = bm->seqs.emplace(child_id, it->second).first->second;\n"
           "        child.stamp = 0;\n"
           "        for (int b : child.blocks)\n"
           "            if (b >= 0) ++bm->refcount[b];\n")
    new = ("        for (int b : it->second.blocks)\n"
           "            if (b >= 0) ++bm->refcount[b];\n"
           "        pa_block_manager::Seq &child = bm->seqs.emplace(child_id, it->second).first->second;\n"
           "        child.stamp = 0;\n")
    assert src.count(old) == 1
    mutant = tmp_path / "pa_block_manager_mutant.cpp"
    mutant.write_text(src.replace(old, new))
    r = _build_and_run(str(mutant), str(tmp_path))
    assert r.returncode == 1 and "changed the manager" in r.stdout, r.stdout + r.stderr
