"""The boundary is a C ABI: a plain C99 program that includes
``include/verify_attn.h`` must compile with ``-std=c99 -pedantic -Werror``,
link against the library and run its host-only calls without a GPU."""
import os
import shutil
import subprocess

import pytest

import mla_speculative_verify_absorb_b200 as va

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c99_consumer_compiles_links_and_runs(tmp_path):
    lib_dir = os.path.dirname(va.lib_path())
    exe = str(tmp_path / "abi_consumer")
    cmd = ["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_consumer.c"),
           "-L", lib_dir, "-lverify_attn", f"-Wl,-rpath,{lib_dir}", "-o", exe]
    build = subprocess.run(cmd, capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "c abi consumer ok" in run.stdout
