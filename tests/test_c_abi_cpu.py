"""The C ABI from plain C: tests/c_abi_check.c is compiled as strict C99 against
include/dsa.h, linked against the built library, and run on the CPU (argument checks,
workspace sizes and status strings only; nothing reaches a kernel launch)."""
import os
import shutil
import subprocess

import pytest

import deepseek_sparse_attention_head_b200 as dsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_caller_compiles_links_and_passes(tmp_path):
    lib_dir = os.path.dirname(dsa._LIB_PATH)
    exe = tmp_path / "c_abi_check"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi_check.c"), "-L", lib_dir, "-ldsa_b200", f"-Wl,-rpath,{lib_dir}",
           "-o", str(exe)]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    p = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert p.returncode == 0 and p.stdout.strip().endswith("OK 0"), p.stdout + p.stderr
