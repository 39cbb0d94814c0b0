"""The C ABI from plain C: include/pa.h compiles as C11 and a C program linked against
libpa.so drives the host calls (pool, copy-on-write, beam re-selection, prefix cache).
CPU only; gcc builds the program into a temporary directory."""

import os
import shutil
import subprocess

import pytest

import paged_kv_cache_436_b200 as pa
from paged_kv_cache_436_b200 import build as pa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_library():
    if pa_build.stale():
        pa_build.build()
    return pa.lib()


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_and_host_calls_from_c(tmp_path):
    exe = tmp_path / "abi_host"
    lib_dir = os.path.dirname(pa.LIB_PATH)
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_host.c"), "-L", lib_dir, "-lpa", f"-Wl,-rpath,{lib_dir}",
           "-o", str(exe)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    assert run.stdout.startswith("c abi ok: ")
