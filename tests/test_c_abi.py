"""The C ABI used from plain C: tests/c_abi_check.c is compiled as C11 with -Wall -Werror
against include/dsa.h, linked to the built libdsa.so and run (host-side calls only)."""
import shutil
import subprocess
from pathlib import Path

import pytest

import sparse_attention_17_b200 as dsa

ROOT = Path(__file__).resolve().parents[1]


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_against_the_header_and_library(tmp_path):
    lib = dsa.lib_path()
    if not lib.exists():
        pytest.skip("libdsa.so is not built")
    exe = tmp_path / "c_abi_check"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", f"-I{ROOT / 'include'}",
                    str(ROOT / "tests" / "c_abi_check.c"), "-o", str(exe),
                    f"-L{lib.parent}", "-ldsa", f"-Wl,-rpath,{lib.parent}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout + r.stderr
