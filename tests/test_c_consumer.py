"""The C ABI from plain C: tests/c_consumer.c is compiled with gcc as C11
against include/sdm.h, linked to the in-tree library, and run (no GPU needed)."""

import shutil
import subprocess
from pathlib import Path

import pytest

from sparse_memory_linear_pkm_b200 import build as build_mod

ROOT = Path(__file__).resolve().parent.parent


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_plain_c_program_uses_the_abi(tmp_path):
    lib = Path(build_mod.build())
    exe = tmp_path / "c_consumer"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", str(ROOT / "include"),
                    str(ROOT / "tests" / "c_consumer.c"), "-o", str(exe), str(lib),
                    f"-Wl,-rpath,{lib.parent}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert "c consumer ok" in out.stdout
