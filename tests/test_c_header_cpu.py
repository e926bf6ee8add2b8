"""include/muon.h as a plain C99 header: a C program compiled with -std=c99
-Wall -Werror links against the built library and exercises the host-only calls
(no GPU needed)."""
import os
import shutil
import subprocess

import pytest

from muon_newton_schulz_04_b200 import build as mbuild

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c99_program_links_and_runs(tmp_path):
    lib = mbuild.build()
    exe = tmp_path / "abi_smoke"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", f"-I{os.path.join(ROOT, 'include')}",
                    os.path.join(HERE, "abi_smoke.c"), lib, f"-Wl,-rpath,{os.path.dirname(lib)}", "-o", str(exe)],
                   check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c abi ok" in r.stdout
