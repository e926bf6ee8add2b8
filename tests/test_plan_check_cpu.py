"""The library's host-side plan check (run before any launch with a new plan):
compiled here with the planner sources and a C++ driver that feeds it every plan
the planner builds for a range of shapes, cluster counts and split modes (all must
pass) and plans with planted defects (each must be reported)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "muon_newton_schulz_04_b200", "csrc")


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_plan_check(tmp_path):
    exe = tmp_path / "plan_check"
    subprocess.run(["g++", "-std=c++17", "-O1", "-Wall", f"-I{CSRC}", os.path.join(HERE, "plan_check.cpp"),
                    os.path.join(CSRC, "plan.cpp"), "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "plan check ok" in r.stdout
