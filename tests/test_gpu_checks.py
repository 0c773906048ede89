"""The range-checked build (libmoe_checks.so): every data-dependent row index is compared
with its buffer's rows before the access.  The parity cases run with it in a child process
must raise no range flag and give the regular build's outputs bit for bit (the checks skip
nothing when every index is in range, and change no arithmetic)."""
import os
import subprocess
import sys

import pytest
import torch

from checks_cases import run_cases

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_checks_build_raises_no_flag_and_matches(moe, tmp_path):
    lib = os.path.join(os.path.dirname(HERE), "expert_router_top_b200", "libmoe_checks.so")
    assert os.path.exists(lib), "libmoe_checks.so is missing: run __graft_entry__.build()"
    assert not moe.checks_enabled() and moe.checks_read() == 0
    ref = {name: outs for name, (outs, _) in run_cases(moe).items()}
    path = tmp_path / "cases.pt"
    torch.save(ref, path)
    env = dict(os.environ, MOE_LIBRARY="checks")
    r = subprocess.run([sys.executable, os.path.join(HERE, "checks_child.py"), str(path)],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "0 problems" in r.stdout
