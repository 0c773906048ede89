"""Runs the parity cases of test_gpu_checks.py with the range-checked library
(MOE_LIBRARY=checks) in a process of its own, and compares every output with the regular
library's outputs that the parent saved: usage  python checks_child.py CASES.pt"""
import os
import sys

_HERE = os.path.dirname(os.path.abspath(__file__))
sys.path[:0] = [_HERE, os.path.dirname(_HERE)]  # tests/ (gen, checks_cases) and the package
import torch  # noqa: E402

import expert_router_top_b200 as moe  # noqa: E402
from checks_cases import run_cases  # noqa: E402


def main():
    assert os.environ.get("MOE_LIBRARY") == "checks"
    assert moe.checks_enabled(), "the range-checked library did not load"
    assert moe.checks_read() == 0
    want = torch.load(sys.argv[1])
    got = run_cases(moe)
    bad = []
    for name, ref in want.items():
        flags = got[name][1]
        if flags:
            bad.append(f"{name}: range flags {flags}")
        for i, (a, b) in enumerate(zip(got[name][0], ref)):
            if not torch.equal(a, b):
                bad.append(f"{name}: output {i} differs from the regular build")
    print(f"checks build: {len(want)} cases, {len(bad)} problems")
    for b in bad:
        print(b)
    return 1 if bad else 0


if __name__ == "__main__":
    sys.exit(main())
