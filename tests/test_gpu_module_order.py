"""The GPU test modules are collected in the order they were established (tests/conftest.py), so that
under -x a failure in a newer module cannot keep the older suites from running."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))


def test_gpu_modules_collect_established_first():
    import conftest
    r = subprocess.run([sys.executable, "-m", "pytest", HERE, "-m", "gpu", "--collect-only", "-q"],
                       capture_output=True, text=True, cwd=os.path.dirname(HERE), timeout=300)
    mods = []
    for line in r.stdout.splitlines():
        if "::" in line:
            m = os.path.basename(line.split("::")[0])
            if not mods or mods[-1] != m:
                mods.append(m)
    assert len(mods) == len(set(mods)), f"a module's tests are not contiguous: {mods}"
    ordered = [m for m in conftest._GPU_MODULE_ORDER if m in mods]
    assert [m for m in mods if m in conftest._GPU_MODULE_ORDER] == ordered
    assert set(mods) <= set(conftest._GPU_MODULE_ORDER), f"GPU module without a place in the order: {mods}"
