"""The checking build (STEPQ_CHECK=1): tests/check_build_cases.py in a process
of its own, so that the binding loads libstepq_check.so."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_checking_build_cases():
    from quantized_recurrent_state_sm_b200 import build
    build.build(check=True)
    env = dict(os.environ, STEPQ_CHECK="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-s", "-p", "no:cacheprovider",
                        os.path.join("tests", "check_build_cases.py")], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=1200)
    print(r.stdout[-4000:])
    print(r.stderr[-2000:])
    assert r.returncode == 0
