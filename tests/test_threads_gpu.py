"""First forwards from two host threads at once (launch state is per device and locked)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_first_forwards_from_two_host_threads_match_the_oracle():
    # a fresh process, so that these are the library's first launches
    r = subprocess.run([sys.executable, os.path.join(HERE, "_first_forwards_two_threads.py")], capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout + r.stderr
