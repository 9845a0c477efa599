"""The parity suite once more under the checked build (liblapsum_checked.so,
-DLAPSUM_CHECKED): every computed index of a store or gather is tested on the
device (an index outside its buffer sets a status bit and the access is
skipped, never a trap) and guard words after every workspace buffer are
verified at the end of each call.  Any such error fails the run
(LAPSUM_ERR_BOUNDS).  It runs in a child process, so this process keeps the
normal library."""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_suite_under_the_checked_build():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    assert os.path.exists(os.path.join(ROOT, "exact_budget_soft_b200", "liblapsum_checked.so"))
    env = dict(os.environ, LAPSUM_CHECKED="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "gpu and not slow",
                        "tests/test_gpu_parity.py", "tests/test_gpu_edges.py", "tests/test_gpu_sharded.py"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert "passed" in r.stdout
