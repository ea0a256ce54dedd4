"""The staged kernels under the bounds-checking build (libsparse_attn_bounds.so,
compiled with SA_DEBUG_BOUNDS): every shared-memory ring row a kernel reads is
checked against the rows it staged, every staging round against the ring's
size, and the query side's key-indexed weight writes against the workspace.
A violation sets bit 1 of the device error word instead of trapping, so this
build runs the staged parity cases -- both forwards, the backward and the
training pair, including the power-of-2 ladder at T = 4096 and the 32-offset
table -- in a child process, where tests/conftest.py checks the error word
after every test and the parity checks run as usual.
"""
import os
import subprocess
import sys

import pytest

import structured_sparse_attention_fibonacci_b200 as sa

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_staged_parity_cases_under_the_bounds_checking_build():
    assert os.path.exists(sa.BOUNDS_LIB_PATH), "build the library first (build.py)"
    env = dict(os.environ, SPARSE_ATTN_LIBRARY=sa.BOUNDS_LIB_PATH)
    which = subprocess.run([sys.executable, "-c", "import structured_sparse_attention_fibonacci_b200"
                            " as s; print(s.LIB_PATH)"], env=env, cwd=os.path.dirname(HERE),
                           capture_output=True, text=True, timeout=300)
    assert which.stdout.strip() == sa.BOUNDS_LIB_PATH, which.stdout + which.stderr
    cmd = [sys.executable, "-m", "pytest", os.path.join(HERE, "test_parity_gpu.py"), "-m", "gpu",
           "-q", "-x", "-p", "no:cacheprovider", "-k",
           "fast or pow2 or offsets32 or stagger or window64 or training_context"]
    r = subprocess.run(cmd, env=env, cwd=os.path.dirname(HERE), capture_output=True, text=True,
                       timeout=1200)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "error" not in r.stdout.splitlines()[-1], r.stdout[-2000:]
