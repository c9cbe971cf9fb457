"""The range-checked build (libcsa2_checked.so, compiled with -DCSA2_CHECKED).

In that build the computed indices that the kernels' bounds rest on (the ordered list
writes of the select and of the shared-key cut, the attention cluster's merge rows, the
ticket merge's tile buffers, the cache append's local rows) are checked before their access and a
violation goes to the status word as CSA2_ERR_RANGE. Here a set of parity tests runs in a child process against that
library: they must pass, and no check may fire (every test checks the status word)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_cases_pass_on_the_checked_build():
    env = dict(os.environ, CSA2_LIBRARY="checked")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "gpu",
           os.path.join(ROOT, "tests", "test_gpu_parity.py"), os.path.join(ROOT, "tests", "test_gpu_decode_step.py"),
           "-k", "tiny or attention_shapes or stack20_schedule_small or paper or reindex or encoder_m2_every or append "
           "or shared_keys"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
