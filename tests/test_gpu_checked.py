"""The GPU parity suites run again against the checked build.

libmilo_checked.so is the library compiled with MILO_CHECKED: every kernel of
the forward path checks its copy ranges and indices against its buffers, and
instead of making an access out of range it skips it and flags
MILO_DEV_BOUNDS.  The parity tests assert a zero device status after every
call, so running them against the checked build shows that no index of the
routing, preparation, both grouped GEMMs (t-items included), the compensator
down-projection and the combine leaves its buffer on any of their shapes and
edge cases -- the stand-in for a memory checker, which this pool does not
offer.  The suites run in a child process (MILO_LIBRARY=checked), whose
library the child confirms before it starts.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_suites_pass_on_the_checked_build():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from int3_gemm_rank_b200 import build
    build.build(checked=True)
    env = dict(os.environ, MILO_LIBRARY="checked")
    probe = subprocess.run(
        [sys.executable, "-c",
         "import int3_gemm_rank_b200 as m; m.lib(); "
         "assert m.LIB_PATH.endswith('libmilo_checked.so'), m.LIB_PATH; print(m.LIB_PATH)"],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert probe.returncode == 0, probe.stdout + probe.stderr
    r = subprocess.run(
        [sys.executable, "-m", "pytest", "tests/test_gpu_parity.py", "tests/test_gpu_scale.py",
         "tests/test_zz_no_alloc.py", "-m", "gpu", "-x", "-q", "-p", "no:cacheprovider"],
        cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
