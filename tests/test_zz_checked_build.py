"""The bounds-checked build (libinfllmv2_checks.so: device index checks that
set INFLLMV2_STATUS_CHECK and skip the access, in place of a memory
sanitizer) runs the smoke prefill and decode step against the oracle with no
check failing.  A separate process, since a process loads one build."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


def test_checked_build_runs_clean(cuda_lib):
    from trainable_block_sparse_compressed_b200 import build
    lib = build.build(checks=True)
    env = dict(os.environ, INFLLMV2_LIB=lib)
    r = subprocess.run([sys.executable, "-c", "import __graft_entry__ as g; g.smoke()"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    assert "smoke ok" in r.stdout
