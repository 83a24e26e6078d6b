"""The debug-bounds build (libftmoe_debug.so, FT_DEBUG_BOUNDS=1) re-checks every permutation
(offsets, bijection with inv_pos, group membership, stability) and the decode slot table on
the device.  The layer and expert-stream parity tests run again against it in a child process:
they must pass, and no check may fire (each run ends in ft_moe_check).  The static-scratch
permutation is compared with the workspace permutation there too (its own status word is not
read back; the workspace call's is)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_parity_suite_passes_under_the_debug_bounds_build():
    from expert_offload_serving_router_b200 import build as ftbuild
    lib = ftbuild.build(debug_bounds=True)
    env = dict(os.environ, FTMOE_LIB=lib)
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_gpu_layer.py", "tests/test_gpu_route_permute.py", "tests/test_gpu_stream.py",
           "tests/test_zz_no_alloc.py",
           "-k", "not 4096 and not 8192 and not 2048"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail
