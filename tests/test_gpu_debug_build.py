"""The bounds-checked build, libkda_debug.so (compiled with KDA_DEBUG), on the GPU.

In that build every kernel checks the indices it derives from the call's data and
arithmetic against their extents and reports an out-of-range one in the status
word (KDA_ERR_DEVICE_BOUNDS) instead of making the access.  Two checks:

* the check itself: a checked write of a four-slot probe at an index outside it
  records BOUNDS and leaves the context usable;
* no false alarms and unchanged results: the small-shape parity tests (the
  oracle comparisons of tests/test_gpu_*.py, config-1-sized and ragged inputs,
  the segmented and windowed state passes)
  pass when run against the debug library, with a clean status word after every
  call that checks it.

The parity run is a child pytest process with KDA_LIB=debug, which makes the
binding load libkda_debug.so.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
IN_DEBUG_PROCESS = os.environ.get("KDA_LIB") == "debug"


@pytest.fixture(scope="module")
def kda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import gated_delta_rule_prologue_b200 as m
    return m


def test_index_check_records_bounds_and_skips_the_access(kda):
    if not kda.kda_debug_build():
        assert not IN_DEBUG_PROCESS, "KDA_LIB=debug, but the release library was loaded"
        pytest.skip("the release build has no index checks (runs in the KDA_LIB=debug process)")
    assert kda.kda_get_device_status() == 0
    for i in range(4):
        kda.kda_selftest_bounds(i)
    assert kda.kda_get_device_status() == 0
    for i in (4, -1, 1 << 20):
        kda.kda_selftest_bounds(i)
        assert kda.kda_get_device_status() == kda.KDA_ERR_DEVICE_BOUNDS
    # The context is still usable: a small prologue call runs clean.
    x = torch.randn((5, 3 * 2 * 16), device="cuda").to(torch.bfloat16)
    w = torch.randn((3 * 2 * 16, 4), device="cuda")
    q = torch.empty((5, 2, 16), device="cuda")
    k, v = torch.empty_like(q), torch.empty_like(q)
    kda.kda_prologue(x, w, q, k, v, H=2, D=16)
    assert kda.kda_get_device_status() == 0
    assert bool(torch.isfinite(q).all())


@pytest.mark.skipif(IN_DEBUG_PROCESS, reason="already the debug-build process")
def test_small_parity_suite_on_the_debug_build():
    lib = os.path.join(ROOT, "gated_delta_rule_prologue_b200", "libkda_debug.so")
    assert os.path.exists(lib), "libkda_debug.so is missing: run __graft_entry__.build()"
    env = dict(os.environ, KDA_LIB="debug")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_gpu_debug_build.py", "tests/test_gpu_parity.py",
           "tests/test_gpu_segmented.py", "tests/test_gpu_windowed.py", "tests/test_gpu_backward.py",
           "tests/test_gpu_degenerate.py", "tests/test_gpu_gate.py",
           "-k", "not full_size and not long_sequence and not k3"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    tail = r.stdout[-3000:] + r.stderr[-2000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail
