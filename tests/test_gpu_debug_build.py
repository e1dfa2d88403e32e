"""The bounds-checked build (libtcq_debug.so) on the small parity shapes.

compute-sanitizer is not used on this library's GPUs, so memory safety is
checked by the library itself: the TCQ_DEBUG build checks every global-memory
index of its encode, decode, matrix-vector and set-partitioned-trellis
kernels against the buffer it addresses and records a failure in the device
error word (tcq_device_errors).  tests/debug_build_run.py runs those kernels
on small seeded shapes through that build, in a process of its own (only one
build of the library may be loaded in a process), checks every result against
the oracle and requires the error word to stay clear.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_small_shapes_clean(cuda_device):
    from trellis_coded_weight_tcq_b200 import build

    build.build(debug=True)
    env = dict(os.environ, TCQ_LIBRARY="debug")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_build_run.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=420)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "DEBUG BUILD OK" in r.stdout


def test_device_error_word_is_clear_after_regular_calls(cuda_device):
    """The regular build's error word: no flag after encode, decode, matvec and
    the error-feedback driver (whose tensor-core waits report there)."""
    import numpy as np
    import torch

    from trellis_coded_weight_tcq_b200 import tcq, workloads

    assert tcq.device_errors() == 0
    wl = workloads.ldlq_random(16, 2, 256, 40, 1024, True, "f16", seed=3)
    tcq.ldlq(torch.from_numpy(wl.w).cuda(), torch.from_numpy(wl.u).cuda(),
             torch.from_numpy(wl.d).cuda(), torch.from_numpy(wl.codebook).cuda(), 16, 2, 256)
    x = torch.randn(64, 256, device="cuda")
    out = tcq.encode(x, None, tcq.MAD, 16, 2)
    tcq.decode(out.bits, out.start_state, tcq.MAD, 16, 2, 256)
    assert tcq.device_errors() == 0
    flags = tcq.ctypes.c_uint32(7)
    assert tcq.tcq_device_errors(None, tcq.ctypes.byref(flags)) == tcq.TCQ_OK and flags.value == 0
    assert np.isfinite(out.path_cost.cpu().numpy()).all()
