"""The allocation-free encoder (tcq_encode_static_scratch) against tcq_encode.

Some callers cannot allocate device memory (their own pool owns the GPU, or a
latency-critical path must not call cudaMalloc); for them the library offers an
encoder whose scratch is a static device array inside the library.  This test
calls it through the C ABI twice in a row, on different inputs, so the second
call runs on whatever the first left in the shared scratch, and checks each
result against tcq_encode's on the same inputs with the tolerance the parity
tests use.  It lives in its own file, collected last, and passes both alone in
a fresh process and after the other tests (the first call on a device does the
one-time set-up either way).
"""
import ctypes

import numpy as np
import pytest

from tests.parity import ABS_TOL_PER_D, REL_TOL, gpu_encode, sum_d
from trellis_coded_weight_tcq_b200 import tcq, workloads

pytestmark = pytest.mark.gpu


def _static_scratch_encode(wl):
    import torch

    dev = torch.device("cuda", 0)
    x = torch.from_numpy(wl.x).to(dev)
    d = None if wl.d is None else torch.from_numpy(wl.d).to(dev)
    cb = torch.from_numpy(wl.codebook).to(dev)
    W = tcq.tcq_words_per_block(wl.k, wl.T)
    start = torch.empty(wl.n_blocks, dtype=torch.int32, device=dev)
    bits = torch.empty((wl.n_blocks, W), dtype=torch.int32, device=dev)
    cost = torch.empty(wl.n_blocks, dtype=torch.float32, device=dev)
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = tcq.tcq_encode_static_scratch(P(x), P(d), P(cb), tcq.cb_dtype_of(cb), wl.L, wl.k, wl.T,
                                       wl.n_blocks, P(start), P(bits), P(cost),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == tcq.TCQ_OK, tcq.tcq_status_string(st)
    torch.cuda.synchronize()
    return (start.cpu().numpy().view(np.uint32), bits.cpu().numpy().view(np.uint32),
            cost.cpu().numpy())


def _path_cost(wl, start, bits):
    from oracle import oracle_decode, oracle_path_cost

    y = oracle_decode(bits, start, wl.codebook, wl.L, wl.k, wl.T)
    return oracle_path_cost(wl.x, wl.d, y)


def test_static_scratch_encoder_matches_tcq_encode_on_two_calls_in_a_row(cuda_device):
    # more blocks than the static scratch holds CTAs at L=16, so each CTA runs
    # several rounds; the second call sees the first call's leftovers
    cases = [workloads.small_random(16, 2, 256, 64, True, "f16", seed=901),
             workloads.small_random(16, 2, 256, 64, False, "f16", seed=902)]
    for wl in cases:
        s_ref, b_ref, c_ref = gpu_encode(wl)
        s_new, b_new, c_new = _static_scratch_encode(wl)
        J_ref = _path_cost(wl, s_ref, b_ref)
        J_new = _path_cost(wl, s_new, b_new)
        tol = REL_TOL * J_ref + ABS_TOL_PER_D * sum_d(wl)
        assert np.all(np.abs(J_new - J_ref) <= tol)
        assert np.all(np.abs(c_new.astype(np.float64) - J_new) <= tol)
        assert np.all(np.abs(c_new.astype(np.float64) - c_ref.astype(np.float64)) <= tol)
        assert np.all(s_new < (1 << (wl.L - wl.k)))


def test_static_scratch_rejects_shapes_beyond_its_size(cuda_device):
    # one CTA at L=16, k=2 needs 4 KiB of backpointers per step, double
    # buffered: T = 8192 needs 64 MiB, above the 32 MiB static array.  The
    # pointers are never dereferenced: the size check comes first.
    fake = ctypes.c_void_p(256)
    st = tcq.tcq_encode_static_scratch(fake, None, fake, tcq.TCQ_F16, 16, 2, 8192, 1, fake, fake,
                                       fake, None)
    assert st == tcq.TCQ_ERR_WORKSPACE
