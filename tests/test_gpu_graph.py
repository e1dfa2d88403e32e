"""The entry points are stream-ordered and allocate nothing, so a CUDA graph can
capture them: an encode, its decode and the matrix-vector product captured once
and replayed on new inputs give exactly the results of direct calls."""
import numpy as np
import pytest

from trellis_coded_weight_tcq_b200 import tcq

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("L,k,cbt,code", [(16, 2, "f16", False), (12, 2, "f32", False),
                                          (16, 2, "f16", True)])
def test_capture_and_replay(L, k, cbt, code, cuda_device):
    import torch

    T, n, nb = 256, 96, 8                 # a 12 x 2048 matrix of 96 blocks
    rows, cols = n // nb, nb * T
    rng = np.random.default_rng(9600 + L)
    cb = rng.standard_normal(1 << L).astype(np.float16 if cbt == "f16" else np.float32)
    cbd = tcq.MAD if code else torch.from_numpy(cb).to(cuda_device)
    dt = tcq.TCQ_MAD if code else tcq.cb_dtype_of(cbd)
    x_s = torch.empty((n, T), device=cuda_device)
    d_s = torch.empty((n, T), device=cuda_device)
    v_s = torch.empty(cols, device=cuda_device)
    ws = tcq.Workspace(L, k, T, n, dt, cuda_device)
    out = tcq.Encoded(torch.empty(n, dtype=torch.int32, device=cuda_device),
                      torch.empty((n, tcq.tcq_words_per_block(k, T)), dtype=torch.int32, device=cuda_device),
                      torch.empty(n, device=cuda_device))
    y_s = torch.empty((n, T), device=cuda_device)
    g_s = torch.empty(rows, device=cuda_device)

    def body():
        tcq.encode(x_s, d_s, cbd, L, k, workspace=ws, out=out)
        tcq.decode(out.bits, out.start_state, cbd, L, k, T, out=y_s)
        tcq.gemv(out.bits, out.start_state, None, cbd, L, k, T, rows, cols, v_s, out=g_s)

    x_s.normal_()
    d_s.uniform_(0.5, 2.0)
    v_s.normal_()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        body()                              # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        body()
    for seed in (1, 2):
        r = np.random.default_rng(seed)
        x = torch.from_numpy(r.standard_normal((n, T)).astype(np.float32)).to(cuda_device)
        d = torch.from_numpy(r.lognormal(0.0, 1.0, (n, T)).astype(np.float32)).to(cuda_device)
        v = torch.from_numpy(r.standard_normal(cols).astype(np.float32)).to(cuda_device)
        x_s.copy_(x)
        d_s.copy_(d)
        v_s.copy_(v)
        graph.replay()
        ref = tcq.encode(x, d, cbd, L, k)
        y_ref = tcq.decode(ref.bits, ref.start_state, cbd, L, k, T)
        g_ref = tcq.gemv(ref.bits, ref.start_state, None, cbd, L, k, T, rows, cols, v)
        torch.cuda.synchronize()
        assert torch.equal(out.bits, ref.bits) and torch.equal(out.start_state, ref.start_state)
        assert torch.equal(out.path_cost, ref.path_cost)
        assert torch.equal(y_s, y_ref) and torch.equal(g_s, g_ref)
    del graph
