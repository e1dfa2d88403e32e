"""The end-to-end host pipeline (pinned host arrays in, overlapped copies and
encodes by parts, results out) returns exactly what one device-side encode
returns, for ragged part sizes."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("chunks", [1, 3, 8])
def test_host_pipeline_matches_device_encode(chunks, cuda_device):
    import torch
    from trellis_coded_weight_tcq_b200 import tcq, workloads

    wl = workloads.small_random(16, 2, 256, 301, True, "f16", seed=77)
    x = torch.from_numpy(wl.x).to(cuda_device)
    d = torch.from_numpy(wl.d).to(cuda_device)
    cb = torch.from_numpy(wl.codebook).to(cuda_device)
    ref = tcq.encode(x, d, cb, wl.L, wl.k)
    pipe = tcq.HostPipeline(wl.n_blocks, wl.T, wl.L, wl.k, True, torch.from_numpy(wl.codebook),
                            cuda_device, chunks=chunks)
    xh = torch.from_numpy(wl.x).pin_memory()
    dh = torch.from_numpy(wl.d).pin_memory()
    for _ in range(2):  # the buffers are reused across runs
        start, bits, cost = pipe.run(xh, dh)
        torch.cuda.synchronize()
        assert torch.equal(start, ref.start_state.cpu())
        assert torch.equal(bits, ref.bits.cpu())
        assert torch.equal(cost, ref.path_cost.cpu())
    # a short lead part, then `chunks` equal parts (one part when chunks is 1)
    assert len(pipe.parts) == (1 if chunks == 1 else min(chunks + 1, wl.n_blocks))
    assert pipe.parts[0][0] == 0 and pipe.parts[-1][1] == wl.n_blocks
    assert all(a[1] == b[0] for a, b in zip(pipe.parts, pipe.parts[1:]))
