"""The allocation-free KMeans entry point against the regular one and against the CPU oracle.

rptq_kmeans_noalloc exists for callers that cannot allocate device memory while running (a
plugin whose host application owns all GPU memory, a serving loop that forbids cudaMalloc and
cudaFree after start-up); it runs the same kernels on a fixed scratch array inside the library.
This file is collected last so that a run stopping at the first failure has run every other
test first; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from post_activation_quantization_b200 import rptq, synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_activation_quantization_b200 import build
    build.build()
    rptq.lib()


def _stats(C, seed):
    m = synthetic.channel_model(C, seed)
    gamma, beta = synthetic.ln_params(C, seed)
    x = synthetic.activations(256, m, seed, dtype="bf16", calibration=True).cuda()
    return rptq.rptq_calib_minmax(x, gamma.cuda(), beta.cuda(), 1e-5)


def _outputs(C, g):
    d = "cuda"
    return dict(labels=torch.empty(C, dtype=torch.int32, device=d),
                centroids=torch.empty((g, 2), dtype=torch.float64, device=d),
                R=torch.empty(C, dtype=torch.int32, device=d),
                col_cluster=torch.empty(C, dtype=torch.int32, device=d),
                offsets=torch.empty(g + 1, dtype=torch.int32, device=d),
                scale=torch.empty(g, dtype=torch.float32, device=d),
                zero=torch.empty(g, dtype=torch.int32, device=d))


def _call_c_abi(mx, mn, g, iters, bits, out):
    """Direct call through the C ABI (no Python wrapper logic)."""
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return rptq.lib().rptq_kmeans_noalloc(
        p(mx), p(mn), mx.numel(), g, iters, bits, p(out["labels"]), p(out["centroids"]), p(out["R"]),
        p(out["col_cluster"]), p(out["offsets"]), p(out["scale"]), p(out["zero"]),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _same(a, b):
    for k in ("labels", "R", "col_cluster", "offsets", "zero"):
        assert torch.equal(a[k], b[k]), k
    torch.testing.assert_close(a["scale"], b["scale"], rtol=0, atol=0)
    np.testing.assert_allclose(a["centroids"].cpu().numpy(), b["centroids"].cpu().numpy(),
                               rtol=1e-6, atol=1e-12)


def test_noalloc_matches_workspace_version_twice_in_a_row():
    cases = [(12288, 64, 50, 3, 4), (4096, 32, 20, 4, 1)]  # two different problems, back to back
    for C, g, iters, bits, seed in cases:
        mx, mn = _stats(C, seed)
        ref = rptq.rptq_kmeans(mx, mn, g, iters, bits)
        out = _outputs(C, g)
        assert _call_c_abi(mx, mn, g, iters, bits, out) == rptq.RPTQ_OK
        torch.cuda.synchronize()
        _same(out, ref)
    # the same problem again right after: the scratch keeps the previous call's contents
    out2 = _outputs(C, g)
    assert _call_c_abi(mx, mn, g, iters, bits, out2) == rptq.RPTQ_OK
    torch.cuda.synchronize()
    _same(out2, ref)
    assert rptq.rptq_device_error() == 0


def test_noalloc_largest_problem_fits_its_scratch():
    C, g = 16384, 512  # the library's largest (C, g): its workspace fits the 2 MiB scratch
    assert rptq.lib().rptq_kmeans_workspace_size(C, g) <= (2 << 20)
    mx, mn = _stats(C, 7)
    ref = rptq.rptq_kmeans(mx, mn, g, 5, 3)
    out = _outputs(C, g)
    assert _call_c_abi(mx, mn, g, 5, 3, out) == rptq.RPTQ_OK
    torch.cuda.synchronize()
    _same(out, ref)
    assert rptq.rptq_device_error() == 0


def test_noalloc_refuses_invalid_sizes():
    C = 1024
    mx = torch.zeros(C, device="cuda")
    out = _outputs(C, 8)
    assert _call_c_abi(mx, mx, C + 1, 1, 3, out) == rptq.RPTQ_ERR_INVALID_ARG   # g > C
    assert _call_c_abi(mx, mx, 8, 1, 5, out) == rptq.RPTQ_ERR_UNSUPPORTED      # bits


def test_noalloc_matches_the_oracle():
    """Standing alone: the entry point's outputs against the oracle's calibration chain on the
    same statistics (labels, R, offsets, s and z exact; centroids to 1e-6)."""
    import oracle
    C, g, iters, bits = 4096, 32, 20, 4
    mx, mn = _stats(C, 21)
    hmx, hmn = mx.cpu().numpy(), mn.cpu().numpy()
    cal = oracle.calibrate(hmx, hmn, g, iters, bits)
    out = _outputs(C, g)
    assert _call_c_abi(mx, mn, g, iters, bits, out) == rptq.RPTQ_OK
    torch.cuda.synchronize()
    for k in ("labels", "R", "col_cluster", "offsets", "scale", "zero"):
        assert np.array_equal(out[k].cpu().numpy(), cal[k]), k
    np.testing.assert_allclose(out["centroids"].cpu().numpy(), cal["centroids"], rtol=1e-6, atol=1e-12)
    assert rptq.rptq_device_error() == 0
