"""Failure detection on the GPU without a fault (allowed form: a bounded wait made to run out).

The KMeans kernel's CTAs exchange per-iteration records through global memory and wait for each
other with bounded waits.  Through the testing hook, the wait limit is cut to a few
milliseconds and one CTA leaves out its first record: every other CTA's wait for it runs out,
the call ends on its own, and the host reads RPTQ_DEVERR_TIMEOUT from the sticky device error
word.  The context stays usable: with the hook reset, the next call matches the oracle.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from post_activation_quantization_b200 import rptq, synthetic
from tests.gpu_common import DEV

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_activation_quantization_b200 import build
    build.build()
    rptq.lib()
    yield
    rptq.rptq_testing_kmeans_wait(0, -1)
    assert rptq.rptq_device_error() == 0


def _points(C, seed):
    m = synthetic.channel_model(C, seed)
    gamma, beta = synthetic.ln_params(C, seed)
    x = synthetic.activations(256, m, seed, dtype="f32", calibration=True)
    return oracle.minmax_ln(x, gamma, beta)


@pytest.mark.parametrize("noalloc", [False, True])
def test_kmeans_wait_runs_out_then_recovers(noalloc):
    C, g, iters, bits = 4096, 32, 10, 3  # 8 CTAs
    mx, mn = _points(C, 31)
    dmx, dmn = torch.from_numpy(mx).to(DEV), torch.from_numpy(mn).to(DEV)
    def run(*a):
        if noalloc:
            out = {k: torch.empty(n, dtype=t, device=DEV) for k, n, t in (
                ("labels", C, torch.int32), ("centroids", (g, 2), torch.float64), ("R", C, torch.int32),
                ("col_cluster", C, torch.int32), ("offsets", g + 1, torch.int32), ("scale", g, torch.float32),
                ("zero", g, torch.int32))}
            rptq.rptq_kmeans_noalloc(*a, out=out)
            return out
        return rptq.rptq_kmeans(*a)
    assert rptq.rptq_device_error() == 0
    try:
        rptq.rptq_testing_kmeans_wait(5_000_000, 3)  # 5 ms; CTA 3 withholds its first record
        t0 = time.perf_counter()
        run(dmx, dmn, g, iters, bits)
        code = rptq.rptq_device_error()  # synchronises
        wall = time.perf_counter() - t0
    finally:
        rptq.rptq_testing_kmeans_wait(0, -1)
    assert code & rptq.RPTQ_DEVERR_TIMEOUT, code
    assert wall < 1.0, wall  # every CTA gave up after about one limit, not 2 s per wait
    # the context is usable and the next call is right
    out = run(dmx, dmn, g, iters, bits)
    assert rptq.rptq_device_error() == 0
    cal = oracle.calibrate(mx, mn, g, iters, bits)
    assert np.array_equal(out["R"].cpu().numpy(), cal["R"])
    assert np.array_equal(out["labels"].cpu().numpy(), cal["labels"])


def test_hook_rejects_bad_arguments():
    with pytest.raises(rptq.RptqError):
        rptq.rptq_testing_kmeans_wait(0, -2)
