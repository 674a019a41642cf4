"""GPU parity of dynamic (per-batch) cluster ranges: rptq_cluster_params is bit-exact against the
oracle's cluster_params on the same statistics (empty, degenerate and zero-range clusters
included), and the whole dynamic path -- LayerNorm statistics of the batch, per-cluster (s, z)
with the offline clusters, fused quantization -- gives the oracle's codes (the +-1 bar)."""
import numpy as np
import pytest
import torch

import oracle
from post_activation_quantization_b200 import rptq, synthetic
from tests.gpu_common import DEV, compare_codes, dev_params, model_inputs, oracle_calibration, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_activation_quantization_b200 import build
    build.build()
    rptq.lib()
    yield
    assert rptq.rptq_device_error() == 0


@pytest.mark.parametrize("C,g,bits", [(768, 8, 4), (12288, 64, 3), (4096, 512, 3), (40, 7, 4)])
def test_cluster_params_bit_exact(C, g, bits):
    rng = np.random.default_rng(C + g)
    mx = (rng.standard_normal(C) * 3).astype(np.float32)
    mn = (mx - np.abs(rng.standard_normal(C)) * 2).astype(np.float32)
    labels = rng.integers(0, g, C).astype(np.int32)
    labels[labels == g - 1] = 0  # an empty cluster
    mx[labels == 1] = mn[labels == 1] = np.float32(2.5)  # a degenerate cluster (M == m)
    if g > 2:
        mx[labels == 2] = mn[labels == 2] = np.float32(0.0)  # M == m == 0
    s, z = rptq.rptq_cluster_params(torch.from_numpy(mx).to(DEV), torch.from_numpy(mn).to(DEV),
                                    torch.from_numpy(labels).to(DEV), g, bits)
    rs, rz = oracle.cluster_params(mx, mn, labels, g, bits)
    assert np.array_equal(to_np(s).view(np.uint32), rs.view(np.uint32)) and np.array_equal(to_np(z), rz)


@pytest.mark.parametrize("dtype,T,C,g,bits", [("bf16", 700, 12288, 64, 3), ("f16", 300, 4096, 32, 4),
                                               ("bf16", 1000, 9216, 64, 3)])
def test_dynamic_ranges_path(dtype, T, C, g, bits):
    seed = T + C + 1
    m, gamma, beta = model_inputs(C, seed)
    xc = synthetic.activations(256, m, seed, dtype=dtype, calibration=True)
    cal = oracle_calibration(xc, gamma, beta, g, 10, bits)
    x = synthetic.activations(T, m, seed + 5, dtype=dtype) * 1.5  # beyond the calibration ranges
    xd, gd, bd = x.to(DEV), gamma.to(DEV), beta.to(DEV)
    p = dev_params(cal)
    # stage-wise: the oracle's batch statistics -> GPU parameters, bit-exact
    omx, omn = oracle.minmax_ln(x, gamma, beta)
    s_o, z_o = oracle.dynamic_params(x, gamma, beta, cal["labels"], g, bits)
    s1, z1 = rptq.rptq_cluster_params(torch.from_numpy(omx).to(DEV), torch.from_numpy(omn).to(DEV), p["labels"], g,
                                      bits)
    assert np.array_equal(to_np(s1).view(np.uint32), s_o.view(np.uint32)) and np.array_equal(to_np(z1), z_o)
    # the whole GPU path: batch statistics, parameters, fused quantization
    mx, mn = rptq.rptq_calib_minmax(xd, gd, bd, 1e-5)
    s2, z2 = rptq.rptq_cluster_params(mx, mn, p["labels"], g, bits)
    codes, _ = rptq.rptq_ln_reorder_quant(xd, gd, bd, p["R"], p["col_cluster"], s2, z2, bits)
    ref, _, _ = oracle.ln_reorder_quant(x, gamma, beta, cal["R"], cal["col_cluster"], s_o, z_o, bits)
    compare_codes(to_np(codes), ref, C, bits, f"dynamic {dtype} C={C}")
