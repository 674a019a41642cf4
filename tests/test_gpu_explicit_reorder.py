"""GPU parity of the explicit-reorder baseline (include/rptq_baseline.h): the unfused pipeline
LayerNorm -> materialised y -> explicit gather through R -> quantize must give the codes of the
definition (the oracle's ln_reorder_quant: LayerNorm, explicit gather, quantize), its y must be
the LayerNorm within the fp32 bar, and its reordered intermediate must be exactly y gathered
through R -- the same results as the fused kernel, with the intermediate tensors in HBM."""
import numpy as np
import pytest
import torch

import oracle
from post_activation_quantization_b200 import rptq, synthetic
from tests.gpu_common import DEV, compare_codes, compare_ln, dev_params, model_inputs, oracle_calibration, to_np

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


@pytest.mark.parametrize("dtype,T,C,g,bits", [
    ("bf16", 300, 12288, 64, 3), ("f16", 129, 4096, 32, 4), ("f32", 77, 768, 8, 4), ("bf16", 600, 9216, 64, 3),
    ("bf16", 5, 64, 4, 3)])
def test_explicit_reorder_baseline_matches_the_definition(dtype, T, C, g, bits):
    seed = 11 * T + C
    m, gamma, beta = model_inputs(C, seed)
    xc = synthetic.activations(64, m, seed, dtype=dtype, calibration=True)
    cal = oracle_calibration(xc, gamma, beta, g, 10, bits)
    x = synthetic.activations(T, m, seed, dtype=dtype)
    p = dev_params(cal)
    codes, y, yr = rptq.rptq_baseline_explicit_reorder_quant(x.to(DEV), gamma.to(DEV), beta.to(DEV), p["R"],
                                                              p["col_cluster"], p["scale"], p["zero"], bits)
    assert torch.equal(yr, y[:, p["R"].long()])
    ref, _, _ = oracle.ln_reorder_quant(x, gamma, beta, cal["R"], cal["col_cluster"], cal["scale"], cal["zero"], bits)
    compare_codes(to_np(codes), ref, C, bits, f"explicit reorder {dtype} C={C}")
    y64, _ = oracle.layernorm(x, gamma, beta)
    compare_ln(to_np(y), y64, gamma.numpy()[None].astype(np.float64), beta.numpy()[None].astype(np.float64), "f32",
               f"explicit reorder LN {dtype} C={C}")
