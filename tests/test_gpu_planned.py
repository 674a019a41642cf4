"""GPU parity of the planned fused path (rptq_ln_quant_plan + rptq_ln_reorder_quant_planned): its
codes are compared with the oracle's ln_reorder_quant (the codes bar) and must equal, byte for
byte, the codes of rptq_ln_reorder_quant on the same inputs (the plan holds the same offsets and
the same fp64-derived coefficients the unplanned kernel builds in every CTA)."""
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


@pytest.mark.parametrize("dtype,T,C,g,bits", [
    ("bf16", 1187, 12288, 64, 3),   # the OPT-175B width, ragged last quad, several quads per CTA
    ("bf16", 2501, 9216, 64, 3),    # the OPT-66B width
    ("f16", 2048, 4096, 32, 4),     # the OPT-6.7B shape
    ("f32", 512, 768, 8, 4),        # the tiny layer
    ("bf16", 3, 1024, 8, 4),        # fewer tokens than one quad
    ("f16", 777, 2560, 16, 3),      # a runtime thread split (no compiled-in width)
])
def test_planned_codes_match_the_oracle_and_the_unplanned_path(dtype, T, C, g, bits):
    seed = 5 * T + C
    m, gamma, beta = model_inputs(C, seed)
    xc = synthetic.activations(64, m, seed, dtype=dtype, calibration=True)
    cal = oracle_calibration(xc, gamma, beta, g, 10, bits)
    x = synthetic.activations(T, m, seed, dtype=dtype)
    p = dev_params(cal)
    xd, gd, bd = x.to(DEV), gamma.to(DEV), beta.to(DEV)
    plan = rptq.rptq_ln_quant_plan(gd, bd, p["R"], p["col_cluster"], p["scale"], p["zero"], bits)
    assert plan.numel() == 12 * C
    got = rptq.rptq_ln_reorder_quant_planned(xd, plan, bits)
    ref_gpu, _ = rptq.rptq_ln_reorder_quant(xd, gd, bd, p["R"], p["col_cluster"], p["scale"], p["zero"], bits)
    assert torch.equal(got, ref_gpu), "planned and unplanned codes differ"
    ref, _, _ = oracle.ln_reorder_quant(x, gamma, beta, cal["R"], cal["col_cluster"], cal["scale"], cal["zero"], bits)
    compare_codes(to_np(got), ref, C, bits, f"planned {dtype} T={T} C={C}")


def test_plan_contents():
    """Offsets: channel R[j] gets the code-buffer offset of stored column j, so the offsets are a
    permutation of those of 0..C-1; coefficients: A = gamma / (s qmax), B = beta / (s qmax) + z / qmax
    of the channel's cluster, within one fp32 rounding of the fp64 values."""
    C, g, bits = 768, 8, 4
    m, gamma, beta = model_inputs(C, 3)
    xc = synthetic.activations(64, m, 3, dtype="f32", calibration=True)
    cal = oracle_calibration(xc, gamma, beta, g, 10, bits)
    p = dev_params(cal)
    plan = to_np(rptq.rptq_ln_quant_plan(gamma.to(DEV), beta.to(DEV), p["R"], p["col_cluster"], p["scale"], p["zero"],
                                         bits))
    off = plan[:4 * C].view(np.uint32)
    A = plan[4 * C:8 * C].view(np.float32).astype(np.float64)
    B = plan[8 * C:].view(np.float32).astype(np.float64)
    assert np.all(off % 4 == 0) and np.all(off < 4 * C) and len(set(off.tolist())) == C
    R, cc = cal["R"], cal["col_cluster"]
    # the code buffer keeps stored column j in 16-byte slot j / 4, slot s at s ^ ((s / 8) mod 8)
    j = np.arange(C)
    slot = j >> 2
    assert np.array_equal(off[R], ((slot ^ ((slot >> 3) & 7)) << 4) | ((j & 3) << 2))
    k_of = np.empty(C, np.int64)
    k_of[R] = cc
    s64 = cal["scale"].astype(np.float64)[k_of] * (2 ** bits - 1)
    a_ref = gamma.numpy().astype(np.float64) / s64
    b_ref = beta.numpy().astype(np.float64) / s64 + cal["zero"].astype(np.float64)[k_of] / (2 ** bits - 1)
    assert np.all(np.abs(A - a_ref) <= 2.0 ** -24 * np.abs(a_ref) * (1 + 1e-9))
    assert np.all(np.abs(B - b_ref) <= 2.0 ** -24 * np.abs(b_ref) * (1 + 1e-9) + 1e-300)


def test_planned_refusals_and_empty():
    C, g, bits = 1024, 8, 4
    m, gamma, beta = model_inputs(C, 4)
    xc = synthetic.activations(64, m, 4, dtype="bf16", calibration=True)
    cal = oracle_calibration(xc, gamma, beta, g, 10, bits)
    p = dev_params(cal)
    plan = rptq.rptq_ln_quant_plan(gamma.to(DEV), beta.to(DEV), p["R"], p["col_cluster"], p["scale"], p["zero"], bits)
    x0 = torch.empty((0, C), dtype=torch.bfloat16, device=DEV)
    assert rptq.rptq_ln_reorder_quant_planned(x0, plan, bits).shape == (0, C * bits // 8)
    # C = 40 is not a multiple of 32: no direct kernel, so no planned path
    x = torch.zeros((4, 40), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(rptq.RptqError) as e:
        rptq.rptq_ln_reorder_quant_planned(x, plan, bits)
    assert e.value.status == -2


def test_plan_with_a_bad_reorder_entry_sets_the_error_word():
    C, g, bits = 256, 4, 3
    m, gamma, beta = model_inputs(C, 6)
    xc = synthetic.activations(64, m, 6, dtype="f32", calibration=True)
    cal = oracle_calibration(xc, gamma, beta, g, 10, bits)
    p = dev_params(cal)
    R = p["R"].clone()
    R[7] = -3
    plan = rptq.rptq_ln_quant_plan(gamma.to(DEV), beta.to(DEV), R, p["col_cluster"], p["scale"], p["zero"], bits)
    assert rptq.rptq_device_error() & 2
    # the damaged plan still keeps every store inside the code buffer
    x = synthetic.activations(9, m, 6, dtype="f32").to(DEV)
    rptq.rptq_ln_reorder_quant_planned(x, plan, bits)
    torch.cuda.synchronize()
    assert rptq.rptq_device_error() == 0
