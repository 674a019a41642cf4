"""Pins of the oracle's dynamic (per-batch) cluster ranges: with the ranges taken from the batch
itself, no value of the batch lies outside its cluster's range, so every element meets the
s/2 error bound ([Basics] 1.1, 1.3; the static ranges of a calibration batch clamp a runtime
batch whose values exceed them); one cluster reduces to per-tensor quantization with the
global LayerNorm range (closed form); and on a batch with values beyond the calibration range,
the dynamic ranges give a smaller quantization error than the static ones."""
import numpy as np

import oracle
from post_activation_quantization_b200 import synthetic


def _setup(C=256, T=64, seed=3, g=8, bits=3):
    m = synthetic.channel_model(C, seed)
    gamma, beta = synthetic.ln_params(C, seed)
    xc = oracle._f32(synthetic.activations(T, m, seed, dtype="f32", calibration=True))
    mx, mn = oracle.minmax_ln(xc, gamma, beta)
    cal = oracle.calibrate(mx, mn, g, 10, bits)
    return m, gamma, beta, cal


def _errors(x, gamma, beta, cal, s, z, bits):
    packed, _, y64 = oracle.ln_reorder_quant(x, gamma, beta, cal["R"], cal["col_cluster"], s, z, bits, want_ln=True)
    q = oracle.unpack(packed, x.shape[1], bits)
    deq = oracle.dequant(q, cal["col_cluster"], s, z)
    return np.abs(deq.astype(np.float64) - y64), s[cal["col_cluster"]].astype(np.float64)


def test_dynamic_ranges_cover_the_batch():
    bits = 3
    m, gamma, beta, cal = _setup(bits=bits)
    x = oracle._f32(synthetic.activations(48, m, 9, dtype="f32")) * np.float32(1.7)  # beyond the calibration
    s, z = oracle.dynamic_params(x, gamma, beta, cal["labels"], 8, bits)
    err, sc = _errors(x, gamma, beta, cal, s, z, bits)
    # half a step, plus the fp32 rounding of y and of the quotient
    assert (err <= sc / 2 * (1 + 1e-5) + 1e-6).all()


def test_one_cluster_is_per_tensor():
    bits = 4
    m, gamma, beta, _ = _setup(bits=bits)
    x = oracle._f32(synthetic.activations(20, m, 5, dtype="f32"))
    labels = np.zeros(256, np.int32)
    s, z = oracle.dynamic_params(x, gamma, beta, labels, 1, bits)
    y64, _ = oracle.layernorm(x, gamma, beta)
    y32 = y64.astype(np.float32)
    M, mn = np.float32(y32.max()), np.float32(y32.min())
    s_ref = np.float32(np.float32(M - mn) / np.float32(15))
    assert s[0] == s_ref and z[0] == np.int32(np.rint(np.float32(-mn / s_ref)))


def test_dynamic_beats_static_on_a_batch_beyond_the_calibration():
    bits = 3
    m, gamma, beta, cal = _setup(bits=bits)
    x = oracle._f32(synthetic.activations(48, m, 11, dtype="f32")) * np.float32(2.5)
    s_d, z_d = oracle.dynamic_params(x, gamma, beta, cal["labels"], 8, bits)
    e_dyn, _ = _errors(x, gamma, beta, cal, s_d, z_d, bits)
    e_sta, _ = _errors(x, gamma, beta, cal, cal["scale"], cal["zero"], bits)
    assert (e_dyn ** 2).mean() < (e_sta ** 2).mean()
