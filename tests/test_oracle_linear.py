"""Pins of the oracle's reordered low-bit linear layer and weight quantizer.
  * Offline reordering leaves the layer's output unchanged ([RPTQ-art], text after Fig. 3): the
    layer on the cluster-ordered codes with weights permuted by R equals the dequantized
    activations put back into the original channel order times the unpermuted weights.  A
    permutation taken the wrong way round (R^-1 for R) fails this on any non-trivial R.
  * A hand-worked case (C = 8, one token, one output) gives the value computed by hand.
  * The per-row weight quantizer meets the s/2 bound and maps each row's minimum and maximum to
    codes 0 and qmax."""
import numpy as np

import oracle
from post_activation_quantization_b200 import synthetic


def test_reordered_layer_equals_the_unreordered_product():
    C, T, N, g, bits = 64, 10, 5, 6, 3
    m = synthetic.channel_model(C, 3)
    gamma, beta = synthetic.ln_params(C, 3)
    x = oracle._f32(synthetic.activations(T, m, 3, dtype="f32"))
    mx, mn = oracle.minmax_ln(x, gamma, beta)
    cal = oracle.calibrate(mx, mn, g, 10, bits)
    assert not np.array_equal(cal["R"], np.arange(C))  # a real permutation
    codes, _, _ = oracle.ln_reorder_quant(x, gamma, beta, cal["R"], cal["col_cluster"], cal["scale"], cal["zero"], bits)
    W = np.random.default_rng(1).standard_normal((N, C)).astype(np.float32)
    qw, sw, zw = oracle.quant_weights(W, 4)
    Y = oracle.reordered_linear(codes, C, cal["col_cluster"], cal["scale"], cal["zero"], bits, cal["R"], qw, sw, zw)
    # independent path: dequantize in cluster order, scatter back to the original channels
    q = oracle.unpack(codes, C, bits).astype(np.float64)
    cc = cal["col_cluster"]
    xs = (q - cal["zero"][cc]) * cal["scale"][cc].astype(np.float64)
    x_orig = np.empty_like(xs)
    x_orig[:, cal["R"]] = xs
    w_deq = (qw.astype(np.float64) - zw[:, None]) * sw[:, None].astype(np.float64)
    Y2 = np.einsum("tc,nc->tn", x_orig, w_deq)
    assert np.allclose(Y, Y2, rtol=1e-12, atol=1e-12)
    # the permutation the wrong way round gives another result
    Rinv = np.argsort(cal["R"])
    Yw = oracle.reordered_linear(codes, C, cc, cal["scale"], cal["zero"], bits, Rinv, qw, sw, zw)
    assert not np.allclose(Yw, Y2)


def test_hand_worked_case():
    # C = 8 channels in two clusters: columns 0-3 -> cluster 0 (s 0.5, z 1), 4-7 -> cluster 1 (s 2, z 0)
    C, bits = 8, 4
    q = np.array([[3, 1, 0, 2, 1, 2, 0, 3]], np.uint8)
    codes = oracle.pack(q, bits)
    cc = np.array([0, 0, 0, 0, 1, 1, 1, 1], np.int32)
    s = np.array([0.5, 2.0], np.float32)
    z = np.array([1, 0], np.int32)
    R = np.array([7, 6, 5, 4, 3, 2, 1, 0], np.int32)  # stored column j holds channel 7 - j
    qw = np.array([[1, 2, 3, 4, 5, 6, 7, 8]], np.uint8)  # original channel order
    sw, zw = np.array([0.25], np.float32), np.array([4], np.int32)
    # activations (cluster order): 0.5*(3-1, 1-1, 0-1, 2-1) = (1, 0, -0.5, 0.5); 2*(1, 2, 0, 3) = (2, 4, 0, 6)
    # weights of channels 7..0: 0.25*(qw - 4) = (1, 0.75, 0.5, 0.25, 0, -0.25, -0.5, -0.75)
    # sum: 1*1 + 0 + -0.5*0.5 + 0.5*0.25 + 0 + 4*-0.25 + 0 + 6*-0.75 = -4.625
    Y = oracle.reordered_linear(codes, C, cc, s, z, bits, R, qw, sw, zw)
    assert Y.shape == (1, 1) and Y[0, 0] == -4.625


def test_weight_quantizer_bound_and_ends():
    W = np.random.default_rng(2).standard_normal((7, 40)).astype(np.float32) * 3
    q, sw, zw = oracle.quant_weights(W, 4)
    deq = (q.astype(np.float64) - zw[:, None]) * sw[:, None]
    assert (np.abs(deq - W) <= sw[:, None] / 2 * (1 + 1e-6)).all()
    assert (q[np.arange(7), W.argmin(1)] == 0).all() and (q[np.arange(7), W.argmax(1)] == 15).all()
