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


def _calibrated_case(C=128, T=12, N=7, g=6, bits=4, seed=5):
    m = synthetic.channel_model(C, seed)
    gamma, beta = synthetic.ln_params(C, seed)
    x = oracle._f32(synthetic.activations(T, m, seed, dtype="f32"))
    mx, mn = oracle.minmax_ln(x, gamma, beta)
    cal = oracle.calibrate(mx, mn, g, 10, bits)
    codes, _, _ = oracle.ln_reorder_quant(x, gamma, beta, cal["R"], cal["col_cluster"], cal["scale"], cal["zero"], bits)
    W = np.random.default_rng(seed + 1).standard_normal((N, C)).astype(np.float32)
    qw, sw, zw = oracle.quant_weights(W, 4)
    return cal, codes, qw, sw, zw


def test_fp16_operand_range_and_rounding():
    """Each row's largest |B| lies in [2^14, 2^15) (lam a power of two), and B lam is within
    fp16's half-ulp bound 2^-11 (relative) of the fp32 product s_k (qw - zw)."""
    cal, _, qw, sw, zw = _calibrated_case()
    B, bz, lam = oracle.linear_fp16_operand(qw, sw, zw, cal["R"], cal["col_cluster"], cal["scale"], cal["zero"])
    cc = cal["col_cluster"]
    for n in range(B.shape[0]):
        assert np.frexp(lam[n])[0] == 0.5  # a power of two
        top = np.abs(B[n].astype(np.float64)).max()
        assert 2.0 ** 14 <= top < 2.0 ** 15
        b = cal["scale"][cc].astype(np.float64) * (qw[n, cal["R"]].astype(np.float64) - zw[n])
        err = np.abs(B[n].astype(np.float64) * lam[n] - b)
        assert np.all(err <= 2.0 ** -11 * np.abs(b) * (1 + 2.0 ** -20) + 1e-30)
        assert np.isclose(bz[n], np.sum(cal["zero"][cc] * B[n].astype(np.float64)), rtol=2.0 ** -23, atol=0)


def test_fp16_operand_reproduces_the_layer():
    """sw lam (q B^T - bz) equals the fp64 layer within the bound that B's rounding allows, and a
    column taken in the original order instead of the cluster order breaks it."""
    bits = 4
    cal, codes, qw, sw, zw = _calibrated_case(bits=bits)
    cc, R = cal["col_cluster"], cal["R"]
    B, bz, lam = oracle.linear_fp16_operand(qw, sw, zw, R, cc, cal["scale"], cal["zero"])
    Y = oracle.reordered_linear(codes, 128, cc, cal["scale"], cal["zero"], bits, R, qw, sw, zw)
    q = oracle.unpack(codes, 128, bits).astype(np.float64)
    Yb = (q @ B.astype(np.float64).T - bz.astype(np.float64)) * (sw.astype(np.float64) * lam)[None, :]
    b = cal["scale"][cc].astype(np.float64)[None, :] * (qw[:, R].astype(np.float64) - zw[:, None])
    A = np.abs(q - cal["zero"][cc][None, :])
    bound = sw[None, :] * (2.0 ** -11 * (A @ np.abs(b).T)) + 2.0 ** -20 * np.abs(Y) + 1e-12
    assert np.all(np.abs(Yb - Y) <= bound)
    Bn, bzn, lamn = oracle.linear_fp16_operand(qw, sw, zw, np.arange(128, dtype=np.int32), cc, cal["scale"],
                                               cal["zero"])
    Ybad = (q @ Bn.astype(np.float64).T - bzn) * (sw.astype(np.float64) * lamn)[None, :]
    assert not np.all(np.abs(Ybad - Y) <= bound)


def test_fp16_operand_zero_row():
    """A weight row whose codes all equal its zero point gives B = 0, bz = 0 and lam = 1."""
    qw = np.full((1, 16), 5, np.uint8)
    B, bz, lam = oracle.linear_fp16_operand(qw, np.array([0.1], np.float32), np.array([5], np.int32),
                                            np.arange(16, dtype=np.int32), np.zeros(16, np.int32),
                                            np.array([0.3], np.float32), np.array([2], np.int32))
    assert not B.any() and bz[0] == 0 and lam[0] == 1
