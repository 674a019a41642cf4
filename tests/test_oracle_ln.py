"""Pins for the oracle's calibration statistics and LayerNorm, and for the reorder-fusion
invariant (RPTQ article, text after Fig. 3: the LayerNorm emits the reordered activations, so the
fused result must equal LayerNorm followed by an explicit gather through R)."""
import numpy as np
import pytest
import torch

from post_activation_quantization_b200 import synthetic


def _x(T, C, seed, dtype="f32"):
    m = synthetic.channel_model(C, seed)
    return synthetic.activations(T, m, seed, dtype=dtype)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_minmax_matches_numpy_and_accumulates(orc, dtype):
    x = _x(300, 40, 3, dtype).float().numpy()
    mx, mn = orc.minmax(x)
    assert np.array_equal(mx, x.max(0)) and np.array_equal(mn, x.min(0))
    mx1, mn1 = orc.minmax(x[:100])
    mx2, mn2 = orc.minmax(x[100:], mx1, mn1)
    assert np.array_equal(mx2, mx) and np.array_equal(mn2, mn)


def test_layernorm_matches_torch_fp64(orc):
    x = _x(64, 96, 4).numpy()
    g, b = synthetic.ln_params(96, 4)
    y64, y32 = orc.layernorm(x, g, b, eps=1e-5)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x).double(), (96,),
                                         g.double(), b.double(), eps=1e-5).numpy()
    assert np.allclose(y64, ref, rtol=1e-12, atol=1e-12)
    assert np.array_equal(y32, y64.astype(np.float32))


def test_layernorm_moments_and_constant_row(orc):
    rng = np.random.default_rng(5)
    C = 128
    x = rng.normal(3.0, 7.0, (8, C)).astype(np.float32)
    x[7] = 2.5  # constant row: normalised part is 0, output is beta
    one, zero = np.ones(C, np.float32), np.zeros(C, np.float32)
    y64, _ = orc.layernorm(x, one, zero, eps=1e-5)
    xd = x.astype(np.float64)
    var = xd.var(axis=1)
    assert np.allclose(y64[:7].mean(1), 0.0, atol=1e-12)
    assert np.allclose(y64[:7].var(1), var[:7] / (var[:7] + 1e-5), rtol=1e-10)
    beta = rng.normal(0, 0.1, C).astype(np.float32)
    y64, _ = orc.layernorm(x, one, beta, eps=1e-5)
    assert np.array_equal(y64[7], beta.astype(np.float64))


def test_minmax_ln_is_minmax_of_rounded_layernorm(orc):
    x = _x(200, 64, 6).numpy()
    g, b = synthetic.ln_params(64, 6)
    _, y32 = orc.layernorm(x, g, b)
    mx, mn = orc.minmax_ln(x, g, b)
    assert np.array_equal(mx, y32.max(0)) and np.array_equal(mn, y32.min(0))
    mx1, mn1 = orc.minmax_ln(x[:77], g, b)
    mx2, mn2 = orc.minmax_ln(x[77:], g, b, ch_max=mx1, ch_min=mn1)
    assert np.array_equal(mx2, mx) and np.array_equal(mn2, mn)


@pytest.mark.parametrize("bits", [3, 4])
def test_fused_ln_reorder_quant_equals_unfused_definition(orc, bits):
    C, T = 256, 96
    x = _x(T, C, 7).numpy()
    g, b = synthetic.ln_params(C, 7)
    mx, mn = orc.minmax_ln(x, g, b)
    cal = orc.calibrate(mx, mn, 8, 10, bits)
    packed, ln32, ln64 = orc.ln_reorder_quant(x, g, b, cal["R"], cal["col_cluster"], cal["scale"],
                                              cal["zero"], bits, want_ln=True)
    y64, y32 = orc.layernorm(x, g, b)
    R = cal["R"]
    assert np.array_equal(ln32, y32[:, R]) and np.array_equal(ln64, y64[:, R])
    q = orc.quantize(y32[:, R], cal["col_cluster"], cal["scale"], cal["zero"], bits)
    assert np.array_equal(packed, orc.pack(q, bits))
    # identity reorder: the stored order is the channel order
    ident = np.arange(C, dtype=np.int32)
    cc0 = np.zeros(C, np.int32)
    p2, l2, _ = orc.ln_reorder_quant(x, g, b, ident, cc0, cal["scale"][:1], cal["zero"][:1], bits,
                                     want_ln=True)
    assert np.array_equal(l2, y32)


@pytest.mark.parametrize("bits", [3, 4])
def test_kv_quant_is_per_channel_quant_of_each_head(orc, bits):
    B, H, S, D = 2, 3, 5, 16
    m = synthetic.channel_model(H * D, 8)
    kv = synthetic.kv_cache(B, H, S, D, m, 8, "k", dtype="f16").float().numpy()
    flat = kv.transpose(0, 2, 1, 3).reshape(B * S, H * D)  # tokens x channels (c = h*D + d)
    mx, mn = orc.minmax(flat)
    cal = orc.calibrate(mx, mn, 6, 10, bits)
    labels = cal["labels"]  # KV keeps its natural layout: channel c uses cluster labels[c]
    packed = orc.kv_quant(kv, labels, cal["scale"], cal["zero"], bits)
    for h in range(H):
        rows = kv[:, h].reshape(B * S, D)
        q = orc.quantize(rows, labels[h * D:(h + 1) * D], cal["scale"], cal["zero"], bits)
        assert np.array_equal(packed[:, h].reshape(B * S, -1), orc.pack(q, bits))
    deq = orc.kv_dequant(packed, D, labels, cal["scale"], cal["zero"], bits)
    s_of_c = cal["scale"][labels].reshape(H, D)
    assert np.all(np.abs(deq - kv) <= s_of_c[None, :, None, :] / 2 * (1 + 1e-6))
