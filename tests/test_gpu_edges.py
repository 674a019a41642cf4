"""Edge cases of the CUDA path against the oracle: empty inputs, degenerate clusters, constant
and ill-conditioned LayerNorm rows, zero points beyond the fast paths' ranges."""
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


def _cal(C, g, bits, seed, dtype="bf16"):
    m, gamma, beta = model_inputs(C, seed)
    xc = synthetic.activations(64, m, seed, dtype=dtype, calibration=True)
    return m, gamma, beta, oracle_calibration(xc, gamma, beta, g, 5, bits)


def test_empty_inputs_launch_nothing_and_succeed():
    C, g, bits = 768, 8, 3
    m, gamma, beta, cal = _cal(C, g, bits, 3)
    p = dev_params(cal)
    x = torch.empty((0, C), dtype=torch.bfloat16, device=DEV)
    codes, _ = rptq.rptq_ln_reorder_quant(x, gamma.to(DEV), beta.to(DEV), p["R"], p["col_cluster"],
                                          p["scale"], p["zero"], bits)
    assert codes.shape == (0, C * bits // 8)
    kv = torch.empty((2, 3, 0, 64), dtype=torch.float16, device=DEV)
    lab = torch.zeros(3 * 64, dtype=torch.int32, device=DEV)
    s = torch.ones(2, device=DEV)
    z = torch.zeros(2, dtype=torch.int32, device=DEV)
    kq, _ = rptq.rptq_kv_quant(kv, None, lab, s, z, None, None, None, bits)
    assert kq.shape == (2, 3, 0, 64 * bits // 8)
    out = rptq.rptq_dequant(torch.empty((0, C * bits // 8), dtype=torch.uint8, device=DEV), p["col_cluster"],
                            p["scale"], p["zero"], bits, C=C)
    assert out.shape == (0, C)
    torch.cuda.synchronize()
    assert rptq.rptq_device_error() == 0


@pytest.mark.parametrize("bits", [3, 4])
def test_kmeans_constant_channels_degenerate_clusters(bits):
    """Channels with max == min (some exactly 0) form clusters with M == m: s = max(|m|,|M|)/qmax
    (1/qmax for zeros) and the values are reproduced exactly by quantize + dequantize."""
    rng = np.random.default_rng(bits)
    C, g = 1536, 24
    mx = rng.normal(0, 1, C).astype(np.float32)
    mn = (mx - rng.lognormal(0, 0.5, C)).astype(np.float32)
    const = rng.choice(C, 300, replace=False)
    vals = np.array([0.0, 0.0, 2.5, -3.25], dtype=np.float32)
    mx[const] = vals[np.arange(300) % 4]
    mn[const] = mx[const]
    ref = oracle.calibrate(mx, mn, g, 10, bits)
    out = rptq.rptq_kmeans(torch.from_numpy(mx).to(DEV), torch.from_numpy(mn).to(DEV), g, 10, bits)
    for k in ("labels", "R", "col_cluster", "offsets", "zero"):
        assert np.array_equal(to_np(out[k]), ref[k]), k
    assert np.array_equal(to_np(out["scale"]), ref["scale"])
    # quantize the constant values with their cluster's (s, z) and back: exact
    q = np.zeros((1, C), dtype=np.uint8)
    packed = oracle.pack(q, bits)
    deq = rptq.rptq_dequant(torch.from_numpy(packed).to(DEV), out["col_cluster"], out["scale"], out["zero"], bits,
                            out_dtype=torch.float32, C=C)
    assert np.array_equal(to_np(deq)[0], oracle.dequant(q, ref["col_cluster"], ref["scale"], ref["zero"])[0])


def _offset_rows(T, m, seed, dtype, all_offset=False):
    """Rows with zero variance (LayerNorm gives beta) and rows with a large common offset, where a
    single-pass variance cancels and -mean*rstd rounded once would shift a whole row."""
    x = synthetic.activations(T, m, seed, dtype=dtype).float()
    if all_offset:  # every row of every quad offset: the quad kernels' full-quad path
        x = x + torch.linspace(300.0, 3000.0, T)[:, None]
    else:
        x[1] = 0.0
        x[5] = 3.0
        x[7] = x[7] + 2000.0
        x[10] = x[10] * 1e-3 + 500.0
    return x.to(synthetic.torch_dtype(dtype))


@pytest.mark.parametrize("all_offset", [False, True])
@pytest.mark.parametrize("dtype,C", [("bf16", 12288), ("f16", 4096), ("f32", 768), ("bf16", 9216)])
def test_ln_quant_constant_and_offset_rows(dtype, C, all_offset):
    g, bits, seed = 16, 3, 11
    m, gamma, beta, cal = _cal(C, g, bits, seed, dtype)
    x = _offset_rows(12, m, seed, dtype, all_offset)
    p = dev_params(cal)
    codes, _ = rptq.rptq_ln_reorder_quant(x.to(DEV), gamma.to(DEV), beta.to(DEV), p["R"], p["col_cluster"],
                                          p["scale"], p["zero"], bits)
    ref, _, _ = oracle.ln_reorder_quant(x, gamma, beta, cal["R"], cal["col_cluster"], cal["scale"], cal["zero"], bits)
    compare_codes(to_np(codes), ref, C, bits, f"{dtype} C={C} constant/offset rows")
    # the general kernel (dense output) on the same rows
    _, ln = rptq.rptq_ln_reorder_quant(x.to(DEV), gamma.to(DEV), beta.to(DEV), p["R"], p["col_cluster"],
                                       p["scale"], p["zero"], bits, codes=None, ln_out=True)
    _, _, ln64 = oracle.ln_reorder_quant(x, gamma, beta, cal["R"], cal["col_cluster"], cal["scale"], cal["zero"],
                                         bits, want_ln=True)
    R = cal["R"]
    compare_ln(to_np(ln), ln64, gamma.numpy()[R][None].astype(np.float64),
               beta.numpy()[R][None].astype(np.float64), dtype, f"{dtype} C={C} dense, offset rows")


@pytest.mark.parametrize("all_offset", [False, True])
@pytest.mark.parametrize("dtype,C", [("bf16", 12288), ("f16", 1000), ("f32", 768), ("f32", 12288)])
def test_calib_layernorm_constant_and_offset_rows(dtype, C, all_offset):
    """LayerNorm calibration statistics over the same ill-conditioned rows (f32 rows of 12288
    channels take the general one-row-per-CTA kernel)."""
    m, gamma, beta = model_inputs(C, 19)
    x = _offset_rows(12, m, 19, dtype, all_offset)
    mx, mn = rptq.rptq_calib_minmax(x.to(DEV), gamma.to(DEV), beta.to(DEV), 1e-5)
    y64, _ = oracle.layernorm(x, gamma, beta)
    gm, bt = gamma.numpy().astype(np.float64), beta.numpy().astype(np.float64)
    compare_ln(to_np(mx)[None], y64.max(0)[None], gm[None], bt[None], "f32", "max")
    compare_ln(to_np(mn)[None], y64.min(0)[None], gm[None], bt[None], "f32", "min")


@pytest.mark.parametrize("S", [40, 128])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_kv_quant_huge_zero_point_integer_path(dtype, S):
    """Zero points beyond +-2^21 take the integer rounding path; codes are still exact (S = 40:
    the warp kernel; S = 128: whole 32 KB stages, the streaming-ring kernel)."""
    B, H, D, g, bits = 2, 3, 128, 4, 3
    mk = synthetic.channel_model(H * D, 17, tag=1)
    k = synthetic.kv_cache(B, H, S, D, mk, 17, "k", dtype)
    kf = oracle._f32(k)
    flat = np.ascontiguousarray(kf.transpose(0, 2, 1, 3).reshape(-1, H * D))
    kmx, kmn = oracle.minmax(flat)
    cal = oracle.calibrate(kmx, kmn, g, 5, bits)
    z = cal["zero"].copy()
    z[0] = 5_000_000
    z[1] = -4_000_000
    pk = oracle.kv_quant(kf, cal["labels"], cal["scale"], z, bits)
    kq, _ = rptq.rptq_kv_quant(k.to(DEV), None, torch.from_numpy(cal["labels"]).to(DEV),
                               torch.from_numpy(cal["scale"]).to(DEV), torch.from_numpy(z).to(DEV), None, None,
                               None, bits)
    assert np.array_equal(to_np(kq), pk)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("S", [40, 128])
def test_kv_quant_extreme_scales_and_overflowing_quotients(dtype, S):
    """Clusters with a scale below 2^-24 (the IEEE-division path) and values whose quotient x / s
    overflows fp32 (a positive overflow must give qmax, a negative one 0, as in the definition):
    codes are exact in both K/V kernels (S = 40: warp kernel; S = 128: streaming ring)."""
    B, H, D, g, bits = 2, 3, 128, 4, 3
    mk = synthetic.channel_model(H * D, 19, tag=1)
    k = synthetic.kv_cache(B, H, S, D, mk, 19, "k", dtype)
    kf = oracle._f32(k)
    flat = np.ascontiguousarray(kf.transpose(0, 2, 1, 3).reshape(-1, H * D))
    kmx, kmn = oracle.minmax(flat)
    cal = oracle.calibrate(kmx, kmn, g, 5, bits)
    s = cal["scale"].copy()
    big = 60000.0 if dtype == "f16" else 3.0e38
    s[0] = np.float32(2.0 ** -30)        # below the fast range
    s[1] = np.float32(1e-3 if dtype == "f16" else 1e-20)  # big values overflow x / s
    k2 = k.clone()
    lab = cal["labels"].reshape(H, D)
    for h in range(H):
        cols = np.nonzero(lab[h] == 1)[0]
        if len(cols):
            k2[:, h, ::3, cols[0]] = big
            k2[:, h, 1::3, cols[0]] = -big
    kf2 = oracle._f32(k2)
    pk = oracle.kv_quant(kf2, cal["labels"], s, cal["zero"], bits)
    kq, _ = rptq.rptq_kv_quant(k2.to(DEV), None, torch.from_numpy(cal["labels"]).to(DEV),
                               torch.from_numpy(s).to(DEV), torch.from_numpy(cal["zero"]).to(DEV), None, None,
                               None, bits)
    assert np.array_equal(to_np(kq), pk)
