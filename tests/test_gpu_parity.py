"""GPU parity: every stage of the CUDA path against the CPU oracle on identical input bytes.

Stage-wise: each stage gets inputs that come from the seeded generator or from the oracle,
never from another CUDA stage, so every bit-exact gate tests one kernel.  Sizes here finish in
seconds on the oracle and still span several CTAs, ragged tails and the edge cases; the
full-size workloads are covered by tests/test_gpu_fullsize.py.
"""
import numpy as np
import pytest
import torch

import oracle
from post_activation_quantization_b200 import rptq, synthetic
from tests.gpu_common import (DEV, compare_codes, compare_ln, dev_params, model_inputs,
                              oracle_calibration, to_np)

pytestmark = pytest.mark.gpu

DTYPES = ["f32", "f16", "bf16"]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_activation_quantization_b200 import build
    build.build()
    rptq.lib()
    yield
    assert rptq.rptq_device_error() == 0


# ---------------------------------------------------------------- calibration min / max
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("T,C", [(1, 8), (37, 40), (1000, 768), (513, 4096), (3, 12288)])
def test_calib_raw_bit_exact(dtype, T, C):
    m, _, _ = model_inputs(C, 11)
    x = synthetic.activations(T, m, 11, dtype=dtype)
    mx, mn = rptq.rptq_calib_minmax(x.to(DEV))
    rmx, rmn = oracle.minmax(x)
    assert np.array_equal(to_np(mx), rmx) and np.array_equal(to_np(mn), rmn)


@pytest.mark.parametrize("dtype", DTYPES)
def test_calib_raw_accumulate_and_empty(dtype):
    C = 256
    m, _, _ = model_inputs(C, 12)
    x = synthetic.activations(300, m, 12, dtype=dtype)
    xd = x.to(DEV)
    mx, mn = rptq.rptq_calib_minmax(xd[:0])
    assert torch.all(torch.isneginf(mx)) and torch.all(torch.isposinf(mn))
    rptq.rptq_calib_minmax(xd[:100].contiguous(), ch_max=mx, ch_min=mn)
    rptq.rptq_calib_minmax(xd[100:].contiguous(), ch_max=mx, ch_min=mn, accumulate=True)
    rmx, rmn = oracle.minmax(x)
    assert np.array_equal(to_np(mx), rmx) and np.array_equal(to_np(mn), rmn)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("T,C", [(1, 8), (9, 40), (257, 768), (130, 4096), (21, 12288)])
def test_calib_layernorm_mode(dtype, T, C):
    m, gamma, beta = model_inputs(C, 13)
    gamma[3] = -gamma[3]  # a negative gamma swaps which extreme of the normalised value is used
    x = synthetic.activations(T, m, 13, dtype=dtype)
    mx, mn = rptq.rptq_calib_minmax(x.to(DEV), gamma.to(DEV), beta.to(DEV), 1e-5)
    y64, _ = oracle.layernorm(x, gamma, beta)
    g, b = gamma.numpy().astype(np.float64), beta.numpy().astype(np.float64)
    hi = y64.max(0)
    lo = y64.min(0)
    compare_ln(to_np(mx)[None], hi[None], g[None], b[None], "f32", "max")
    compare_ln(to_np(mn)[None], lo[None], g[None], b[None], "f32", "min")


# ---------------------------------------------------------------- KMeans + reorder + params
def _kmeans_case(C, g, iters, bits, seed, T=512, dtype="f32"):
    m, gamma, beta = model_inputs(C, seed)
    x = synthetic.activations(T, m, seed, dtype=dtype, calibration=True)
    mx, mn = oracle.minmax_ln(x, gamma, beta)
    return mx, mn


def _check_kmeans(mx, mn, g, iters, bits):
    ref = oracle.calibrate(mx, mn, g, iters, bits)
    out = rptq.rptq_kmeans(torch.from_numpy(mx).to(DEV), torch.from_numpy(mn).to(DEV), g, iters, bits)
    # the exact-label gate is meaningful when no point is near-equidistant from two centroids
    P = np.stack([mx, mn], 1).astype(np.float64)
    d = ((P[:, None, :] - ref["centroids"][None]) ** 2).sum(-1)
    if g > 1:
        part = np.partition(d, 1, axis=1)
        gap = (part[:, 1] - part[:, 0]) / np.maximum(part[:, 1], 1e-300)
        # exact ties (coinciding centroids) resolve to the lowest index on both sides
        assert np.all((gap == 0) | (gap > 1e-12)), "near-tie in the oracle's final assignment"
    assert np.array_equal(to_np(out["labels"]), ref["labels"])
    assert np.array_equal(to_np(out["R"]), ref["R"])
    assert np.array_equal(to_np(out["col_cluster"]), ref["col_cluster"])
    assert np.array_equal(to_np(out["offsets"]), ref["offsets"])
    np.testing.assert_allclose(to_np(out["centroids"]), ref["centroids"], rtol=1e-6, atol=1e-12)
    assert np.array_equal(to_np(out["scale"]), ref["scale"])
    assert np.array_equal(to_np(out["zero"]), ref["zero"])
    return out, ref


@pytest.mark.parametrize("C,g,iters,bits,seed", [
    (768, 8, 10, 4, 0), (4096, 32, 20, 4, 1), (4096, 32, 20, 3, 2), (9216, 64, 30, 3, 3),
    (12288, 64, 50, 3, 4), (1000, 7, 0, 3, 5), (40, 40, 5, 4, 6), (64, 1, 3, 4, 7), (8, 3, 4, 3, 8),
    (513, 16, 10, 4, 11), (16384, 512, 8, 3, 10), (16384, 64, 50, 3, 12)])
def test_kmeans_reorder_params(C, g, iters, bits, seed):
    mx, mn = _kmeans_case(C, g, iters, bits, seed, T=256 if C > 4096 else 512)
    _check_kmeans(mx, mn, g, iters, bits)


@pytest.mark.parametrize("C,distinct", [(512, 8), (2048, 8), (1500, 5)])
def test_kmeans_duplicate_points_and_empty_clusters(C, distinct):
    # few distinct points, each repeated across many channels (equal keys inside and across the
    # 512-channel segments the ranking is split into): ranks of equal keys follow the index
    rng = np.random.default_rng(9 + C)
    mx = rng.normal(0, 1, distinct)[rng.integers(0, distinct, C)].astype(np.float32)
    mn = (mx - 1.0).astype(np.float32)
    _check_kmeans(mx, mn, 16, 10, 3)


# ---------------------------------------------------------------- fused LN + reorder + quant
LN_CASES = [  # (dtype, T, C, g, bits)
    ("f32", 512, 768, 8, 4), ("f32", 7, 768, 8, 3), ("f16", 203, 4096, 32, 4),
    ("bf16", 130, 9216, 64, 3), ("bf16", 65, 12288, 64, 3), ("bf16", 1, 12288, 64, 4),
    ("f16", 6, 256, 5, 3), ("bf16", 33, 2048, 16, 4), ("f32", 9, 4096, 16, 3),
    ("bf16", 1203, 12288, 64, 3), ("f16", 97, 16384, 512, 4), ("bf16", 70, 8192, 300, 3),
    # several quads of four rows per CTA (148 CTAs): the double code buffer in turn, the kernels
    # compiled for fixed channel counts (4096, 9216, 12288), the generic 4-chunk split (8192)
    # and ragged last quads
    ("bf16", 2001, 9216, 64, 3), ("f16", 1779, 9216, 64, 4), ("bf16", 1802, 8192, 300, 3),
    ("f16", 2501, 4096, 32, 4), ("bf16", 1777, 12288, 64, 4), ("bf16", 3000, 5120, 40, 3)]


@pytest.mark.parametrize("dtype,T,C,g,bits", LN_CASES)
def test_ln_reorder_quant_codes(dtype, T, C, g, bits):
    seed = T + C
    m, gamma, beta = model_inputs(C, seed)
    xc = synthetic.activations(max(64, T), m, seed, dtype=dtype, calibration=True)
    cal = oracle_calibration(xc, gamma, beta, g, 10, bits)
    x = synthetic.activations(T, m, seed, dtype=dtype)
    p = dev_params(cal)
    codes, _ = rptq.rptq_ln_reorder_quant(x.to(DEV), gamma.to(DEV), beta.to(DEV), p["R"],
                                          p["col_cluster"], p["scale"], p["zero"], bits)
    ref, _, _ = oracle.ln_reorder_quant(x, gamma, beta, cal["R"], cal["col_cluster"], cal["scale"],
                                        cal["zero"], bits)
    compare_codes(to_np(codes), ref, C, bits, f"{dtype} T={T} C={C}")


@pytest.mark.parametrize("dtype,T,C,g,bits", [("bf16", 37, 12288, 64, 3), ("f16", 9, 4096, 32, 4),
                                               ("bf16", 21, 9216, 64, 3)])
def test_ln_reorder_quant_unaligned_tables(dtype, T, C, g, bits):
    """R and col_cluster 4 bytes off a 16-byte boundary: the kernel that stages rows through the
    shared-memory ring (no vector loads of the tables) gives the same codes."""
    seed = 5 * T + C
    m, gamma, beta = model_inputs(C, seed)
    xc = synthetic.activations(64, m, seed, dtype=dtype, calibration=True)
    cal = oracle_calibration(xc, gamma, beta, g, 10, bits)
    x = synthetic.activations(T, m, seed, dtype=dtype)
    p = dev_params(cal)
    bufR = torch.empty(C + 4, dtype=torch.int32, device=DEV)
    bufK = torch.empty(C + 4, dtype=torch.int32, device=DEV)
    R, K = bufR[1:C + 1], bufK[1:C + 1]
    R.copy_(p["R"])
    K.copy_(p["col_cluster"])
    assert R.data_ptr() % 16 != 0
    codes, _ = rptq.rptq_ln_reorder_quant(x.to(DEV), gamma.to(DEV), beta.to(DEV), R, K, p["scale"], p["zero"], bits)
    ref, _, _ = oracle.ln_reorder_quant(x, gamma, beta, cal["R"], cal["col_cluster"], cal["scale"],
                                        cal["zero"], bits)
    compare_codes(to_np(codes), ref, C, bits, f"unaligned {dtype} T={T} C={C}")


@pytest.mark.parametrize("dtype,T,C,g,bits", [
    ("f32", 64, 768, 8, 4), ("f16", 40, 4096, 32, 4), ("bf16", 17, 12288, 64, 3),
    ("bf16", 5, 16384, 64, 3), ("f32", 3, 72, 4, 3)])
@pytest.mark.parametrize("want_codes", [True, False])
def test_ln_reorder_dense_output_and_general_path(dtype, T, C, g, bits, want_codes):
    """The dense cluster-ordered LayerNorm output (and the general kernel that writes it)."""
    seed = 3 * T + C
    m, gamma, beta = model_inputs(C, seed)
    xc = synthetic.activations(64, m, seed, dtype=dtype, calibration=True)
    cal = oracle_calibration(xc, gamma, beta, g, 10, bits)
    x = synthetic.activations(T, m, seed, dtype=dtype)
    p = dev_params(cal)
    codes, ln = rptq.rptq_ln_reorder_quant(x.to(DEV), gamma.to(DEV), beta.to(DEV), p["R"],
                                           p["col_cluster"], p["scale"], p["zero"], bits,
                                           codes=want_codes or None, ln_out=True)
    ref, ln32, ln64 = oracle.ln_reorder_quant(x, gamma, beta, cal["R"], cal["col_cluster"],
                                              cal["scale"], cal["zero"], bits, want_ln=True)
    R = cal["R"]
    compare_ln(to_np(ln), ln64, gamma.numpy()[R][None].astype(np.float64),
               beta.numpy()[R][None].astype(np.float64), dtype, f"{dtype} C={C}")
    if want_codes:
        compare_codes(to_np(codes), ref, C, bits, "general path")


def test_ln_reorder_is_ln_then_gather():
    """Fusion invariant on the GPU: with R = identity and one cluster the dense output equals
    LayerNorm in channel order; with a permutation it equals that output gathered by R."""
    C, T = 1024, 12
    m, gamma, beta = model_inputs(C, 21)
    x = synthetic.activations(T, m, 21, dtype="f32").to(DEV)
    one = torch.zeros(C, dtype=torch.int32, device=DEV)
    s = torch.ones(1, device=DEV)
    z = torch.zeros(1, dtype=torch.int32, device=DEV)
    ident = torch.arange(C, dtype=torch.int32, device=DEV)
    perm = torch.randperm(C, generator=torch.Generator().manual_seed(0)).to(torch.int32).to(DEV)
    _, ln_id = rptq.rptq_ln_reorder_quant(x, gamma.to(DEV), beta.to(DEV), ident, one, s, z, 4,
                                          codes=None, ln_out=True)
    _, ln_p = rptq.rptq_ln_reorder_quant(x, gamma.to(DEV), beta.to(DEV), perm, one, s, z, 4,
                                         codes=None, ln_out=True)
    assert torch.equal(ln_p, ln_id[:, perm.long()])


# ---------------------------------------------------------------- K/V cache
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("B,H,S,D", [(2, 3, 37, 128), (1, 2, 5, 40), (3, 1, 300, 8), (1, 4, 64, 256),
                                     # whole 32 KB stages (16-bit): the streaming-ring kernel; the
                                     # last case has more stages than CTAs, so CTAs cross heads
                                     (2, 3, 128, 128), (1, 2, 2048, 8), (2, 5, 512, 32), (1, 2, 8, 2048),
                                     (2, 4, 16384, 128),
                                     # channel groups spanning two warps (D = 512); many short heads
                                     (2, 2, 64, 512), (3, 6, 256, 64)])
def test_kv_calib_bit_exact(dtype, B, H, S, D):
    m = synthetic.channel_model(H * D, S, tag=1)
    kv = synthetic.kv_cache(B, H, S, D, m, S, "k", dtype=dtype)
    mx, mn = rptq.rptq_kv_calib_minmax(kv.to(DEV))
    flat = kv.float().permute(0, 2, 1, 3).reshape(B * S, H * D)
    rmx, rmn = oracle.minmax(flat)
    assert np.array_equal(to_np(mx), rmx) and np.array_equal(to_np(mn), rmn)
    # accumulate: fold a second batch in
    kv2 = synthetic.kv_cache(B, H, S, D, m, S + 1, "k", dtype=dtype)
    rptq.rptq_kv_calib_minmax(kv2.to(DEV), ch_max=mx, ch_min=mn, accumulate=True)
    rmx2, rmn2 = oracle.minmax(kv2.float().permute(0, 2, 1, 3).reshape(B * S, H * D), rmx, rmn)
    assert np.array_equal(to_np(mx), rmx2) and np.array_equal(to_np(mn), rmn2)


KV_CASES = [("f16", 2, 4, 33, 128, 6, 3), ("bf16", 1, 3, 17, 64, 5, 4), ("f32", 2, 2, 9, 128, 8, 4),
            ("f16", 1, 2, 11, 40, 4, 3), ("bf16", 3, 5, 7, 256, 7, 3), ("bf16", 2, 3, 300, 128, 6, 3),
            ("f16", 1, 2, 5, 512, 4, 4), ("bf16", 2, 2, 130, 32, 5, 3), ("f32", 1, 3, 19, 8, 3, 4),
            # whole 32 KB stages per (b, h) block (S a multiple of 16384 / D): the streaming-ring kernel
            ("bf16", 2, 3, 128, 128, 6, 3), ("f16", 2, 3, 384, 128, 5, 4), ("bf16", 1, 4, 256, 64, 7, 4),
            ("f16", 3, 2, 64, 256, 6, 3), ("bf16", 1, 2, 8, 2048, 4, 3), ("f16", 1, 3, 2048, 8, 3, 4),
            ("bf16", 2, 5, 512, 32, 9, 3), ("bf16", 1, 3, 192, 128, 5, 3),
            ("bf16", 2, 4, 4096, 128, 6, 3)]  # more stages than CTAs: CTAs cross heads and tensors


@pytest.mark.parametrize("dtype,B,H,S,D,g,bits", KV_CASES)
def test_kv_quant(dtype, B, H, S, D, g, bits):
    seed = B * 100 + H * 10 + D
    mk = synthetic.channel_model(H * D, seed, tag=1)
    mv = synthetic.channel_model(H * D, seed, tag=2)
    k = synthetic.kv_cache(B, H, S, D, mk, seed, "k", dtype=dtype)
    v = synthetic.kv_cache(B, H, S, D, mv, seed, "v", dtype=dtype)
    cals = []
    for t in (k, v):
        flat = t.float().permute(0, 2, 1, 3).reshape(B * S, H * D).numpy()
        mx, mn = oracle.minmax(flat)
        cals.append(oracle.calibrate(mx, mn, g, 10, bits))
    pk, pv = dev_params(cals[0]), dev_params(cals[1])
    kq, vq = rptq.rptq_kv_quant(k.to(DEV), v.to(DEV), pk["labels"], pk["scale"], pk["zero"],
                                pv["labels"], pv["scale"], pv["zero"], bits)
    for t, cal, got in ((k, cals[0], kq), (v, cals[1], vq)):
        ref = oracle.kv_quant(t, cal["labels"], cal["scale"], cal["zero"], bits)
        compare_codes(to_np(got).reshape(-1, D * bits // 8), ref.reshape(-1, D * bits // 8), D, bits,
                      f"kv {dtype}")
    # one tensor alone
    kq2, vq2 = rptq.rptq_kv_quant(k.to(DEV), None, pk["labels"], pk["scale"], pk["zero"], None, None,
                                  None, bits)
    assert vq2 is None and torch.equal(kq2, kq)
    kq3, vq3 = rptq.rptq_kv_quant(None, v.to(DEV), None, None, None, pv["labels"], pv["scale"], pv["zero"], bits)
    assert kq3 is None and torch.equal(vq3, vq)


# ---------------------------------------------------------------- dequantization
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("rows,C,bits", [(37, 768, 4), (5, 4096, 3), (3, 72, 3), (2, 40, 4), (9, 12288, 3),
                                         (6, 12288, 4), (11, 9216, 3), (4, 256, 3), (3, 16384, 4),
                                         # rows split over several CTAs (column ranges), one row among them
                                         (7, 5120, 4), (1, 9216, 3)])
def test_dequant_rows_bit_exact(out_dtype, rows, C, bits):
    rng = np.random.default_rng(rows * C)
    g = 9
    cc = np.sort(rng.integers(0, g, C)).astype(np.int32)
    s = rng.lognormal(-3, 1, g).astype(np.float32)
    z = rng.integers(-70, 80, g).astype(np.int32)
    z[0] = 9_000_000  # beyond the exact float path: the integer path is used for that thread
    q = rng.integers(0, 2 ** bits, (rows, C)).astype(np.uint8)
    packed = oracle.pack(q, bits)
    out = rptq.rptq_dequant(torch.from_numpy(packed).to(DEV), torch.from_numpy(cc).to(DEV),
                            torch.from_numpy(s).to(DEV), torch.from_numpy(z).to(DEV), bits,
                            out_dtype=out_dtype, C=C)
    ref = torch.from_numpy(oracle.dequant(q, cc, s, z)).to(out_dtype)
    assert torch.equal(out.cpu(), ref)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("B,H,S,D,bits", [(2, 3, 5, 128, 3), (1, 2, 4, 40, 4), (1, 4, 3, 64, 4), (2, 2, 67, 128, 3),
                                          (1, 3, 9, 256, 4), (2, 1, 35, 8, 3), (2, 1, 36, 8, 3), (1, 2, 13, 32, 3),
                                          (1, 1, 16, 16, 4),
                                          # whole 32 KB output stages (16-bit outputs): the ring kernel;
                                          # the last case has more stages than CTAs
                                          (2, 3, 128, 128, 3), (1, 4, 256, 64, 4), (2, 2, 64, 256, 3),
                                          (1, 2, 2048, 8, 4), (1, 2, 8, 2048, 3), (2, 4, 8192, 128, 3)])
@pytest.mark.parametrize("huge_z", [False, True])
def test_dequant_bhsd_bit_exact(B, H, S, D, bits, huge_z, out_dtype):
    rng = np.random.default_rng(B * H * S * D)
    g = 6
    labels = rng.integers(0, g, H * D).astype(np.int32)
    s = rng.lognormal(-2, 1, g).astype(np.float32)
    z = rng.integers(-30, 30, g).astype(np.int32)
    if huge_z:
        z[labels[0]] = -9_000_000  # beyond the exact float path
    q = rng.integers(0, 2 ** bits, (B * H * S, D)).astype(np.uint8)
    packed = oracle.pack(q, bits).reshape(B, H, S, D * bits // 8)
    out = rptq.rptq_dequant(torch.from_numpy(packed).to(DEV), torch.from_numpy(labels).to(DEV),
                            torch.from_numpy(s).to(DEV), torch.from_numpy(z).to(DEV), bits,
                            out_dtype=out_dtype, layout=rptq.RPTQ_LAYOUT_BHSD, D=D)
    ref = torch.from_numpy(oracle.kv_dequant(packed, D, labels, s, z, bits)).to(out_dtype)
    assert torch.equal(out.cpu(), ref)


# ---------------------------------------------------------------- device error word
def test_device_error_flags_bad_tables():
    C, T = 256, 8
    m, gamma, beta = model_inputs(C, 31)
    x = synthetic.activations(T, m, 31, dtype="bf16").to(DEV)
    R = torch.arange(C, dtype=torch.int32, device=DEV)
    cc = torch.zeros(C, dtype=torch.int32, device=DEV)
    cc[5] = 7  # outside [0, g) with g = 2
    s = torch.ones(2, device=DEV)
    z = torch.zeros(2, dtype=torch.int32, device=DEV)
    assert rptq.rptq_device_error() == 0
    rptq.rptq_ln_reorder_quant(x, gamma.to(DEV), beta.to(DEV), R, cc, s, z, 3)
    assert rptq.rptq_device_error() & rptq.RPTQ_DEVERR_CLUSTER_ID
    R2 = R.clone()
    R2[3] = C + 5
    rptq.rptq_ln_reorder_quant(x, gamma.to(DEV), beta.to(DEV), R2, torch.zeros_like(cc), s, z, 3)
    assert rptq.rptq_device_error() & rptq.RPTQ_DEVERR_REORDER
    assert rptq.rptq_device_error() == 0  # read-and-clear


def test_invalid_calls_raise():
    x = torch.zeros((4, 60), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(rptq.RptqError) as e:
        rptq.rptq_calib_minmax(x)
    assert e.value.status == rptq.RPTQ_ERR_UNSUPPORTED


# ---------------------------------------------------------------- whole chain, both sides
@pytest.mark.parametrize("name", ["tiny-768"])
def test_chain_gpu_vs_oracle(name):
    """GPU chain (calib -> kmeans -> fused quant) against the oracle chain on the same bytes."""
    from post_activation_quantization_b200.workloads import WORKLOADS
    w = WORKLOADS[name]
    m, gamma, beta = model_inputs(w.C, w.seed, w.outlier_frac, w.outlier_factor)
    x = synthetic.activations(w.T, m, w.seed, dtype=w.dtype)  # calibrate on the same X
    xd, gd, bd = x.to(DEV), gamma.to(DEV), beta.to(DEV)
    mx, mn = rptq.rptq_calib_minmax(xd, gd, bd, w.eps)
    out = rptq.rptq_kmeans(mx, mn, w.g, w.iters, w.bits)
    codes, _ = rptq.rptq_ln_reorder_quant(xd, gd, bd, out["R"], out["col_cluster"], out["scale"],
                                          out["zero"], w.bits, eps=w.eps)
    rmx, rmn = oracle.minmax_ln(x, gamma, beta, w.eps)
    cal = oracle.calibrate(rmx, rmn, w.g, w.iters, w.bits)
    assert np.array_equal(to_np(out["R"]), cal["R"])
    np.testing.assert_allclose(to_np(out["scale"]), cal["scale"], rtol=1e-5)
    assert np.abs(to_np(out["zero"]) - cal["zero"]).max() <= 1
    ref, _, _ = oracle.ln_reorder_quant(x, gamma, beta, cal["R"], cal["col_cluster"], cal["scale"],
                                        cal["zero"], w.bits, eps=w.eps)
    compare_codes(to_np(codes), ref, w.C, w.bits, "chain")
