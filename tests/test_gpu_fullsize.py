"""Parity at the full workload sizes, in the launch configurations the benchmark times.

Inputs are generated on the GPU with the seeded generator; the oracle recomputes sampled
outputs one by one (token rows for the fused quantizer and the K/V quantizer, channel columns
for raw calibration), and properties that hold at any size cover the LayerNorm calibration
over the full calibration batch.  Quantization parameters come from the oracle's calibration
on a slice of the calibration batch.
"""
import numpy as np
import pytest
import torch

import oracle
from post_activation_quantization_b200 import rptq, synthetic
from post_activation_quantization_b200.workloads import WORKLOADS
from tests.gpu_common import (DEV, compare_codes, compare_ln, dev_params, model_inputs,
                              oracle_calibration, to_np)

pytestmark = pytest.mark.gpu
ACT = ["tiny-768", "opt6.7b-4096", "opt66b-9216", "opt175b-12288"]
KVW = ["kv-4096", "opt175b-12288"]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_activation_quantization_b200 import build
    build.build()
    yield
    torch.cuda.empty_cache()
    assert rptq.rptq_device_error() == 0


def _act_setup(w):
    m, gamma, beta = model_inputs(w.C, w.seed, w.outlier_frac, w.outlier_factor)
    x = synthetic.activations(w.T, m, w.seed, dtype=w.dtype, device=DEV)
    if w.T_cal:
        xc = synthetic.activations(min(w.T_cal, 1024), m, w.seed, dtype=w.dtype, calibration=True,
                                   device=DEV).cpu()
    else:
        xc = x.cpu()
    cal = oracle_calibration(xc, gamma, beta, w.g, w.iters, w.bits)
    return m, gamma, beta, x, cal


@pytest.mark.parametrize("name", ACT)
def test_fused_quant_full_size_sampled_rows(name):
    w = WORKLOADS[name]
    m, gamma, beta, x, cal = _act_setup(w)
    p = dev_params(cal)
    codes, _ = rptq.rptq_ln_reorder_quant(x, gamma.to(DEV), beta.to(DEV), p["R"], p["col_cluster"],
                                          p["scale"], p["zero"], w.bits, eps=w.eps)
    torch.cuda.synchronize()
    n = min(w.T, 384)
    rows = np.unique(np.concatenate([[0, w.T - 1], np.random.default_rng(w.seed).choice(w.T, n, False)]))
    ri = torch.from_numpy(rows).to(DEV)
    xs = x[ri].cpu()
    ref, _, _ = oracle.ln_reorder_quant(xs, gamma, beta, cal["R"], cal["col_cluster"], cal["scale"],
                                        cal["zero"], w.bits, eps=w.eps)
    compare_codes(to_np(codes[ri]), ref, w.C, w.bits, name)
    # the planned launch the bench reports, on the same batch: every byte equal
    plan = rptq.rptq_ln_quant_plan(gamma.to(DEV), beta.to(DEV), p["R"], p["col_cluster"], p["scale"], p["zero"],
                                   w.bits)
    assert torch.equal(rptq.rptq_ln_reorder_quant_planned(x, plan, w.bits, eps=w.eps), codes), name


@pytest.mark.parametrize("name", [n for n in ACT if WORKLOADS[n].T_cal])
def test_calibration_full_batch_properties(name):
    """LayerNorm-mode statistics over the whole calibration batch: (a) two accumulated halves
    give exactly the one-call result (per-row arithmetic does not depend on the grid); (b) every
    sampled token's oracle LayerNorm lies inside [min, max] up to the LN tolerance; (c) on a
    1024-row slice the statistics match the oracle's."""
    w = WORKLOADS[name]
    m, gamma, beta = model_inputs(w.C, w.seed, w.outlier_frac, w.outlier_factor)
    xc = synthetic.activations(w.T_cal, m, w.seed, dtype=w.dtype, calibration=True, device=DEV)
    gd, bd = gamma.to(DEV), beta.to(DEV)
    mx, mn = rptq.rptq_calib_minmax(xc, gd, bd, w.eps)
    h = w.T_cal // 2 + 3
    mx2, mn2 = rptq.rptq_calib_minmax(xc[:h], gd, bd, w.eps)
    rptq.rptq_calib_minmax(xc[h:], gd, bd, w.eps, ch_max=mx2, ch_min=mn2, accumulate=True)
    assert torch.equal(mx, mx2) and torch.equal(mn, mn2)
    rows = np.random.default_rng(1).choice(w.T_cal, 256, replace=False)
    y64, _ = oracle.layernorm(xc[torch.from_numpy(rows).to(DEV)].cpu(), gamma, beta, w.eps)
    g64, b64 = gamma.numpy().astype(np.float64), beta.numpy().astype(np.float64)
    xhat = (y64 - b64) / g64
    tol = 1e-5 * (np.abs(g64) * (1 + np.abs(xhat)) + np.abs(b64))
    assert np.all(y64 <= to_np(mx)[None] + tol) and np.all(y64 >= to_np(mn)[None] - tol)
    sl = xc[:1024].contiguous()
    smx, smn = rptq.rptq_calib_minmax(sl, gd, bd, w.eps)
    rmx, rmn = oracle.minmax_ln(sl.cpu(), gamma, beta, w.eps)
    rng = (rmx.astype(np.float64) - b64) / g64
    compare_ln(to_np(smx)[None], rmx.astype(np.float64)[None], g64[None], b64[None], "f32", "max")
    compare_ln(to_np(smn)[None], rmn.astype(np.float64)[None], g64[None], b64[None], "f32", "min")
    del xc
    torch.cuda.empty_cache()


def _kv_setup(name):
    w = WORKLOADS[name]
    kvw = w.kv
    out = []
    for which, tag in (("k", 1), ("v", 2)):
        m = synthetic.channel_model(kvw.channels, w.seed, kvw.outlier_frac, kvw.outlier_factor, tag=tag)
        t = synthetic.kv_cache(kvw.B, kvw.H, kvw.S, kvw.D, m, w.seed, which, dtype=kvw.dtype, device=DEV)
        out.append(t)
    return w, kvw, out


@pytest.mark.parametrize("name", KVW)
def test_kv_full_size(name):
    w, kvw, (k, v) = _kv_setup(name)
    B, H, S, D = kvw.B, kvw.H, kvw.S, kvw.D
    rng = np.random.default_rng(w.seed)
    cals = []
    for t in (k, v):
        # raw calibration over the whole tensor: bit-exact on sampled channels
        mx, mn = rptq.rptq_calib_minmax(t.permute(0, 2, 1, 3).reshape(B * S, H * D).contiguous())
        ch = np.sort(rng.choice(H * D, 48, replace=False))
        cols = t.permute(0, 2, 1, 3).reshape(B * S, H * D)[:, torch.from_numpy(ch).to(DEV)].cpu()
        rmx, rmn = oracle.minmax(cols)
        assert np.array_equal(to_np(mx)[ch], rmx) and np.array_equal(to_np(mn)[ch], rmn)
        # parameters from the oracle's calibration on a token slice
        tok = t.permute(0, 2, 1, 3).reshape(B * S, H * D)[:2048].cpu()
        omx, omn = oracle.minmax(tok)
        cals.append(oracle.calibrate(omx, omn, kvw.g, kvw.iters, kvw.bits))
    pk, pv = dev_params(cals[0]), dev_params(cals[1])
    kq, vq = rptq.rptq_kv_quant(k, v, pk["labels"], pk["scale"], pk["zero"], pv["labels"],
                                pv["scale"], pv["zero"], kvw.bits)
    torch.cuda.synchronize()
    nrow = B * H * S
    rows = np.unique(np.concatenate([[0, nrow - 1], rng.choice(nrow, 2048, replace=False)]))
    ri = torch.from_numpy(rows).to(DEV)
    for t, cal, got in ((k, cals[0], kq), (v, cals[1], vq)):
        flat = t.reshape(nrow, D)[ri].cpu()
        hh = (rows // S) % H
        ref = np.empty((len(rows), D * kvw.bits // 8), np.uint8)
        for h in np.unique(hh):
            sel = hh == h
            q = oracle.quantize(flat[torch.from_numpy(np.nonzero(sel)[0])], cal["labels"][h * D:(h + 1) * D],
                                cal["scale"], cal["zero"], kvw.bits)
            ref[sel] = oracle.pack(q, kvw.bits)
        compare_codes(to_np(got.reshape(nrow, -1)[ri]), ref, D, kvw.bits, f"{name} kv")


@pytest.mark.parametrize("name", ["opt66b-9216", "opt175b-12288"])
def test_dequant_and_dynamic_ranges_full_size(name):
    """The rows-layout dequantization of the whole batch's codes into the batch's dtype (the call
    the benchmark times), bit-exact on sampled rows against oracle.dequant of the same codes; and
    the dynamic ranges of the whole batch: rptq_cluster_params of the GPU's LayerNorm statistics
    bit-exact against oracle.cluster_params of the same statistics (the statistics themselves are
    covered by the calibration tests above)."""
    w = WORKLOADS[name]
    m, gamma, beta, x, cal = _act_setup(w)
    p = dev_params(cal)
    gd, bd = gamma.to(DEV), beta.to(DEV)
    codes, _ = rptq.rptq_ln_reorder_quant(x, gd, bd, p["R"], p["col_cluster"], p["scale"], p["zero"], w.bits,
                                          eps=w.eps)
    out = torch.empty((w.T, w.C), dtype=x.dtype, device=DEV)
    rptq.rptq_dequant(codes, p["col_cluster"], p["scale"], p["zero"], w.bits, out=out)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, w.T - 1], np.random.default_rng(w.seed + 1).choice(w.T, 256, False)]))
    ri = torch.from_numpy(rows).to(DEV)
    q = oracle.unpack(to_np(codes[ri]), w.C, w.bits)
    ref = torch.from_numpy(oracle.dequant(q, cal["col_cluster"], cal["scale"], cal["zero"])).to(x.dtype)
    assert torch.equal(out[ri].cpu(), ref), name
    mx, mn = rptq.rptq_calib_minmax(x, gd, bd, w.eps)
    s, z = rptq.rptq_cluster_params(mx, mn, p["labels"], w.g, w.bits)
    rs, rz = oracle.cluster_params(to_np(mx), to_np(mn), cal["labels"], w.g, w.bits)
    assert np.array_equal(to_np(s).view(np.uint32), rs.view(np.uint32)) and np.array_equal(to_np(z), rz), name
    del x, out, codes
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", KVW)
def test_kv_cluster_order_and_dequant_full_size(name):
    """The K cache at full size stored in cluster order (rptq_kv_quant_cluster_ordered, as the
    benchmark launches it), sampled token rows against oracle.kv_quant_cluster_ordered of the
    same tokens; and the kept-layout codes of K and V read back by rptq_dequant's [B, H, S, D]
    layout, sampled rows bit-exact against oracle.kv_dequant."""
    w, kvw, (k, v) = _kv_setup(name)
    B, H, S, D, bits = kvw.B, kvw.H, kvw.S, kvw.D, kvw.bits
    C = H * D
    rng = np.random.default_rng(w.seed + 2)
    cals = []
    for t in (k, v):
        tok = t.permute(0, 2, 1, 3).reshape(B * S, C)[:2048].cpu()
        omx, omn = oracle.minmax(tok)
        cals.append(oracle.calibrate(omx, omn, kvw.g, kvw.iters, bits))
    pk, pv = dev_params(cals[0]), dev_params(cals[1])
    co = rptq.rptq_kv_quant_cluster_ordered(k, pk["R"], pk["col_cluster"], pk["scale"], pk["zero"], bits)
    torch.cuda.synchronize()
    tok = np.unique(np.concatenate([[0, B * S - 1], rng.choice(B * S, 384, replace=False)]))
    bi, si = torch.from_numpy(tok // S).to(DEV), torch.from_numpy(tok % S).to(DEV)
    sub = k[bi, :, si, :].unsqueeze(2).cpu()  # [n, H, 1, D]: every sampled token as its own batch row
    ref = oracle.kv_quant_cluster_ordered(sub, cals[0]["R"], cals[0]["col_cluster"], cals[0]["scale"],
                                          cals[0]["zero"], bits)
    compare_codes(to_np(co[bi, si]), ref.reshape(len(tok), -1), C, bits, f"{name} k cluster order")
    del co
    kq, vq = rptq.rptq_kv_quant(k, v, pk["labels"], pk["scale"], pk["zero"], pv["labels"], pv["scale"],
                                pv["zero"], bits)
    nrow = B * H * S
    rows = np.unique(np.concatenate([[0, nrow - 1], rng.choice(nrow, 1024, replace=False)]))
    ri = torch.from_numpy(rows).to(DEV)
    for codes, cal, pd, t in ((kq, cals[0], pk, k), (vq, cals[1], pv, v)):
        out = torch.empty((B, H, S, D), dtype=t.dtype, device=DEV)
        rptq.rptq_dequant(codes, pd["labels"], pd["scale"], pd["zero"], bits, layout=rptq.RPTQ_LAYOUT_BHSD, out=out)
        torch.cuda.synchronize()
        sel = codes.reshape(nrow, -1)[ri].cpu().numpy()
        hh = (rows // S) % H
        want = np.empty((len(rows), D), np.float32)
        for h in np.unique(hh):
            m_ = hh == h
            want[m_] = oracle.kv_dequant(sel[m_].reshape(1, 1, -1, D * bits // 8), D,
                                         cal["labels"][h * D:(h + 1) * D], cal["scale"], cal["zero"],
                                         bits).reshape(-1, D)
        assert torch.equal(out.reshape(nrow, D)[ri].cpu(), torch.from_numpy(want).to(t.dtype)), name
    del k, v, kq, vq
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", KVW)
def test_kv_decode_step_full_size(name):
    """The decode step as the benchmark launches it on the full caches: one new token appended
    at position S - 1 of the packed K and V caches, then attention of one query per (b, h) over
    all S positions.  The appended rows against oracle.kv_quant of the new token (codes bar, on
    every (b, h)); the attention of the first and last batch entries (all heads) against
    oracle.kv_decode_attention within the bound derived from the kernel's fp32 evaluation order."""
    from tests.test_gpu_kv_decode import _attn_bound
    w, kvw, (k, v) = _kv_setup(name)
    B, H, S, D, bits = kvw.B, kvw.H, kvw.S, kvw.D, kvw.bits
    C = H * D
    cals = []
    for t in (k, v):
        tok = t.permute(0, 2, 1, 3).reshape(B * S, C)[:2048].cpu()
        omx, omn = oracle.minmax(tok)
        cals.append(oracle.calibrate(omx, omn, kvw.g, kvw.iters, bits))
    pk, pv = dev_params(cals[0]), dev_params(cals[1])
    kq, vq = rptq.rptq_kv_quant(k, v, pk["labels"], pk["scale"], pk["zero"], pv["labels"], pv["scale"],
                                pv["zero"], bits)
    del k, v
    mk = synthetic.channel_model(kvw.channels, w.seed, kvw.outlier_frac, kvw.outlier_factor, tag=1)
    mv = synthetic.channel_model(kvw.channels, w.seed, kvw.outlier_frac, kvw.outlier_factor, tag=2)
    knew = synthetic.kv_cache(B, H, 1, D, mk, w.seed + 1, "k", dtype=kvw.dtype, device=DEV)
    vnew = synthetic.kv_cache(B, H, 1, D, mv, w.seed + 1, "v", dtype=kvw.dtype, device=DEV)
    rptq.rptq_kv_append(knew, vnew, pk["labels"], pk["scale"], pk["zero"], pv["labels"], pv["scale"], pv["zero"],
                        bits, k_cache=kq, v_cache=vq, s_begin=S - 1)
    for new, cal, cache in ((knew, cals[0], kq), (vnew, cals[1], vq)):
        ref = oracle.kv_quant(new.cpu(), cal["labels"], cal["scale"], cal["zero"], bits)
        compare_codes(to_np(cache[:, :, S - 1:S]), ref, D, bits, f"{name} appended row")
    gq = torch.Generator(device=DEV)
    gq.manual_seed(w.seed * 31)
    q = torch.randn((B, H, D), generator=gq, device=DEV, dtype=torch.float32) * 0.05
    out = rptq.rptq_kv_decode_attention(q, kq, vq, S, pk["labels"], pk["scale"], pk["zero"], pv["labels"],
                                        pv["scale"], pv["zero"], bits)
    torch.cuda.synchronize()
    bsel = torch.tensor([0, B - 1], device=DEV)
    qs, kc, vc = to_np(q[bsel]), kq[bsel].cpu().numpy(), vq[bsel].cpu().numpy()
    ref, _ = oracle.kv_decode_attention(qs, kc, vc, S, D, cals[0]["labels"], cals[0]["scale"], cals[0]["zero"],
                                        cals[1]["labels"], cals[1]["scale"], cals[1]["zero"], bits)
    Kd = oracle.kv_dequant(kc, D, cals[0]["labels"], cals[0]["scale"], cals[0]["zero"], bits)
    Vd = oracle.kv_dequant(vc, D, cals[1]["labels"], cals[1]["scale"], cals[1]["zero"], bits)
    tol = _attn_bound(qs, Kd, Vd, S, D, 1.0 / np.sqrt(D))
    err = np.abs(to_np(out[bsel]).astype(np.float64) - ref)
    assert (err <= tol).all(), f"{name}: worst excess {(err - tol).max():.3e}"
    del kq, vq
    torch.cuda.empty_cache()
