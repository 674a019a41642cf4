"""GPU parity of the reordered low-bit linear layer (rptq_linear_prepare + rptq_reordered_linear)
against the oracle's reordered_linear (the fp64 definition) and linear_fp16_operand (the fp16
operand the library computes with).

Three comparisons per case, each with its own bound:
  1. the prepared operand: w_prep (its columns put back in cluster order) and w_lambda equal the
     oracle's bit for bit; w_bias within one fp32 ulp (both sum in fp64, in different orders);
  2. the GEMM against the fp64 value on the SAME fp16 operand, Yb = f (q B^T - bz), f = s_w lam:
     only the tensor core's fp32 accumulation and the epilogue's two fp32 roundings remain,
         |Y - Yb| <= f [gam (q |B|^T) + 2^-23 (|acc| + |bz|)] + 2^-23 |Yb|,
     gam = (K/16 + 16) 2^-22 (one fp32 rounding per K = 16 step, at most one ulp each, plus
     slack for the adder's alignment inside a step, doubled).  A single wrong column (a code
     paired with another column's weight) moves Y by |q B| >> this bound;
  3. against the fp64 definition: bound 2 plus fp16's rounding of the operand,
         s_w 2^-11 (|q - z| |b|^T) (1 + 2^-20),  b = s_k (w - z_w) (the oracle's weights).
Tokens and outputs not multiples of the 128 x 256 tile, one-slab K, the vector and the scalar
store paths, A3 and A4, a zero weight row and the bench's full shape (sampled) are covered."""
import numpy as np
import pytest
import torch

import oracle
from post_activation_quantization_b200 import rptq, synthetic
from tests.gpu_common import DEV, REPORT, _key, dev_params, model_inputs, oracle_calibration, to_np

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


def _interleaved_to_cluster_order(wp: np.ndarray) -> np.ndarray:
    """Stored column 8m + 2i holds cluster-order column 8m + i, 8m + 2i + 1 holds 8m + 4 + i."""
    N, C = wp.shape
    js = np.arange(C)
    j = (js & ~7) | ((js & 1) << 2) | ((js >> 1) & 3)
    out = np.empty_like(wp)
    out[:, j] = wp
    return out


def _case(T, C, N, g, bits, seed, zero_row=None):
    m, gamma, beta = model_inputs(C, seed)
    xc = synthetic.activations(64, m, seed, dtype="f32", calibration=True)
    cal = oracle_calibration(xc, gamma, beta, g, 10, bits)
    x = synthetic.activations(T, m, seed, dtype="f32")
    codes, _, _ = oracle.ln_reorder_quant(x, gamma, beta, cal["R"], cal["col_cluster"], cal["scale"], cal["zero"],
                                          bits)
    W = synthetic.weights(N, C, seed).numpy()
    qw, sw, zw = oracle.quant_weights(W, 4)
    if zero_row is not None:  # every code at the row's zero point: b = 0
        qw[zero_row] = zw[zero_row]
    return cal, codes, qw, sw, zw


def _run(cal, codes, qw, sw, zw, C, bits):
    p = dev_params(cal)
    wq = torch.from_numpy(oracle.pack(qw, 4)).to(DEV)
    sw_d, zw_d = torch.from_numpy(sw).to(DEV), torch.from_numpy(zw).to(DEV)
    w_prep, w_bias, w_lam = rptq.rptq_linear_prepare(wq, zw_d, p["R"], p["col_cluster"], p["scale"], p["zero"])
    Y = rptq.rptq_reordered_linear(torch.from_numpy(codes).to(DEV), C, bits, w_prep, w_bias, w_lam, sw_d)
    torch.cuda.synchronize()
    return to_np(Y), to_np(w_prep), to_np(w_bias), to_np(w_lam)


def _check(Y, wp, wb, wl, cal, codes, qw, sw, zw, C, bits, what, rows=None, cols=None):
    """The three comparisons on the sampled rows x cols (all of them by default)."""
    cc, R, s, z = cal["col_cluster"], cal["R"], cal["scale"], cal["zero"]
    rows = np.arange(Y.shape[0]) if rows is None else rows
    cols = np.arange(Y.shape[1]) if cols is None else cols
    B, bz, lam = oracle.linear_fp16_operand(qw[cols], sw[cols], zw[cols], R, cc, s, z)
    # 1. the operand
    got = _interleaved_to_cluster_order(wp[cols].astype(np.float16))
    assert np.array_equal(got.view(np.uint16), B.view(np.uint16)), f"{what}: prepared weights differ"
    assert np.array_equal(wl[cols], lam), f"{what}: lambda differs"
    assert np.all(np.abs(wb[cols] - bz) <= 2.0 ** -23 * np.abs(bz)), f"{what}: bias beyond one ulp"
    # 2. the GEMM on the same operand
    q = oracle.unpack(codes[rows], C, bits).astype(np.float64)
    B64 = B.astype(np.float64)
    acc = q @ B64.T
    f = sw[cols].astype(np.float64) * lam.astype(np.float64)
    Yb = (acc - bz.astype(np.float64)[None, :]) * f[None, :]
    gam = (C / 16 + 16) * 2.0 ** -22
    tol2 = f[None, :] * (gam * (q @ np.abs(B64).T) + 2.0 ** -23 * (np.abs(acc) + np.abs(bz)[None, :])) \
        + 2.0 ** -23 * np.abs(Yb)
    Ys = Y[np.ix_(rows, cols)].astype(np.float64)
    err2 = np.abs(Ys - Yb)
    # 3. the definition
    Yd = oracle.reordered_linear(codes[rows], C, cc, s, z, bits, R, qw[cols], sw[cols], zw[cols])
    b = s[cc].astype(np.float64)[None, :] * (qw[cols][:, R].astype(np.float64) - zw[cols].astype(np.float64)[:, None])
    A = np.abs(q - z[cc].astype(np.float64)[None, :])
    tol3 = tol2 + sw[cols].astype(np.float64)[None, :] * 2.0 ** -11 * (A @ np.abs(b).T) * (1 + 2.0 ** -20)
    err3 = np.abs(Ys - Yd)
    REPORT.setdefault("linear", {})[_key(REPORT.setdefault("linear", {}), what)] = {
        "outputs": int(err2.size), "max_err_over_bound_operand": float((err2 / (tol2 + 1e-300)).max(initial=0)),
        "max_err_over_bound_definition": float((err3 / (tol3 + 1e-300)).max(initial=0)),
        "max_rel_to_definition": float((err3 / (np.abs(Yd) + 1e-30)).max(initial=0))}
    assert np.all(err2 <= tol2), f"{what}: {int((err2 > tol2).sum())} outputs off the fp16-operand value"
    assert np.all(err3 <= tol3), f"{what}: {int((err3 > tol3).sum())} outputs off the definition"


@pytest.mark.parametrize("T,C,N,g,bits", [
    (200, 256, 300, 8, 4),     # ragged token and output tiles, N % 4 == 0: vector stores with a tail
    (200, 256, 301, 8, 3),     # N % 4 != 0: scalar stores
    (128, 64, 256, 4, 4),      # exactly one tile, one K slab
    (1, 64, 1, 2, 3),          # one token, one output
    (1000, 768, 1000, 8, 4),   # the tiny layer's width, several tiles each way
    (257, 768, 520, 8, 3),
    (300, 1280, 384, 16, 4),   # K = 20 slabs: the six-slot ring wraps three times
])
def test_reordered_linear_matches_the_oracle(T, C, N, g, bits):
    seed = 3 * T + C + N
    cal, codes, qw, sw, zw = _case(T, C, N, g, bits, seed)
    Y, wp, wb, wl = _run(cal, codes, qw, sw, zw, C, bits)
    _check(Y, wp, wb, wl, cal, codes, qw, sw, zw, C, bits, f"linear T={T} C={C} N={N} A{bits}")


def test_zero_weight_row():
    T, C, N, g, bits = 130, 128, 40, 4, 4
    cal, codes, qw, sw, zw = _case(T, C, N, g, bits, 17, zero_row=5)
    Y, wp, wb, wl = _run(cal, codes, qw, sw, zw, C, bits)
    assert wl[5] == 1.0 and wb[5] == 0.0 and not wp[5].any()
    assert not Y[:, 5].any()
    _check(Y, wp, wb, wl, cal, codes, qw, sw, zw, C, bits, "linear zero weight row")


@pytest.mark.parametrize("bits", [4, 3])
def test_full_shape_sampled(bits):
    """The bench's layer: 2048 tokens x 4096 channels (the OPT-6.7B-shaped activations) into a
    12288-wide output (that model's fused Q/K/V projection), in the launch configuration the bench
    times; 96 sampled tokens x 96 sampled outputs, the last of each included."""
    T, C, N, g = 2048, 4096, 12288, 32
    cal, codes, qw, sw, zw = _case(T, C, N, g, bits, 29)
    Y, wp, wb, wl = _run(cal, codes, qw, sw, zw, C, bits)
    rng = np.random.default_rng(7)
    rows = np.unique(np.r_[rng.choice(T, 95, replace=False), T - 1])
    cols = np.unique(np.r_[rng.choice(N, 95, replace=False), N - 1])
    _check(Y, wp, wb, wl, cal, codes, qw, sw, zw, C, bits, f"linear full shape A{bits} (sampled)", rows, cols)
    assert np.isfinite(Y).all()


@pytest.mark.parametrize("C,g", [(12288, 64), (9216, 64)])
def test_bench_shape_sampled(C, g):
    """The layers the bench step runs for the OPT-175B- and OPT-66B-shaped workloads: 2048 tokens
    of A3 codes into the 3C-wide Q/K/V projection, with the bench's synthetic 4-bit weight codes;
    64 x 64 sampled outputs (the last token and output included)."""
    T, N, bits = 2048, 3 * C, 3
    cal, codes, _, _, _ = _case(T, C, 8, g, bits, 31)
    wq, sw_t, zw_t = synthetic.weight_codes(N, C, 31)
    p = dev_params(cal)
    sw_d, zw_d = sw_t.to(DEV), zw_t.to(DEV)
    w_prep, w_bias, w_lam = rptq.rptq_linear_prepare(wq.to(DEV), zw_d, p["R"], p["col_cluster"], p["scale"], p["zero"])
    Y = rptq.rptq_reordered_linear(torch.from_numpy(codes).to(DEV), C, bits, w_prep, w_bias, w_lam, sw_d)
    torch.cuda.synchronize()
    rng = np.random.default_rng(11)
    rows = np.unique(np.r_[rng.choice(T, 63, replace=False), T - 1])
    cols = np.unique(np.r_[rng.choice(N, 63, replace=False), N - 1])
    ci = torch.from_numpy(cols).to(DEV)
    # the sampled outputs' columns of Y and rows of the operand, gathered on the device
    Ys, wps, wbs, wls = to_np(Y[:, ci]), to_np(w_prep[ci]), to_np(w_bias[ci]), to_np(w_lam[ci])
    qws = oracle.unpack(wq.numpy()[cols], C, 4)
    _check(Ys, wps, wbs, wls, cal, codes, qws, sw_t.numpy()[cols], zw_t.numpy()[cols], C, bits,
           f"linear bench shape C={C} A3 (sampled)", rows)


@pytest.mark.parametrize("C,bits", [(4096, 4), (4096, 3), (768, 4), (1280, 3)])
def test_repeated_launches_are_bit_identical(C, bits):
    """The GEMM has a fixed accumulation order, so every launch on the same inputs must give the
    same bits: a race between the rings (a slot refilled while it is still read) shows up here as
    launches that differ, even where each result stays within the parity bounds.  2048 tokens into
    3C outputs (the bench's layer shape at C = 4096), 40 launches against the first."""
    T, N = 2048, 3 * C
    g = torch.Generator().manual_seed(C + bits)
    codes = torch.randint(0, 256, (T, C * bits // 8), dtype=torch.uint8, generator=g).to(DEV)
    w_prep = (torch.randn(N, C, generator=g) * 1000).half().to(DEV)
    bz, lam, sw = torch.randn(N, generator=g).to(DEV), torch.ones(N).to(DEV), torch.rand(N, generator=g).to(DEV)
    ref = rptq.rptq_reordered_linear(codes, C, bits, w_prep, bz, lam, sw)
    out = torch.empty_like(ref)
    differing = 0
    for _ in range(40):
        rptq.rptq_reordered_linear(codes, C, bits, w_prep, bz, lam, sw, out=out)
        differing += int(not torch.equal(out, ref))
    assert differing == 0, f"{differing} of 40 launches differ from the first"


def test_no_tokens_and_refused_shapes():
    C, N, g = 128, 64, 4
    cal, codes, qw, sw, zw = _case(4, C, N, g, 4, 5)
    p = dev_params(cal)
    wq = torch.from_numpy(oracle.pack(qw, 4)).to(DEV)
    sw_d, zw_d = torch.from_numpy(sw).to(DEV), torch.from_numpy(zw).to(DEV)
    w_prep, w_bias, w_lam = rptq.rptq_linear_prepare(wq, zw_d, p["R"], p["col_cluster"], p["scale"], p["zero"])
    empty = torch.empty((0, C // 2), dtype=torch.uint8, device=DEV)
    out = rptq.rptq_reordered_linear(empty, C, 4, w_prep, w_bias, w_lam, sw_d)
    assert out.shape == (0, N)
    bad = torch.zeros((4, 96 // 2), dtype=torch.uint8, device=DEV)  # C = 96: not a multiple of 64
    with pytest.raises(rptq.RptqError) as e:
        rptq.rptq_reordered_linear(bad, 96, 4, w_prep[:, :96].contiguous(), w_bias, w_lam, sw_d)
    assert e.value.status == -2
    with pytest.raises(rptq.RptqError) as e:
        rptq.rptq_reordered_linear(torch.from_numpy(codes).to(DEV), C, 5, w_prep, w_bias, w_lam, sw_d)
    assert e.value.status == -2


def test_out_of_range_reorder_entry_sets_the_error_word():
    C, N, g = 64, 8, 2
    cal, codes, qw, sw, zw = _case(4, C, N, g, 4, 9)
    p = dev_params(cal)
    R_bad = p["R"].clone()
    R_bad[3] = C + 5
    wq = torch.from_numpy(oracle.pack(qw, 4)).to(DEV)
    rptq.rptq_linear_prepare(wq, torch.from_numpy(zw).to(DEV), R_bad, p["col_cluster"], p["scale"], p["zero"])
    assert rptq.rptq_device_error() & 2
