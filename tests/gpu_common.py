"""Helpers for the GPU parity tests: seeded inputs, oracle calls and the comparison rules.

Tolerances (each follows from the arithmetic of the two sides):
  * min/max in raw mode, R, labels, offsets, col_cluster, scale, zero, dequantized values:
    bit-exact;
  * centroids: relative 1e-6 (the GPU sums cluster members in a different fixed order);
  * codes: identical except +-1 at rounding boundaries, on at most 1e-4 of the elements;
  * LayerNorm output (fp32): |gpu - y| <= 1e-5 |y| + 2.5e-7, y from the oracle's fp64
    LayerNorm.  Measured on a B200 over the suite's 63 fp32 comparisons (dense outputs and
    LayerNorm-mode calibration statistics, all three input types, offset rows included): the
    worst error is within 1e-5 |y| + 6.6e-8, so the floor keeps a factor of about 4; where
    |y| ~ 1e-3 the relative error alone reaches 4.8e-5 (the fp32 rounding of the mean and of
    rstd moves y by a few 1e-8 absolute).  A bf16 output adds one round-to-nearest of 8
    significant bits, at most 2^-8 |y|; fp16 adds 2^-11 |y| + 2^-25.
"""
import numpy as np
import torch

import oracle
from post_activation_quantization_b200 import synthetic

DEV = "cuda"
CODE_OFF_BY_ONE_MAX = 1e-4


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype in (torch.float16, torch.bfloat16):
        t = t.float()
    return t.detach().cpu().numpy()


# measured agreement of every comparison in this session (written out by conftest.py when
# RPTQ_PARITY_REPORT names a file): codes -> off-by-one fraction, LN -> worst errors
REPORT = {"codes": {}, "ln": {}}


def compare_codes(gpu_packed: np.ndarray, ref_packed: np.ndarray, C: int, bits: int, what=""):
    """Unpack both and apply the codes bar; returns the off-by-one fraction."""
    g = oracle.unpack(gpu_packed.reshape(-1, C * bits // 8), C, bits).astype(np.int16)
    r = oracle.unpack(ref_packed.reshape(-1, C * bits // 8), C, bits).astype(np.int16)
    d = np.abs(g - r)
    frac = float((d == 1).mean()) if d.size else 0.0
    REPORT["codes"][_key(REPORT["codes"], what)] = {"elements": int(d.size), "off_by_one": int((d == 1).sum()), "fraction": frac,
                             "max_diff": int(d.max(initial=0))}
    assert d.max(initial=0) <= 1, f"{what}: code differs by {d.max()} (> 1)"
    assert frac <= CODE_OFF_BY_ONE_MAX, f"{what}: off-by-one fraction {frac:.2e}"
    return frac


LN_REL32, LN_ABS32 = 1e-5, 2.5e-7


def ln_tol32(y64: np.ndarray, gamma_s=None, beta_s=None) -> np.ndarray:
    return LN_REL32 * np.abs(y64) + LN_ABS32


def _key(table: dict, what: str) -> str:
    k, n = what, 1
    while k in table:
        n += 1
        k = f"{what} #{n}"
    return k


def compare_ln(gpu: np.ndarray, y64: np.ndarray, gamma_s, beta_s, dtype: str, what=""):
    tol = ln_tol32(y64, gamma_s, beta_s)
    if dtype == "bf16":
        tol = tol + 2.0 ** -8 * np.abs(y64) * (1 + 1e-5)
    elif dtype == "f16":
        tol = tol + 2.0 ** -11 * np.abs(y64) * (1 + 1e-5) + 2.0 ** -25
    err = np.abs(gpu.astype(np.float64) - y64)
    ay = np.abs(y64)
    rel = err[ay > 1e-3] / ay[ay > 1e-3]
    REPORT["ln"][_key(REPORT["ln"], f"{what} ({dtype})")] = {
        "values": int(err.size), "max_abs": float(err.max(initial=0)),
        "max_rel_where_abs_y_gt_1e-3": float(rel.max(initial=0)),
        "max_excess_over_1e-5_rel": float((err - 1e-5 * ay).max(initial=0))}
    bad = err > tol
    assert not bad.any(), f"{what}: {bad.sum()} LN values out of tolerance, worst {(err - tol).max():.3e}"


def model_inputs(C, seed, outlier_frac=0.01, outlier_factor=100.0):
    m = synthetic.channel_model(C, seed, outlier_frac, outlier_factor)
    gamma, beta = synthetic.ln_params(C, seed)
    return m, gamma, beta


def oracle_calibration(x_cal_cpu, gamma, beta, g, iters, bits):
    """Oracle statistics of LN(x_cal) and the oracle's calibration chain on them."""
    mx, mn = oracle.minmax_ln(x_cal_cpu, gamma, beta)
    cal = oracle.calibrate(mx, mn, g, iters, bits)
    cal["ch_max"], cal["ch_min"] = mx, mn
    return cal


def dev_params(cal):
    """Oracle calibration outputs as device tensors (inputs to the CUDA path)."""
    return {k: torch.from_numpy(np.ascontiguousarray(cal[k])).to(DEV)
            for k in ("R", "col_cluster", "scale", "zero", "labels")}
