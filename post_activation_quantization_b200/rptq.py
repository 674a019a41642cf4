"""ctypes binding of librptq.so (C ABI in include/rptq.h), entry points under the same names.

Argument marshalling only: every step runs in the library's CUDA kernels.  Tensors are torch
CUDA tensors (contiguous, on the current device); PyTorch supplies device memory and streams.
Outputs that are not passed in are allocated here with torch (plumbing, not compute).  There is
no CPU fallback: if the shared library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librptq.so")

RPTQ_OK = 0
RPTQ_ERR_INVALID_ARG = -1
RPTQ_ERR_UNSUPPORTED = -2
RPTQ_ERR_WORKSPACE = -3
RPTQ_ERR_CUDA = -4
RPTQ_ERR_DEVICE = -5
RPTQ_F32, RPTQ_F16, RPTQ_BF16 = 0, 1, 2
RPTQ_LAYOUT_ROWS, RPTQ_LAYOUT_BHSD = 0, 1
RPTQ_DEVERR_CLUSTER_ID, RPTQ_DEVERR_REORDER, RPTQ_DEVERR_TIMEOUT = 1, 2, 4
RPTQ_MAX_CHANNELS = 16384
RPTQ_MAX_CLUSTERS = 512

_DT = {torch.float32: RPTQ_F32, torch.float16: RPTQ_F16, torch.bfloat16: RPTQ_BF16}
_TD = {v: k for k, v in _DT.items()}

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SZ = ctypes.c_size_t

# name -> (restype, argtypes), mirroring include/rptq.h
SIGNATURES = {
    "rptq_status_string": (ctypes.c_char_p, [_I]),
    "rptq_version": (_I, []),
    "rptq_device_error": (_I, [_P, ctypes.POINTER(_I)]),
    "rptq_calib_minmax": (_I, [_P, _I, _I64, _I, _P, _P, _F, _P, _P, _I, _P]),
    "rptq_kv_calib_minmax": (_I, [_P, _I, _I, _I, _I64, _I, _P, _P, _I, _P]),
    "rptq_kmeans_workspace_size": (_SZ, [_I, _I]),
    "rptq_kmeans": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "rptq_kmeans_noalloc": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
    "rptq_ln_reorder_quant": (_I, [_P, _I, _I64, _I, _P, _P, _F, _P, _P, _P, _P, _I, _I, _P, _P, _P]),
    "rptq_kv_quant": (_I, [_P, _P, _I, _I, _I, _I64, _I, _P, _P, _P, _P, _P, _P, _I, _I, _P, _P, _P]),
    "rptq_kv_quant_cluster_ordered": (_I, [_P, _I, _I, _I, _I64, _I, _P, _P, _P, _P, _I, _I, _P, _P]),
    "rptq_dequant": (_I, [_P, _I, _I64, _I, _I64, _I, _P, _P, _P, _I, _I, _P, _I, _P]),
    "rptq_cluster_params": (_I, [_P, _P, _I, _P, _I, _I, _P, _P, _P]),
    "rptq_kv_append": (_I, [_P, _P, _I, _I, _I, _I64, _I, _I64, _I64, _P, _P, _P, _P, _P, _P, _I, _I, _P, _P, _P]),
    "rptq_kv_decode_attention": (_I, [_P, _I, _I, _I, _P, _P, _I64, _I64, _P, _P, _P, _P, _P, _P, _I, _I, _F, _P, _P]),
    "rptq_ln_quant_plan_bytes": (ctypes.c_size_t, [_I]),
    "rptq_ln_quant_plan": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P]),
    "rptq_ln_reorder_quant_planned": (_I, [_P, _I, _I64, _I, _F, _P, _I, _P, _P]),
    "rptq_linear_prepare": (_I, [_P, _P, _I, _I, _P, _P, _P, _P, _I, _P, _P, _P, _P]),
    "rptq_reordered_linear": (_I, [_P, _I64, _I, _I, _P, _P, _P, _P, _I, _P, _P]),
    # include/rptq_baseline.h
    "rptq_baseline_explicit_reorder_quant": (_I, [_P, _I, _I64, _I, _P, _P, _F, _P, _P, _P, _P, _I, _I, _P, _P, _P,
                                                  _P]),
    # include/rptq_testing.h
    "rptq_testing_kv_quotient": (_I, [_P, _I64, _F, _P, _P]),
    "rptq_testing_kmeans_wait": (_I, [ctypes.c_ulonglong, _I]),
}

_lib = None


class RptqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_text(status)} ({status})")


def lib() -> ctypes.CDLL:
    """The loaded library with argument types set (loads it on first use; raises if absent)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m post_activation_quantization_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _lib = h
    return _lib


def status_text(status: int) -> str:
    return lib().rptq_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != RPTQ_OK:
        raise RptqError(status, where)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "expected a contiguous CUDA tensor"
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


# ---------------------------------------------------------------------------------------------
def rptq_version() -> int:
    return lib().rptq_version()


def rptq_status_string(status: int) -> str:
    return status_text(status)


def rptq_device_error(stream=None) -> int:
    code = _I(0)
    _check(lib().rptq_device_error(_stream(stream), ctypes.byref(code)), "rptq_device_error")
    return code.value


def rptq_calib_minmax(x: torch.Tensor, gamma=None, beta=None, eps: float = 1e-5, ch_max=None,
                      ch_min=None, accumulate: bool = False, stream=None):
    """Per-channel (max, min) of x [T, C] (of LayerNorm(x) when gamma/beta are given)."""
    T, C = x.shape
    if ch_max is None:
        ch_max = torch.empty(C, dtype=torch.float32, device=x.device)
        ch_min = torch.empty(C, dtype=torch.float32, device=x.device)
    st = lib().rptq_calib_minmax(_ptr(x), _DT[x.dtype], T, C, _ptr(gamma), _ptr(beta), eps,
                                 _ptr(ch_max), _ptr(ch_min), int(bool(accumulate)), _stream(stream))
    _check(st, "rptq_calib_minmax")
    return ch_max, ch_min


def rptq_kv_calib_minmax(kv: torch.Tensor, ch_max=None, ch_min=None, accumulate: bool = False,
                         stream=None):
    """Per-channel (max, min) of a [B, H, S, D] cache, channel c = h*D + d, over B*S tokens."""
    B, H, S, D = kv.shape
    if ch_max is None:
        ch_max = torch.empty(H * D, dtype=torch.float32, device=kv.device)
        ch_min = torch.empty(H * D, dtype=torch.float32, device=kv.device)
    st = lib().rptq_kv_calib_minmax(_ptr(kv), _DT[kv.dtype], B, H, S, D, _ptr(ch_max), _ptr(ch_min),
                                    int(bool(accumulate)), _stream(stream))
    _check(st, "rptq_kv_calib_minmax")
    return ch_max, ch_min


def rptq_kmeans_workspace_size(C: int, g: int) -> int:
    return int(lib().rptq_kmeans_workspace_size(C, g))


def rptq_kmeans(ch_max: torch.Tensor, ch_min: torch.Tensor, g: int, iters: int, bits: int,
                workspace: torch.Tensor | None = None, out: dict | None = None, stream=None) -> dict:
    """KMeans + reorder + per-cluster (s, z).  Returns a dict of device tensors."""
    C = ch_max.numel()
    dev = ch_max.device
    if out is None:
        out = dict(
            labels=torch.empty(C, dtype=torch.int32, device=dev),
            centroids=torch.empty((g, 2), dtype=torch.float64, device=dev),
            R=torch.empty(C, dtype=torch.int32, device=dev),
            col_cluster=torch.empty(C, dtype=torch.int32, device=dev),
            offsets=torch.empty(g + 1, dtype=torch.int32, device=dev),
            scale=torch.empty(g, dtype=torch.float32, device=dev),
            zero=torch.empty(g, dtype=torch.int32, device=dev))
    if workspace is None:
        workspace = torch.empty(max(1, rptq_kmeans_workspace_size(C, g)), dtype=torch.uint8, device=dev)
    st = lib().rptq_kmeans(_ptr(ch_max), _ptr(ch_min), C, g, iters, bits, _ptr(out["labels"]),
                           _ptr(out["centroids"]), _ptr(out["R"]), _ptr(out["col_cluster"]),
                           _ptr(out["offsets"]), _ptr(out["scale"]), _ptr(out["zero"]),
                           _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "rptq_kmeans")
    return out


def rptq_kmeans_noalloc(ch_max: torch.Tensor, ch_min: torch.Tensor, g: int, iters: int, bits: int,
                        out: dict, stream=None) -> dict:
    """rptq_kmeans without a workspace (the library's fixed device scratch is used); `out` holds
    caller-allocated output tensors with the keys rptq_kmeans returns."""
    C = ch_max.numel()
    st = lib().rptq_kmeans_noalloc(_ptr(ch_max), _ptr(ch_min), C, g, iters, bits, _ptr(out["labels"]),
                                   _ptr(out["centroids"]), _ptr(out["R"]), _ptr(out["col_cluster"]),
                                   _ptr(out["offsets"]), _ptr(out["scale"]), _ptr(out["zero"]),
                                   _stream(stream))
    _check(st, "rptq_kmeans_noalloc")
    return out


def rptq_ln_reorder_quant(x: torch.Tensor, gamma, beta, R, col_cluster, scale, zero, bits: int,
                          eps: float = 1e-5, codes=True, ln_out=None, stream=None):
    """Reorder-fused LayerNorm + per-cluster quantization of x [T, C].

    codes: True (allocate), a uint8 [T, C*bits/8] tensor, or None; ln_out: None, True
    (allocate, x's dtype) or a [T, C] tensor.  Returns (codes, ln_out)."""
    T, C = x.shape
    if codes is True:
        codes = torch.empty((T, C * bits // 8), dtype=torch.uint8, device=x.device)
    if ln_out is True:
        ln_out = torch.empty((T, C), dtype=x.dtype, device=x.device)
    st = lib().rptq_ln_reorder_quant(_ptr(x), _DT[x.dtype], T, C, _ptr(gamma), _ptr(beta), eps,
                                     _ptr(R), _ptr(col_cluster), _ptr(scale), _ptr(zero),
                                     scale.numel(), bits, _ptr(codes), _ptr(ln_out), _stream(stream))
    _check(st, "rptq_ln_reorder_quant")
    return codes, ln_out


def rptq_kv_quant(k, v, cluster_k, scale_k, zero_k, cluster_v, scale_v, zero_v, bits: int,
                  k_codes=None, v_codes=None, stream=None):
    """Per-cluster quantization of K and V [B, H, S, D] (either may be None)."""
    ref = k if k is not None else v
    B, H, S, D = ref.shape
    shape = (B, H, S, D * bits // 8)
    if k is not None and k_codes is None:
        k_codes = torch.empty(shape, dtype=torch.uint8, device=ref.device)
    if v is not None and v_codes is None:
        v_codes = torch.empty(shape, dtype=torch.uint8, device=ref.device)
    g = (scale_k if scale_k is not None else scale_v).numel()
    st = lib().rptq_kv_quant(_ptr(k), _ptr(v), _DT[ref.dtype], B, H, S, D, _ptr(cluster_k),
                             _ptr(scale_k), _ptr(zero_k), _ptr(cluster_v), _ptr(scale_v),
                             _ptr(zero_v), g, bits, _ptr(k_codes), _ptr(v_codes), _stream(stream))
    _check(st, "rptq_kv_quant")
    return k_codes, v_codes


def rptq_kv_quant_cluster_ordered(kv, R, col_cluster, scale, zero, bits: int, codes=None, stream=None):
    """K or V [B, H, S, D] quantized per cluster and stored in cluster order: codes [B, S, C*bits/8]
    (C = H*D; stored column j holds channel R[j])."""
    B, H, S, D = kv.shape
    if codes is None:
        codes = torch.empty((B, S, H * D * bits // 8), dtype=torch.uint8, device=kv.device)
    st = lib().rptq_kv_quant_cluster_ordered(_ptr(kv), _DT[kv.dtype], B, H, S, D, _ptr(R), _ptr(col_cluster),
                                             _ptr(scale), _ptr(zero), scale.numel(), bits, _ptr(codes),
                                             _stream(stream))
    _check(st, "rptq_kv_quant_cluster_ordered")
    return codes


def rptq_dequant(codes: torch.Tensor, cluster, scale, zero, bits: int, out_dtype=torch.float32,
                 layout: int = RPTQ_LAYOUT_ROWS, C: int | None = None, D: int | None = None,
                 out=None, stream=None):
    """value = s * (q - z).  ROWS: codes [rows, C*bits/8] -> [rows, C]; BHSD: codes
    [B, H, S, D*bits/8] -> [B, H, S, D]."""
    if layout == RPTQ_LAYOUT_ROWS:
        rows = codes.shape[0]
        C = C if C is not None else codes.shape[1] * 8 // bits
        shape, n0, n1, S, Dd = (rows, C), rows, C, 0, 0
    else:
        B, H, S, pb = codes.shape
        Dd = D if D is not None else pb * 8 // bits
        shape, n0, n1 = (B, H, S, Dd), B, H
    if out is None:
        out = torch.empty(shape, dtype=out_dtype, device=codes.device)
    st = lib().rptq_dequant(_ptr(codes), layout, n0, n1, S, Dd, _ptr(cluster), _ptr(scale),
                            _ptr(zero), scale.numel(), bits, _ptr(out), _DT[out.dtype],
                            _stream(stream))
    _check(st, "rptq_dequant")
    return out


def rptq_cluster_params(ch_max, ch_min, labels, g: int, bits: int, scale=None, zero=None, stream=None):
    """Per-cluster (s, z) of fixed clusters from per-channel statistics (dynamic ranges)."""
    C = ch_max.numel()
    if scale is None:
        scale = torch.empty(g, dtype=torch.float32, device=ch_max.device)
        zero = torch.empty(g, dtype=torch.int32, device=ch_max.device)
    st = lib().rptq_cluster_params(_ptr(ch_max), _ptr(ch_min), C, _ptr(labels), g, bits, _ptr(scale), _ptr(zero),
                                   _stream(stream))
    _check(st, "rptq_cluster_params")
    return scale, zero


def rptq_kv_append(k_new, v_new, cluster_k, scale_k, zero_k, cluster_v, scale_v, zero_v, bits: int,
                   k_cache=None, v_cache=None, s_begin: int = 0, stream=None):
    """Quantize the new tokens [B, H, s_len, D] into positions s_begin.. of the packed caches
    [B, H, S_max, D*bits/8] (in place)."""
    t = k_new if k_new is not None else v_new
    B, H, s_len, D = t.shape
    cache = k_cache if k_cache is not None else v_cache
    S_max = cache.shape[2]
    g = (scale_k if scale_k is not None else scale_v).numel()
    st = lib().rptq_kv_append(_ptr(k_new), _ptr(v_new), _DT[t.dtype], B, H, s_len, D, S_max, s_begin,
                              _ptr(cluster_k), _ptr(scale_k), _ptr(zero_k), _ptr(cluster_v), _ptr(scale_v),
                              _ptr(zero_v), g, bits, _ptr(k_cache), _ptr(v_cache), _stream(stream))
    _check(st, "rptq_kv_append")
    return k_cache, v_cache


def rptq_kv_decode_attention(q, k_cache, v_cache, L: int, cluster_k, scale_k, zero_k, cluster_v, scale_v,
                             zero_v, bits: int, scale: float = 0.0, out=None, stream=None):
    """Softmax attention of q [B, H, D] (fp32) over positions 0..L-1 of the packed caches."""
    B, H, D = q.shape
    if out is None:
        out = torch.empty((B, H, D), dtype=torch.float32, device=q.device)
    st = lib().rptq_kv_decode_attention(_ptr(q), B, H, D, _ptr(k_cache), _ptr(v_cache), k_cache.shape[2], L,
                                        _ptr(cluster_k), _ptr(scale_k), _ptr(zero_k), _ptr(cluster_v),
                                        _ptr(scale_v), _ptr(zero_v), scale_k.numel(), bits, float(scale),
                                        _ptr(out), _stream(stream))
    _check(st, "rptq_kv_decode_attention")
    return out


def rptq_ln_quant_plan_bytes(C: int) -> int:
    """Bytes of the LayerNorm plan for C channels."""
    return int(lib().rptq_ln_quant_plan_bytes(C))


def rptq_ln_quant_plan(gamma, beta, R, col_cluster, scale, zero, bits: int, plan=None, stream=None):
    """The per-channel plan (code-buffer offsets and LayerNorm-quantization coefficients) of one
    calibration; returns the uint8 plan buffer."""
    C = R.numel()
    if plan is None:
        plan = torch.empty(rptq_ln_quant_plan_bytes(C), dtype=torch.uint8, device=R.device)
    st = lib().rptq_ln_quant_plan(_ptr(gamma), _ptr(beta), _ptr(R), _ptr(col_cluster), _ptr(scale), _ptr(zero), C,
                                  scale.numel(), bits, _ptr(plan), _stream(stream))
    _check(st, "rptq_ln_quant_plan")
    return plan


def rptq_ln_reorder_quant_planned(x: torch.Tensor, plan, bits: int, eps: float = 1e-5, codes=None, stream=None):
    """Packed cluster-ordered codes of x [T, C] from a plan (rptq_ln_quant_plan)."""
    T, C = x.shape
    if codes is None:
        codes = torch.empty((T, C * bits // 8), dtype=torch.uint8, device=x.device)
    st = lib().rptq_ln_reorder_quant_planned(_ptr(x), _DT[x.dtype], T, C, eps, _ptr(plan), bits, _ptr(codes),
                                             _stream(stream))
    _check(st, "rptq_ln_reorder_quant_planned")
    return codes


def rptq_linear_prepare(w_codes, w_zero, R, col_cluster, scale, zero, w_prep=None, w_bias=None, w_lambda=None,
                        stream=None):
    """Offline operand of the reordered linear layer from 4-bit weight codes w_codes [N, C/2]
    (original channel order) and the activation calibration; returns (w_prep fp16 [N, C],
    w_bias fp32 [N], w_lambda fp32 [N])."""
    N = w_codes.shape[0]
    C = R.numel()
    dev = w_codes.device
    if w_prep is None:
        w_prep = torch.empty((N, C), dtype=torch.float16, device=dev)
    if w_bias is None:
        w_bias = torch.empty(N, dtype=torch.float32, device=dev)
    if w_lambda is None:
        w_lambda = torch.empty(N, dtype=torch.float32, device=dev)
    st = lib().rptq_linear_prepare(_ptr(w_codes), _ptr(w_zero), N, C, _ptr(R), _ptr(col_cluster),
                                   _ptr(scale), _ptr(zero), scale.numel(), _ptr(w_prep), _ptr(w_bias),
                                   _ptr(w_lambda), _stream(stream))
    _check(st, "rptq_linear_prepare")
    return w_prep, w_bias, w_lambda


def rptq_reordered_linear(codes, C: int, bits: int, w_prep, w_bias, w_lambda, w_scale, out=None, stream=None):
    """out [T, N] fp32 = the linear layer applied to the packed cluster-ordered codes [T, C*bits/8]."""
    T = codes.shape[0]
    N = w_prep.shape[0]
    if out is None:
        out = torch.empty((T, N), dtype=torch.float32, device=codes.device)
    st = lib().rptq_reordered_linear(_ptr(codes), T, C, bits, _ptr(w_prep), _ptr(w_bias), _ptr(w_lambda),
                                     _ptr(w_scale), N, _ptr(out), _stream(stream))
    _check(st, "rptq_reordered_linear")
    return out


# ---------------------------------------------------------------------------------------------
# Measurement baselines (include/rptq_baseline.h)
def rptq_baseline_explicit_reorder_quant(x, gamma, beta, R, col_cluster, scale, zero, bits: int, eps: float = 1e-5,
                                         y=None, y_reordered=None, codes=None, stream=None):
    """The unfused LayerNorm -> explicit gather through R -> quantize pipeline (fp32
    intermediates in HBM); returns (codes, y, y_reordered)."""
    T, C = x.shape
    if y is None:
        y = torch.empty((T, C), dtype=torch.float32, device=x.device)
    if y_reordered is None:
        y_reordered = torch.empty((T, C), dtype=torch.float32, device=x.device)
    if codes is None:
        codes = torch.empty((T, C * bits // 8), dtype=torch.uint8, device=x.device)
    st = lib().rptq_baseline_explicit_reorder_quant(_ptr(x), _DT[x.dtype], T, C, _ptr(gamma), _ptr(beta), eps,
                                                    _ptr(R), _ptr(col_cluster), _ptr(scale), _ptr(zero),
                                                    scale.numel(), bits, _ptr(y), _ptr(y_reordered), _ptr(codes),
                                                    _stream(stream))
    _check(st, "rptq_baseline_explicit_reorder_quant")
    return codes, y, y_reordered


# ---------------------------------------------------------------------------------------------
# Test hooks (include/rptq_testing.h)
def rptq_testing_kv_quotient(x: torch.Tensor, s: float, q=None, stream=None) -> torch.Tensor:
    """The K/V quantizer's quotient x / s for every value of the fp32 tensor x."""
    assert x.dtype == torch.float32
    if q is None:
        q = torch.empty_like(x)
    _check(lib().rptq_testing_kv_quotient(_ptr(x), x.numel(), float(s), _ptr(q), _stream(stream)),
           "rptq_testing_kv_quotient")
    return q


def rptq_testing_kmeans_wait(limit_ns: int = 0, withhold_cta: int = -1) -> None:
    """KMeans exchange wait limit (0: the default) and a CTA that leaves out its first record."""
    _check(lib().rptq_testing_kmeans_wait(int(limit_ns), int(withhold_cta)), "rptq_testing_kmeans_wait")
