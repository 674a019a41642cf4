"""CPU oracle for the RPTQ data path -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import this package.  The product path (``post_activation_quantization_b200``)
never imports it and fails loudly when its CUDA library is missing.

The arithmetic lives in ``rptq_oracle.c`` (plain single-threaded C, fp64 unless a step fixes
fp32, built with ``-ffp-contract=off``); this module only marshals numpy arrays into it.
Inputs in fp16/bf16 are widened to fp32 here, which is exact.

Sources (page title + part), the same as in the C file:
  [RPTQ-art]  "基于重排序的新量化方法RPTQ：实现大型语言模型的 3 比特量化": Fig. 1 caption, the text
              after Fig. 2 (calibration, KMeans, reorder, per-cluster s/z), the text after Fig. 3
              (LayerNorm emits reordered activations), the results paragraph (K/V quantization).
  [Basics]    quantization-basics article (gitcode.csdn.net), sections 一, 1.1, 1.3, 1.4.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rptq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library in place (gcc, -O2 -ffp-contract=off)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB)
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(x) -> np.ndarray:
    """Exact widening of an fp16/bf16/fp32 array (numpy or torch CPU tensor) to fp32."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float32).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


_I64 = ctypes.c_int64
_INT = ctypes.c_int
_DBL = ctypes.c_double


def minmax(x, ch_max=None, ch_min=None):
    """Per-channel (max, min) of x [T, C].  With ch_max/ch_min given, folds into them."""
    x = _f32(x)
    T, C = x.shape
    acc = ch_max is not None
    mx = np.array(ch_max, dtype=np.float32) if acc else np.empty(C, np.float32)
    mn = np.array(ch_min, dtype=np.float32) if acc else np.empty(C, np.float32)
    _load().orc_minmax(_p(x), _I64(T), _INT(C), _p(mx), _p(mn), _INT(int(acc)))
    return mx, mn


def layernorm(x, gamma, beta, eps=1e-5):
    """LayerNorm in fp64; returns (y64, y32) in the ORIGINAL channel order."""
    x = _f32(x)
    T, C = x.shape
    g, b = _f32(gamma), _f32(beta)
    y64 = np.empty((T, C), np.float64)
    y32 = np.empty((T, C), np.float32)
    _load().orc_layernorm(_p(x), _I64(T), _INT(C), _p(g), _p(b), _DBL(eps), _p(y64), _p(y32))
    return y64, y32


def minmax_ln(x, gamma, beta, eps=1e-5, ch_max=None, ch_min=None):
    """Per-channel (max, min) of the fp32-rounded LayerNorm output of x."""
    x = _f32(x)
    T, C = x.shape
    acc = ch_max is not None
    mx = np.array(ch_max, dtype=np.float32) if acc else np.empty(C, np.float32)
    mn = np.array(ch_min, dtype=np.float32) if acc else np.empty(C, np.float32)
    _load().orc_minmax_ln(_p(x), _I64(T), _INT(C), _p(_f32(gamma)), _p(_f32(beta)), _DBL(eps),
                          _p(mx), _p(mn), _INT(int(acc)))
    return mx, mn


def kmeans_init(ch_max, ch_min, g):
    mx, mn = _f32(ch_max), _f32(ch_min)
    cent = np.empty((g, 2), np.float64)
    rc = _load().orc_kmeans_init(_p(mx), _p(mn), _INT(mx.size), _INT(g), _p(cent))
    if rc != 0:
        raise ValueError("kmeans_init: need 1 <= g <= C")
    return cent


def kmeans_assign(ch_max, ch_min, cent, labels=None):
    mx, mn = _f32(ch_max), _f32(ch_min)
    cent = np.ascontiguousarray(cent, dtype=np.float64)
    lab = np.full(mx.size, -1, np.int32) if labels is None else _i32(labels).copy()
    changed = _load().orc_kmeans_assign(_p(mx), _p(mn), _INT(mx.size), _INT(cent.shape[0]),
                                        _p(cent), _p(lab))
    return lab, changed


def kmeans_update(ch_max, ch_min, labels, cent):
    mx, mn = _f32(ch_max), _f32(ch_min)
    out = np.array(cent, dtype=np.float64, copy=True)
    _load().orc_kmeans_update(_p(mx), _p(mn), _INT(mx.size), _INT(out.shape[0]), _p(_i32(labels)),
                              _p(out))
    return out


def kmeans(ch_max, ch_min, g, iters):
    """Deterministic Lloyd KMeans; returns (labels int32[C], centroids fp64[g, 2])."""
    mx, mn = _f32(ch_max), _f32(ch_min)
    C = mx.size
    labels = np.empty(C, np.int32)
    cent = np.empty((g, 2), np.float64)
    rc = _load().orc_kmeans(_p(mx), _p(mn), _INT(C), _INT(g), _INT(iters), _p(labels), _p(cent))
    if rc != 0:
        raise ValueError("kmeans: need 1 <= g <= C and iters >= 0")
    return labels, cent


def reorder(labels, g):
    """Stable counting sort by cluster: returns (R, col_cluster, offsets)."""
    lab = _i32(labels)
    C = lab.size
    R = np.empty(C, np.int32)
    cc = np.empty(C, np.int32)
    off = np.empty(g + 1, np.int32)
    _load().orc_reorder(_p(lab), _INT(C), _INT(g), _p(R), _p(cc), _p(off))
    return R, cc, off


def cluster_params(ch_max, ch_min, labels, g, bits):
    """Per-cluster fp32 scale and int32 zero point."""
    mx, mn = _f32(ch_max), _f32(ch_min)
    s = np.empty(g, np.float32)
    z = np.empty(g, np.int32)
    _load().orc_cluster_params(_p(mx), _p(mn), _p(_i32(labels)), _INT(mx.size), _INT(g),
                               _INT(bits), _p(s), _p(z))
    return s, z


def quantize(y, col_cluster, s, z, bits):
    """Unpacked codes (uint8) of y [rows, C], column j in cluster col_cluster[j]."""
    y = _f32(y)
    rows, C = y.shape
    q = np.empty((rows, C), np.uint8)
    _load().orc_quantize(_p(y), _I64(rows), _INT(C), _p(_i32(col_cluster)), _p(_f32(s)),
                         _p(_i32(z)), _INT(bits), _p(q))
    return q


def pack(q, bits):
    q = np.ascontiguousarray(q, dtype=np.uint8)
    rows, C = q.shape
    out = np.empty((rows, C * bits // 8), np.uint8)
    _load().orc_pack(_p(q), _I64(rows), _INT(C), _INT(bits), _p(out))
    return out


def unpack(packed, C, bits):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    rows = packed.shape[0]
    q = np.empty((rows, C), np.uint8)
    _load().orc_unpack(_p(packed), _I64(rows), _INT(C), _INT(bits), _p(q))
    return q


def dequant(q, col_cluster, s, z):
    """fp32 values s*(q - z) of unpacked codes q [rows, C]."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    rows, C = q.shape
    out = np.empty((rows, C), np.float32)
    _load().orc_dequant(_p(q), _I64(rows), _INT(C), _p(_i32(col_cluster)), _p(_f32(s)),
                        _p(_i32(z)), _p(out))
    return out


def ln_reorder_quant(x, gamma, beta, R, col_cluster, s, z, bits, eps=1e-5, want_codes=True,
                     want_ln=False):
    """Unfused definition: LN -> gather(R) -> quantize -> pack.

    Returns (packed or None, ln32 or None, ln64 or None); ln outputs are in stored order.
    """
    x = _f32(x)
    T, C = x.shape
    packed = np.empty((T, C * bits // 8), np.uint8) if want_codes else None
    ln32 = np.empty((T, C), np.float32) if want_ln else None
    ln64 = np.empty((T, C), np.float64) if want_ln else None
    _load().orc_ln_reorder_quant(_p(x), _I64(T), _INT(C), _p(_f32(gamma)), _p(_f32(beta)),
                                 _DBL(eps), _p(_i32(R)), _p(_i32(col_cluster)), _p(_f32(s)),
                                 _p(_i32(z)), _INT(bits), _p(packed), _p(ln32), _p(ln64))
    return packed, ln32, ln64


def kv_quant(kv, col_cluster, s, z, bits):
    """Packed codes of a [B, H, S, D] tensor, channel c = h*D + d, layout kept."""
    kv = _f32(kv)
    B, H, S, D = kv.shape
    out = np.empty((B, H, S, D * bits // 8), np.uint8)
    _load().orc_kv_quant(_p(kv), _I64(B), _INT(H), _I64(S), _INT(D), _p(_i32(col_cluster)),
                         _p(_f32(s)), _p(_i32(z)), _INT(bits), _p(out))
    return out


def kv_quant_cluster_ordered(kv, R, col_cluster, s, z, bits):
    """The K/V cache stored in cluster order ([RPTQ-art] text after Fig. 2: the channels of one
    cluster placed side by side, each cluster with its own s and z; results paragraph: the K/V
    cache quantized per cluster) -- the layout variant of the cache, beside kv_quant's kept
    [B, H, S, D] layout.  For every token (b, s) the C = H*D channels (channel c = h*D + d) are
    gathered through the reorder index (stored column j holds channel R[j]), quantized with the
    cluster of the stored column (col_cluster[j]) and packed as one row: codes [B, S, C*bits/8],
    the layout of the activation codes.  Definition written out: transpose to token rows, gather,
    then the oracle's quantize and pack."""
    kv = _f32(kv)
    B, H, S, D = kv.shape
    rows = np.ascontiguousarray(kv.transpose(0, 2, 1, 3).reshape(B * S, H * D))
    q = quantize(rows[:, np.asarray(R, dtype=np.int64)], col_cluster, s, z, bits)
    return pack(q, bits).reshape(B, S, H * D * bits // 8)


def kv_dequant(packed, D, col_cluster, s, z, bits):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    B, H, S, _ = packed.shape
    out = np.empty((B, H, S, D), np.float32)
    _load().orc_kv_dequant(_p(packed), _I64(B), _INT(H), _I64(S), _INT(D), _p(_i32(col_cluster)),
                           _p(_f32(s)), _p(_i32(z)), _INT(bits), _p(out))
    return out


def dynamic_params(x, gamma, beta, labels, g, bits, eps=1e-5):
    """Dynamic (per-batch) cluster ranges ([Basics] section 1.1: a static range is fixed from
    calibration data, a dynamic one is taken from the data being quantized; [RPTQ-art] text after
    Fig. 2: one (s, z) per cluster of channels).  The clusters (labels) stay those of the offline
    calibration; the per-channel max / min are those of LayerNorm(x) over this batch, and every
    cluster's (s, z) follow from them exactly as in the calibration.  Definition written out: the
    oracle's minmax_ln, then its cluster_params."""
    mx, mn = minmax_ln(x, gamma, beta, eps)
    return cluster_params(mx, mn, labels, g, bits)


def quant_weights(W, bits=4):
    """Per-output-channel asymmetric weight quantization ([Basics] section 1.4, per-channel
    granularity; section 1.3, s = range / (2^b - 1), z = rint(-min / s)): row n of W [N, C] gets
    its own (s_w, z_w) from its min and max, codes q = clamp(rint(w / s_w) + z_w, 0, qmax).
    fp32 operations as in the activation quantizer.  Returns (q uint8 [N, C], s_w fp32 [N],
    z_w int32 [N])."""
    W = np.asarray(W, np.float32)
    N, C = W.shape
    q = np.empty((N, C), np.uint8)
    sw = np.empty(N, np.float32)
    zw = np.empty(N, np.int32)
    for n in range(N):
        # one cluster spanning the whole row: its range is the row's min and max
        s1, z1 = cluster_params(np.array([W[n].max()], np.float32), np.array([W[n].min()], np.float32),
                                np.zeros(1, np.int32), 1, bits)
        sw[n], zw[n] = s1[0], z1[0]
        q[n] = quantize(W[n:n + 1], np.zeros(C, np.int32), s1, z1, bits)[0]
    return q, sw, zw


def reordered_linear(codes, C, col_cluster, s, z, bits, R, qw, sw, zw):
    """The linear layer after the reorder-fused LayerNorm ([RPTQ-art], Fig. 3 caption and the text
    after it: the next layer's weights are permuted offline by the same reorder index, so the
    layer consumes the activations in cluster order and its output is unchanged).  codes
    [T, C*bits/8] are the packed cluster-ordered activation codes (column j in cluster
    col_cluster[j]); qw [N, C] the 4-bit weight codes in the ORIGINAL channel order with
    per-row (sw, zw).  Y[t, n] = sum_j s_k (q[t, j] - z_k) * sw[n] (qw[n, R[j]] - zw[n]),
    k = col_cluster[j], in fp64.  Returns fp64 [T, N]."""
    q = unpack(np.asarray(codes, np.uint8).reshape(-1, C * bits // 8), C, bits).astype(np.float64)
    cc = np.asarray(col_cluster)
    xa = (q - np.asarray(z, np.float64)[cc]) * np.asarray(s, np.float64)[cc]          # [T, C], cluster order
    wd = (np.asarray(qw, np.float64) - np.asarray(zw, np.float64)[:, None]) * np.asarray(sw, np.float64)[:, None]
    wr = wd[:, np.asarray(R)]                                                          # [N, C], permuted offline
    return xa @ wr.T


def linear_fp16_operand(qw, sw, zw, R, col_cluster, s, z):
    """The fp16 weight operand with which the library computes reordered_linear (a design reading,
    not a step of the pages: [RPTQ-art] Fig. 3 text permutes the weights offline; folding the
    per-cluster activation scale into them leaves only the integer codes q on the activation
    side).  For output row n and cluster-order column j (k = col_cluster[j]):
        b[n][j]  = RN32(s_k * (qw[n][R[j]] - zw[n]))            one fp32 product
        lam[n]   = 2^(e - 14) with max_j |b[n][j]| in [2^e, 2^(e+1))  (1 for an all-zero row)
        B[n][j]  = RN16(b[n][j] / lam[n])                        the division is exact
        bz[n]    = sum_j z_k B[n][j]                             fp64, rounded to fp32 once
    so that reordered_linear = sw[n] lam[n] (q @ B^T - bz) up to the fp16 rounding of B.
    Returns (B fp16 [N, C] in cluster order, bz fp32 [N], lam fp32 [N])."""
    qw = np.asarray(qw)
    N, C = qw.shape
    cc = np.asarray(col_cluster)
    s32 = _f32(s)
    B = np.empty((N, C), np.float16)
    bz = np.empty(N, np.float32)
    lam = np.empty(N, np.float32)
    for n in range(N):
        d = (qw[n, np.asarray(R)].astype(np.int64) - int(zw[n])).astype(np.float32)
        b = (s32[cc] * d).astype(np.float32)                      # numpy fp32 multiply: RN
        m = float(np.abs(b).max())
        if m > 0.0:
            e = int(np.floor(np.log2(m)))
            if 2.0 ** e > m:                                       # guard log2's rounding
                e -= 1
            elif 2.0 ** (e + 1) <= m:
                e += 1
            lam[n] = np.float32(2.0 ** (e - 14))
        else:
            lam[n] = np.float32(1.0)
        B[n] = (b.astype(np.float64) / float(lam[n])).astype(np.float16)   # RN to fp16
        bz[n] = np.float32(np.sum(np.asarray(z, np.float64)[cc] * B[n].astype(np.float64)))
    return B, bz, lam


def kv_append(cache, new, s_begin, col_cluster, s, z, bits):
    """Decode-time append ([RPTQ-art] results paragraph: the K/V cache is quantized per cluster;
    closing paragraph: the cache dominates memory at large batch x sequence).  A copy of the
    packed cache [B, H, S_max, D*bits/8] whose positions s_begin .. s_begin + s_len - 1 hold the
    codes of the new tokens [B, H, s_len, D] (quantized exactly as kv_quant does); every other
    position is unchanged.  Definition written out: quantize the new rows, store them in place."""
    out = np.array(cache, dtype=np.uint8, copy=True)
    n = np.asarray(new).shape[2]
    assert 0 <= s_begin and s_begin + n <= out.shape[2]
    out[:, :, s_begin:s_begin + n] = kv_quant(new, col_cluster, s, z, bits)
    return out


def kv_decode_attention(q, k_codes, v_codes, L, D, clk, sk, zk, clv, sv, zv, bits, scale=None):
    """One decode step of attention reading the packed caches (the consumer of the K/V codes;
    [RPTQ-art] results paragraph and closing memory paragraph).  For every (b, h):
    K, V = the fp32 dequantized rows 0 .. L-1 (exactly kv_dequant), scores = (q . K_s) * scale
    (scale = 1/sqrt(D) by default), p = softmax over the L positions, out = sum_s p_s V_s; the
    products, sums and the softmax in fp64.  q [B, H, D]; returns fp64 [B, H, D] and the fp64
    scores [B, H, L] (for error bounds)."""
    q = np.asarray(_f32(q), dtype=np.float64)
    K = kv_dequant(np.ascontiguousarray(k_codes[:, :, :L]), D, clk, sk, zk, bits).astype(np.float64)
    V = kv_dequant(np.ascontiguousarray(v_codes[:, :, :L]), D, clv, sv, zv, bits).astype(np.float64)
    sc = (1.0 / np.sqrt(D)) if scale is None else float(scale)
    scores = np.einsum("bhd,bhsd->bhs", q, K) * sc
    m = scores.max(axis=2, keepdims=True)
    e = np.exp(scores - m)
    p = e / e.sum(axis=2, keepdims=True)
    return np.einsum("bhs,bhsd->bhd", p, V), scores


def calibrate(ch_max, ch_min, g, iters, bits):
    """The whole offline chain on given statistics: KMeans -> reorder -> cluster params."""
    labels, cent = kmeans(ch_max, ch_min, g, iters)
    R, cc, off = reorder(labels, g)
    s, z = cluster_params(ch_max, ch_min, labels, g, bits)
    return dict(labels=labels, centroids=cent, R=R, col_cluster=cc, offsets=off, scale=s, zero=z)
