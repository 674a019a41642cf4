"""GPU parity of the decode-time K/V path: the append of one step's tokens into preallocated
packed caches, and decode attention reading those caches (codes dequantized in registers).

Append: byte-exact against oracle.kv_append (the untouched positions of a cache pre-filled with
random bytes must survive), and token-by-token appends reproduce the whole-cache quantization.
Attention: against oracle.kv_decode_attention (fp64 on the same dequantized values), with a
bar derived from the kernel's fp32 arithmetic.  A lane owns CPL = min(32, D) channels; a row's
score is two interleaved sums of CPL/2 fused multiply-adds of (q_d s_d scale) (q - z), one add,
and a log2(D/CPL)-level shuffle tree, and q_d s_d scale and s (q - z) differ from the oracle's
products by a rounding each, so |d score| <= (CPL/2 + 4 + log2(D/CPL)) u scale sum|q K|
(u = 2^-24); a weight moves by at most p (2 max|d score| + the relative error of its exp and
of the sums); the output is a fixed-order sum of ceil(L / (8 * rows per warp step)) products
per lane, a shuffle tree, 8 warp partials and two final products.  Everything is bounded by a
multiple of sum_s p_s |V_s,d|."""
import math

import numpy as np
import pytest
import torch

import oracle
from post_activation_quantization_b200 import rptq, synthetic
from tests.gpu_common import DEV, to_np

pytestmark = pytest.mark.gpu
U = 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_activation_quantization_b200 import build
    build.build()
    rptq.lib()
    yield
    assert rptq.rptq_device_error() == 0


def _cal(kv_f32, H, D, g, bits):
    flat = np.ascontiguousarray(kv_f32.transpose(0, 2, 1, 3).reshape(-1, H * D))
    mx, mn = oracle.minmax(flat)
    return oracle.calibrate(mx, mn, g, 5, bits)


def _dev(cal):
    return [torch.from_numpy(np.ascontiguousarray(cal[k])).to(DEV) for k in ("labels", "scale", "zero")]


@pytest.mark.parametrize("dtype,B,H,D,s_len,S_max,s_begin,bits", [
    ("bf16", 8, 96, 128, 1, 64, 63, 3), ("bf16", 2, 5, 128, 3, 40, 17, 4), ("f16", 3, 4, 64, 17, 33, 0, 3),
    ("f32", 2, 3, 8, 5, 9, 4, 4), ("f16", 1, 7, 256, 1, 2, 1, 3), ("bf16", 4, 2, 2048, 2, 5, 2, 3)])
def test_kv_append_matches_oracle(dtype, B, H, D, s_len, S_max, s_begin, bits):
    seed = B * 131 + H * 7 + D
    mk = synthetic.channel_model(H * D, seed, tag=1)
    mv = synthetic.channel_model(H * D, seed, tag=2)
    calib_k = synthetic.kv_cache(B, H, 16, D, mk, seed, "k", dtype)
    calib_v = synthetic.kv_cache(B, H, 16, D, mv, seed, "v", dtype)
    g = 8
    ck, cv = _cal(oracle._f32(calib_k), H, D, g, bits), _cal(oracle._f32(calib_v), H, D, g, bits)
    knew = synthetic.kv_cache(B, H, s_len, D, mk, seed + 1, "k", dtype)
    vnew = synthetic.kv_cache(B, H, s_len, D, mv, seed + 1, "v", dtype)
    rng = np.random.default_rng(seed)
    shape = (B, H, S_max, D * bits // 8)
    k0 = rng.integers(0, 256, shape, dtype=np.uint8)
    v0 = rng.integers(0, 256, shape, dtype=np.uint8)
    kc, vc = torch.from_numpy(k0).to(DEV), torch.from_numpy(v0).to(DEV)
    rptq.rptq_kv_append(knew.to(DEV), vnew.to(DEV), *_dev(ck), *_dev(cv), bits, k_cache=kc, v_cache=vc,
                        s_begin=s_begin)
    kref = oracle.kv_append(k0, oracle._f32(knew), s_begin, ck["labels"], ck["scale"], ck["zero"], bits)
    vref = oracle.kv_append(v0, oracle._f32(vnew), s_begin, cv["labels"], cv["scale"], cv["zero"], bits)
    assert np.array_equal(to_np(kc), kref) and np.array_equal(to_np(vc), vref)


def test_token_by_token_appends_equal_the_whole_cache_quantization():
    B, H, S, D, bits, g = 2, 6, 24, 128, 3, 8
    mk = synthetic.channel_model(H * D, 3, tag=1)
    k = synthetic.kv_cache(B, H, S, D, mk, 3, "k", "bf16")
    cal = _cal(oracle._f32(k), H, D, g, bits)
    lab, sc, zp = _dev(cal)
    kd = k.to(DEV)
    whole, _ = rptq.rptq_kv_quant(kd, None, lab, sc, zp, None, None, None, bits)
    cache = torch.zeros((B, H, S, D * bits // 8), dtype=torch.uint8, device=DEV)
    for t in range(S):
        rptq.rptq_kv_append(kd[:, :, t:t + 1].contiguous(), None, lab, sc, zp, None, None, None, bits,
                            k_cache=cache, s_begin=t)
    assert torch.equal(cache, whole)


def test_kv_append_rejects_positions_past_the_end():
    B, H, D = 1, 2, 64
    x = torch.zeros((B, H, 2, D), dtype=torch.bfloat16, device=DEV)
    cache = torch.zeros((B, H, 4, D * 3 // 8), dtype=torch.uint8, device=DEV)
    t = torch.zeros(H * D, dtype=torch.int32, device=DEV)
    s = torch.ones(1, device=DEV)
    z = torch.zeros(1, dtype=torch.int32, device=DEV)
    with pytest.raises(rptq.RptqError):
        rptq.rptq_kv_append(x, None, t, s, z, None, None, None, 3, k_cache=cache, s_begin=3)


def _attn_bound(q, Kd, Vd, L, D, scale):
    """Per-output bound on |gpu - fp64| for the kernel's fp32 evaluation order (module docstring)."""
    q64, K, V = q.astype(np.float64), Kd[:, :, :L].astype(np.float64), Vd[:, :, :L].astype(np.float64)
    cpl = min(32, D)
    lpp = D // cpl
    ppw = 32 // lpp
    dscore = (cpl / 2 + 4 + math.log2(lpp)) * U * scale * np.einsum("bhd,bhsd->bhs", np.abs(q64), np.abs(K))
    sc = np.einsum("bhd,bhsd->bhs", q64, K) * scale
    p = np.exp(sc - sc.max(axis=2, keepdims=True))
    p /= p.sum(axis=2, keepdims=True)
    n_sum = math.ceil(L / 256) + 5 + 8
    n_out = math.ceil(L / (8 * ppw)) + math.log2(ppw) + 8 + 1 + 3
    rel = 2 * dscore.max(axis=2) + (n_sum + n_out + 8) * U
    mag = np.einsum("bhs,bhsd->bhd", p, np.abs(V))
    return 2 * rel[..., None] * mag + 1e-30


@pytest.mark.parametrize("B,H,D,S_max,L,bits,scale", [
    (2, 4, 128, 300, 300, 3, 0.0), (2, 4, 128, 300, 37, 4, 0.0), (1, 3, 64, 50, 1, 3, 0.0),
    (3, 2, 8, 20, 19, 4, 0.5), (1, 2, 256, 130, 129, 3, 0.0), (8, 96, 128, 512, 512, 3, 0.0),
    (2, 3, 16, 40, 33, 3, 0.0), (2, 3, 16, 40, 40, 4, 0.0), (1, 2, 32, 70, 70, 3, 0.0), (2, 2, 8, 12, 9, 3, 0.0)])
def test_kv_decode_attention_matches_oracle(B, H, D, S_max, L, bits, scale):
    seed = 7 * B + H + D + L
    mk = synthetic.channel_model(H * D, seed, tag=1)
    mv = synthetic.channel_model(H * D, seed, tag=2)
    k = oracle._f32(synthetic.kv_cache(B, H, S_max, D, mk, seed, "k", "bf16"))
    v = oracle._f32(synthetic.kv_cache(B, H, S_max, D, mv, seed, "v", "bf16"))
    g = 16
    ck, cv = _cal(k, H, D, g, bits), _cal(v, H, D, g, bits)
    kc = oracle.kv_quant(k, ck["labels"], ck["scale"], ck["zero"], bits)
    vc = oracle.kv_quant(v, cv["labels"], cv["scale"], cv["zero"], bits)
    q = (np.random.default_rng(seed).standard_normal((B, H, D)) * 0.05).astype(np.float32)
    out = rptq.rptq_kv_decode_attention(torch.from_numpy(q).to(DEV), torch.from_numpy(kc).to(DEV),
                                        torch.from_numpy(vc).to(DEV), L, *_dev(ck), *_dev(cv), bits, scale=scale)
    ref, _ = oracle.kv_decode_attention(q, kc, vc, L, D, ck["labels"], ck["scale"], ck["zero"], cv["labels"],
                                        cv["scale"], cv["zero"], bits, scale=scale or None)
    sc = scale or 1.0 / math.sqrt(D)
    Kd = oracle.kv_dequant(kc, D, ck["labels"], ck["scale"], ck["zero"], bits)
    Vd = oracle.kv_dequant(vc, D, cv["labels"], cv["scale"], cv["zero"], bits)
    tol = _attn_bound(q, Kd, Vd, L, D, sc)
    err = np.abs(to_np(out).astype(np.float64) - ref)
    assert (err <= tol).all(), f"worst excess {(err - tol).max():.3e}, worst error {err.max():.3e}"


def test_kv_decode_attention_rejects_bad_shapes():
    q = torch.zeros((1, 2, 96), device=DEV)
    c = torch.zeros((1, 2, 4, 96 * 3 // 8), dtype=torch.uint8, device=DEV)
    t = torch.zeros(2 * 96, dtype=torch.int32, device=DEV)
    s = torch.ones(1, device=DEV)
    z = torch.zeros(1, dtype=torch.int32, device=DEV)
    with pytest.raises(rptq.RptqError):  # D not a power of two
        rptq.rptq_kv_decode_attention(q, c, c, 2, t, s, z, t, s, z, 3)
    q = torch.zeros((1, 2, 64), device=DEV)
    c = torch.zeros((1, 2, 4, 24), dtype=torch.uint8, device=DEV)
    t = torch.zeros(128, dtype=torch.int32, device=DEV)
    with pytest.raises(rptq.RptqError):  # L beyond the cache
        rptq.rptq_kv_decode_attention(q, c, c, 5, t, s, z, t, s, z, 3)
