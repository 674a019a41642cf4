"""Pins of the oracle's decode-time K/V functions, against what the definitions fix:
  * appending one token at a time into an empty cache gives, byte for byte, the whole-cache
    quantization of the same tokens (kv_quant), and untouched positions keep their bytes;
  * decode attention: with one position the output is that position's dequantized V row; with
    identical K rows the weights are uniform and the output is the mean of the V rows; a
    brute-force pure-Python loop (explicit max, exp, normalisation) on a tiny case agrees to
    fp64 rounding."""
import math

import numpy as np

import oracle
from post_activation_quantization_b200 import synthetic


def _kv_case(B, H, S, D, seed, bits, g=4):
    m = synthetic.channel_model(H * D, seed, tag=1)
    k = oracle._f32(synthetic.kv_cache(B, H, S, D, m, seed, "k", "f32"))
    flat = np.ascontiguousarray(k.transpose(0, 2, 1, 3).reshape(-1, H * D))
    mx, mn = oracle.minmax(flat)
    cal = oracle.calibrate(mx, mn, g, 5, bits)
    return k, cal


def test_append_one_token_at_a_time_equals_whole_cache():
    B, H, S, D, bits = 2, 3, 9, 16, 3
    k, cal = _kv_case(B, H, S, D, 5, bits)
    whole = oracle.kv_quant(k, cal["labels"], cal["scale"], cal["zero"], bits)
    cache = np.zeros((B, H, S + 3, D * bits // 8), np.uint8)
    for t in range(S):
        cache = oracle.kv_append(cache, k[:, :, t:t + 1], t, cal["labels"], cal["scale"], cal["zero"], bits)
    assert np.array_equal(cache[:, :, :S], whole)
    assert not cache[:, :, S:].any()  # never written
    # a block append in the middle leaves the other positions as they were
    c2 = oracle.kv_append(cache, k[:, :, 2:5], 6, cal["labels"], cal["scale"], cal["zero"], bits)
    assert np.array_equal(c2[:, :, 6:9], whole[:, :, 2:5])
    assert np.array_equal(c2[:, :, :6], cache[:, :, :6]) and np.array_equal(c2[:, :, 9:], cache[:, :, 9:])


def test_decode_attention_special_cases():
    B, H, S, D, bits = 1, 2, 6, 8, 4
    k, cal = _kv_case(B, H, S, D, 7, bits)
    kc = oracle.kv_quant(k, cal["labels"], cal["scale"], cal["zero"], bits)
    vc = oracle.kv_quant(k[:, :, ::-1].copy(), cal["labels"], cal["scale"], cal["zero"], bits)
    args = (cal["labels"], cal["scale"], cal["zero"]) * 2
    q = np.random.default_rng(0).standard_normal((B, H, D)).astype(np.float32)
    # one position: the output is that V row
    out, _ = oracle.kv_decode_attention(q, kc, vc, 1, D, *args, bits)
    V = oracle.kv_dequant(vc, D, cal["labels"], cal["scale"], cal["zero"], bits)
    assert np.allclose(out, V[:, :, 0], rtol=0, atol=1e-12)
    # identical K rows: uniform weights, the mean of the V rows
    kc_same = np.repeat(kc[:, :, :1], S, axis=2)
    out, _ = oracle.kv_decode_attention(q, kc_same, vc, S, D, *args, bits)
    assert np.allclose(out, V.astype(np.float64).mean(axis=2), rtol=1e-12, atol=1e-12)


def test_decode_attention_brute_force():
    B, H, S, D, bits = 1, 2, 5, 8, 3
    k, cal = _kv_case(B, H, S, D, 9, bits)
    kc = oracle.kv_quant(k, cal["labels"], cal["scale"], cal["zero"], bits)
    vc = oracle.kv_quant(k * np.float32(0.5), cal["labels"], cal["scale"], cal["zero"], bits)
    q = np.random.default_rng(1).standard_normal((B, H, D)).astype(np.float32)
    L = 4
    out, _ = oracle.kv_decode_attention(q, kc, vc, L, D, cal["labels"], cal["scale"], cal["zero"],
                                        cal["labels"], cal["scale"], cal["zero"], bits)
    Kd = oracle.kv_dequant(kc, D, cal["labels"], cal["scale"], cal["zero"], bits)
    Vd = oracle.kv_dequant(vc, D, cal["labels"], cal["scale"], cal["zero"], bits)
    for h in range(H):
        sc = [sum(float(q[0, h, d]) * float(Kd[0, h, s, d]) for d in range(D)) / math.sqrt(D) for s in range(L)]
        mx = max(sc)
        w = [math.exp(v - mx) for v in sc]
        tot = sum(w)
        for d in range(D):
            ref = sum(w[s] / tot * float(Vd[0, h, s, d]) for s in range(L))
            assert abs(out[0, h, d] - ref) <= 1e-12 * (1 + abs(ref))
