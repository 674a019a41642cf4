"""Pins of oracle.kv_quant_cluster_ordered (the K/V cache stored in cluster order).

1. Against kv_quant (the kept [B, H, S, D] layout, pinned on its own): the same per-channel codes,
   moved to token rows and gathered through R.  A transposed token/head order, a gather through
   R^-1 instead of R, or a cluster taken from the channel instead of the stored column all fail it.
2. Brute force from the definition on a tiny cache: clamp(rint(x / s) + z, 0, qmax) in IEEE fp32
   written out per element with numpy, packed by hand (3-bit: code j at bits [3j, 3j + 3) of the
   little-endian row; 4-bit: low nibble first).
"""
import numpy as np
import pytest

import oracle


def _setup(B, H, S, D, g, bits, seed):
    rng = np.random.default_rng(seed)
    C = H * D
    kv = (rng.standard_normal((B, H, S, D)) * rng.uniform(0.5, 4.0, (1, H, 1, D))).astype(np.float32)
    labels = rng.integers(0, g, C).astype(np.int32)
    R, col_cluster, _ = oracle.reorder(labels, g)
    s = rng.uniform(0.05, 0.6, g).astype(np.float32)
    z = rng.integers(0, 2 ** bits, g).astype(np.int32)
    return kv, labels, R, col_cluster, s, z


@pytest.mark.parametrize("B,H,S,D,g,bits", [(2, 3, 5, 8, 4, 3), (1, 4, 7, 16, 6, 4), (3, 2, 4, 32, 5, 3)])
def test_equals_kept_layout_codes_gathered(B, H, S, D, g, bits):
    kv, labels, R, cc, s, z = _setup(B, H, S, D, g, bits, 7 * B + H + S + D)
    C = H * D
    got = oracle.kv_quant_cluster_ordered(kv, R, cc, s, z, bits)
    assert got.shape == (B, S, C * bits // 8)
    kept = oracle.kv_quant(kv, labels, s, z, bits)                         # [B, H, S, D*bits/8]
    q_kept = oracle.unpack(kept.reshape(-1, D * bits // 8), D, bits).reshape(B, H, S, D)
    q_tok = q_kept.transpose(0, 2, 1, 3).reshape(B * S, C)                  # token rows, channel h*D + d
    q_got = oracle.unpack(got.reshape(B * S, -1), C, bits)
    assert np.array_equal(q_got, q_tok[:, R])


def test_brute_force_tiny():
    B, H, S, D, g, bits = 1, 2, 3, 8, 3, 3
    kv, labels, R, cc, s, z = _setup(B, H, S, D, g, bits, 11)
    C, qmax = H * D, 2 ** bits - 1
    got = oracle.kv_quant_cluster_ordered(kv, R, cc, s, z, bits)
    for t in range(S):
        codes = []
        for j in range(C):
            c = int(R[j])
            h, d = divmod(c, D)
            k = int(cc[j])
            q = np.rint(np.float32(kv[0, h, t, d]) / np.float32(s[k])) + z[k]   # IEEE fp32 divide, half to even
            codes.append(int(min(max(q, 0), qmax)))
        bitsum = 0
        for j, q in enumerate(codes):
            bitsum |= q << (3 * j)
        expect = np.array([(bitsum >> (8 * i)) & 0xFF for i in range(C * 3 // 8)], np.uint8)
        assert np.array_equal(got[0, t], expect), f"token {t}"
