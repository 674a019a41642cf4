"""Pins for the oracle's packing: hand-computed bytes and exhaustive round trips."""
import os

import numpy as np
import pytest

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _cases():
    out = []
    with open(os.path.join(GOLD, "pack_bytes.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            bits, codes, hexs = (p.strip() for p in line.split(";"))
            out.append((int(bits), [int(c) for c in codes.split(",")],
                        bytes(int(h, 16) for h in hexs.split())))
    return out


@pytest.mark.parametrize("bits,codes,expect", _cases())
def test_pack_hand_bytes(orc, bits, codes, expect):
    q = np.array([codes], np.uint8)
    assert orc.pack(q, bits).tobytes() == expect
    assert orc.unpack(np.frombuffer(expect, np.uint8)[None, :], len(codes), bits)[0].tolist() == codes


@pytest.mark.parametrize("bits", [3, 4])
def test_round_trip_every_value_every_position(orc, bits):
    qmax = 2 ** bits - 1
    C = 64
    rows = []
    for v in range(qmax + 1):
        for pos in range(C):
            r = np.zeros(C, np.uint8)
            r[pos] = v
            rows.append(r)
    q = np.stack(rows)
    rng = np.random.default_rng(0)
    q = np.concatenate([q, rng.integers(0, qmax + 1, (50, C), dtype=np.uint8)])
    p = orc.pack(q, bits)
    assert p.shape == (q.shape[0], C * bits // 8)
    assert np.array_equal(orc.unpack(p, C, bits), q)
