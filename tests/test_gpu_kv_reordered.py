"""GPU parity of the K/V cache in cluster order (rptq_kv_quant_cluster_ordered).

Three comparisons per case:
  1. against oracle.kv_quant_cluster_ordered (the definition: token rows gathered through R,
     quantized per stored column's cluster, packed), with the codes bar of the other quantizers;
  2. bit for bit against rptq_kv_quant's codes of the kept [B, H, S, D] layout moved to token rows
     and gathered through R on the host (the two kernels share the quotient, rounding and clamp);
  3. the cluster-ordered rows read back by rptq_dequant's rows layout with col_cluster, bit for bit
     against oracle.dequant of the oracle's codes.
Token counts that are not a multiple of the kernel's quad of 4, fp32 / fp16 / bf16 caches, A3 and
A4, the OPT-175B cache width (96 heads x 128), refusals and a damaged reorder index are covered."""
import numpy as np
import pytest
import torch

import oracle
from post_activation_quantization_b200 import rptq, synthetic
from tests.gpu_common import DEV, compare_codes, to_np

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


def _case(B, H, S, D, dtype, g, bits, seed):
    m = synthetic.channel_model(H * D, seed, tag=1)
    kv = synthetic.kv_cache(B, H, S, D, m, seed, "k", dtype)
    kv32 = oracle._f32(kv)
    flat = np.ascontiguousarray(kv32.transpose(0, 2, 1, 3).reshape(-1, H * D))
    mx, mn = oracle.minmax(flat)
    cal = oracle.calibrate(mx, mn, g, 5, bits)
    dev = {k: torch.from_numpy(np.ascontiguousarray(cal[k])).to(DEV) for k in ("R", "col_cluster", "labels", "scale", "zero")}
    return kv, kv32, cal, dev


@pytest.mark.parametrize("B,H,S,D,dtype,g,bits", [
    (2, 4, 37, 64, "bf16", 8, 3),     # S not a multiple of 4
    (1, 8, 16, 128, "f16", 16, 4),
    (3, 2, 5, 32, "f32", 4, 3),       # C = 64
    (2, 96, 64, 128, "bf16", 64, 3),  # the OPT-175B cache width
    (1, 3, 2, 256, "bf16", 12, 4),    # fewer tokens than one quad
    (2, 5, 19, 96, "f16", 10, 3),     # D = 96 (not a power of two), C = 480
    (1, 128, 9, 128, "bf16", 512, 4), # the largest width (16384 channels) and cluster count
    (1, 64, 6, 256, "f32", 100, 3),   # 16384 channels of fp32
])
def test_cluster_ordered_cache_matches_oracle_and_kept_layout(B, H, S, D, dtype, g, bits):
    C = H * D
    kv, kv32, cal, p = _case(B, H, S, D, dtype, g, bits, 17 * B + H + S + D)
    kvd = kv.to(DEV)
    got = rptq.rptq_kv_quant_cluster_ordered(kvd, p["R"], p["col_cluster"], p["scale"], p["zero"], bits)
    torch.cuda.synchronize()
    assert got.shape == (B, S, C * bits // 8)
    g_np = to_np(got)
    # 1. the definition
    ref = oracle.kv_quant_cluster_ordered(kv32, cal["R"], cal["col_cluster"], cal["scale"], cal["zero"], bits)
    compare_codes(g_np.reshape(B * S, -1), ref.reshape(B * S, -1), C, bits, f"kv cluster order {dtype} B={B} H={H} S={S} D={D}")
    # 2. the kept layout's codes, moved and gathered on the host
    kept, _ = rptq.rptq_kv_quant(kvd, None, p["labels"], p["scale"], p["zero"], None, None, None, bits)
    qk = oracle.unpack(to_np(kept).reshape(-1, D * bits // 8), D, bits).reshape(B, H, S, D)
    q_tok = qk.transpose(0, 2, 1, 3).reshape(B * S, C)[:, cal["R"]]
    assert np.array_equal(oracle.unpack(g_np.reshape(B * S, -1), C, bits), q_tok)
    # 3. read back through the rows layout of rptq_dequant
    deq = rptq.rptq_dequant(torch.from_numpy(ref.reshape(B * S, -1)).to(DEV), p["col_cluster"], p["scale"], p["zero"],
                            bits, C=C)
    want = oracle.dequant(oracle.unpack(ref.reshape(B * S, -1), C, bits), cal["col_cluster"], cal["scale"], cal["zero"])
    assert np.array_equal(to_np(deq), want)


def test_huge_zero_point_takes_the_ieee_division():
    """A zero point beyond 2^21 leaves the fast quotient's range: every element then takes the IEEE
    division and the definition directly; the codes still equal the oracle's exactly."""
    B, H, S, D, g, bits = 2, 4, 9, 32, 6, 4
    kv, kv32, cal, p = _case(B, H, S, D, "bf16", g, bits, 23)
    z = cal["zero"].copy()
    z[1] = (1 << 22) + 5  # every channel of cluster 1 clamps to 15 (or 0 for very negative x)
    ref = oracle.kv_quant_cluster_ordered(kv32, cal["R"], cal["col_cluster"], cal["scale"], z, bits)
    got = rptq.rptq_kv_quant_cluster_ordered(kv.to(DEV), p["R"], p["col_cluster"], p["scale"],
                                             torch.from_numpy(z).to(DEV), bits)
    assert np.array_equal(to_np(got), ref)


def test_refusals_and_empty():
    kv, kv32, cal, p = _case(1, 2, 8, 16, "bf16", 4, 3, 5)  # C = 32
    args = (p["R"], p["col_cluster"], p["scale"], p["zero"])
    e = rptq.rptq_kv_quant_cluster_ordered(kv[:, :, :0].contiguous().to(DEV), *args, 3)
    assert e.shape == (1, 0, 12)
    bad = torch.zeros((1, 3, 4, 8), dtype=torch.bfloat16, device=DEV)  # C = 24: not a multiple of 32
    with pytest.raises(rptq.RptqError) as err:
        rptq.rptq_kv_quant_cluster_ordered(bad, *args, 3)
    assert err.value.status == -2
    with pytest.raises(rptq.RptqError) as err:
        rptq.rptq_kv_quant_cluster_ordered(kv.to(DEV), *args, 5)
    assert err.value.status == -2


def test_damaged_reorder_index_sets_the_error_word():
    kv, kv32, cal, p = _case(2, 2, 9, 32, "bf16", 4, 4, 6)
    R = p["R"].clone()
    R[3] = 9999
    rptq.rptq_kv_quant_cluster_ordered(kv.to(DEV), R, p["col_cluster"], p["scale"], p["zero"], 4)
    assert rptq.rptq_device_error() & rptq.RPTQ_DEVERR_REORDER
    assert rptq.rptq_device_error() == 0  # the read clears the word
