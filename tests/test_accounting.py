"""Pins for the byte accounting that the benchmark's GB/s figures rest on, against the memory
claims of the pages: RPTQ article, memory paragraph at the end (OPT-66b, batch 64, sequence
8192: W4A4 saves over 900 GB against W4A16, the K/V cache dominating) and the Houmo article's
RPTQ section (up to 80 % less memory with 3-bit activations)."""
from post_activation_quantization_b200 import workloads as W


def test_kv_cache_saving_opt66b():
    # hidden 9216 is the OPT-66B width used by the opt66b-9216 workload; 64 layers is OPT-66B's
    # depth (model fact, not on the pages)
    fp16 = W.kv_cache_bytes(64, 64, 8192, 9216, 16)
    int4 = W.kv_cache_bytes(64, 64, 8192, 9216, 4)
    assert fp16 == 2 * 64 * 64 * 8192 * 9216 * 2
    assert (fp16 - int4) / 1e9 > 900
    assert 1 - W.kv_cache_bytes(1, 1, 1, 8, 3) / W.kv_cache_bytes(1, 1, 1, 8, 16) >= 0.80


def test_kernel_bytes_by_hand():
    assert W.bytes_ln_quant(32768, 12288, "bf16", 3) == 32768 * (24576 + 4608)
    assert W.bytes_ln_quant(512, 768, "f32", 4) == 512 * (3072 + 384)
    assert W.bytes_kv_quant(8 * 96 * 2048 * 128, "bf16", 3) == 8 * 2048 * 2 * (24576 + 4608)
    assert W.bytes_calib(262144, 9216, "bf16") == 262144 * 18432
    assert W.bytes_dequant(16, "bf16", 3) == 6 + 32
