"""RPTQ data path on B200: calibration min/max, KMeans reorder, reorder-fused LayerNorm with
per-cluster 3/4-bit quantization, K/V-cache quantization and dequantization.

The compute lives in ``librptq.so`` (hand-written sm_100a CUDA kernels behind a C ABI declared
in ``include/rptq.h``); :mod:`.rptq` is a thin ctypes binding with the same entry-point names.
Importing this package does not load the library; the first call into :mod:`.rptq` does, and
raises if it is missing (there is no CPU fallback).
"""
__all__ = ["rptq", "synthetic", "workloads"]
