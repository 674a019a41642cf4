"""Seeded synthetic inputs shared by the CUDA path's tests/bench and by the oracle's tests.

This module holds none of the RPTQ arithmetic: it only draws random numbers.  The
distribution follows the workload descriptions used for this library's parity cases and
benchmarks: per channel c a centre ~ N(0, 2) (standard deviation 2), a half-width
~ LogNormal(0, 1) (parameters of the underlying normal), and x[t, c] ~ U(centre - hw,
centre + hw) independently over tokens.  floor(p * C) "outlier" channels, picked by a seeded
permutation, have both centre and half-width multiplied by a factor (x100 or x200).  The
channel draw is the "model": the calibration batch and the runtime batch of one model share
it and differ only in their element draws.  LayerNorm gamma ~ U(0.5, 1.5) and
beta ~ N(0, 0.1) (standard deviation 0.1).  Linear-layer weights (no trained weights exist
here) are W[n, c] ~ N(0, 1/C), the usual fan-in scaling.

Every stream has its own derived seed, so any tensor can be regenerated alone.  Generation
runs on the requested device with torch's generator for that device; CPU and CUDA streams
differ, so a test that compares two implementations generates once and copies the bytes.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

# sub-stream identifiers (mixed into the seed)
_S_CHANNEL, _S_OUTLIER, _S_LN, _S_X, _S_CALIB, _S_K, _S_V, _S_W, _S_WQ = range(9)

_DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def torch_dtype(name: str) -> torch.dtype:
    return _DTYPES[name]


def _gen(seed: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + 7919 * (stream + 1)) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


@dataclass
class ChannelModel:
    center: torch.Tensor      # fp32 [C] (on CPU)
    half_width: torch.Tensor  # fp32 [C] (on CPU)
    outliers: torch.Tensor    # int64 indices of the outlier channels


def channel_model(C: int, seed: int, outlier_frac: float = 0.01, outlier_factor: float = 100.0,
                  tag: int = 0) -> ChannelModel:
    """Per-channel (centre, half-width) draw; `tag` separates independent models (K vs V)."""
    g = _gen(seed * 16 + tag, _S_CHANNEL, "cpu")
    center = torch.randn(C, generator=g, dtype=torch.float64) * 2.0
    hw = torch.exp(torch.randn(C, generator=g, dtype=torch.float64))
    n_out = int(outlier_frac * C)
    go = _gen(seed * 16 + tag, _S_OUTLIER, "cpu")
    idx = torch.randperm(C, generator=go)[:n_out]
    center[idx] *= outlier_factor
    hw[idx] *= outlier_factor
    return ChannelModel(center.float(), hw.float(), idx)


def ln_params(C: int, seed: int):
    """LayerNorm gamma ~ U(0.5, 1.5), beta ~ N(0, 0.1); fp32 on CPU, original channel order."""
    g = _gen(seed, _S_LN, "cpu")
    gamma = torch.rand(C, generator=g, dtype=torch.float64) + 0.5
    beta = torch.randn(C, generator=g, dtype=torch.float64) * 0.1
    return gamma.float(), beta.float()


def _fill_rows(out: torch.Tensor, model: ChannelModel, g: torch.Generator, chunk_rows: int):
    """out[T, C] <- centre + hw * (2u - 1), u ~ U(0, 1), drawn in row chunks."""
    T, C = out.shape
    dev = out.device
    center = model.center.to(dev)
    hw = model.half_width.to(dev)
    for t0 in range(0, T, chunk_rows):
        t1 = min(T, t0 + chunk_rows)
        u = torch.rand((t1 - t0, C), generator=g, device=dev, dtype=torch.float32)
        out[t0:t1] = (center + hw * (2.0 * u - 1.0)).to(out.dtype)
    return out


def activations(T: int, model: ChannelModel, seed: int, dtype: str = "bf16", device="cpu",
                calibration: bool = False, chunk_rows: int = 8192) -> torch.Tensor:
    """Token activations [T, C] of one model; `calibration` selects the independent
    calibration-batch stream instead of the runtime-batch stream."""
    C = model.center.numel()
    out = torch.empty((T, C), dtype=_DTYPES[dtype], device=device)
    g = _gen(seed, _S_CALIB if calibration else _S_X, device)
    return _fill_rows(out, model, g, chunk_rows)


def kv_cache(B: int, H: int, S: int, D: int, model: ChannelModel, seed: int, which: str = "k",
             dtype: str = "f16", device="cpu", chunk_rows: int = 8192) -> torch.Tensor:
    """A K or V cache [B, H, S, D] whose channel c = h*D + d follows `model` (C = H*D)."""
    assert model.center.numel() == H * D
    out = torch.empty((B, S, H * D), dtype=_DTYPES[dtype], device=device)
    g = _gen(seed, _S_K if which == "k" else _S_V, device)
    _fill_rows(out.view(B * S, H * D), model, g, chunk_rows)
    # tokens were drawn as rows of H*D channels; lay them out as [B, H, S, D]
    return out.view(B, S, H, D).permute(0, 2, 1, 3).contiguous()


def weights(N: int, C: int, seed: int) -> torch.Tensor:
    """Synthetic weights [N, C] of the linear layer that reads the activations (original channel
    order), W ~ N(0, 1/C); fp32 on CPU."""
    g = _gen(seed, _S_W, "cpu")
    return (torch.randn((N, C), generator=g, dtype=torch.float32) * (1.0 / C) ** 0.5).contiguous()


def weight_codes(N: int, C: int, seed: int, device="cpu"):
    """Synthetic 4-bit weight codes of the linear layer for the benchmark, already packed
    (uniform random bytes: every nibble uniform on 0..15, low nibble = even channel), with per-row
    scales s_w ~ U(0.5, 1.5) / (15 sqrt(C)) and zero points z_w ~ U{0..15}."""
    g = _gen(seed, _S_WQ, "cpu")
    packed = torch.randint(0, 256, (N, C // 2), generator=g, dtype=torch.uint8)
    sw = ((torch.rand(N, generator=g, dtype=torch.float64) + 0.5) / (15.0 * C ** 0.5)).float()
    zw = torch.randint(0, 16, (N,), generator=g, dtype=torch.int32)
    return packed.to(device), sw.to(device), zw.to(device)
