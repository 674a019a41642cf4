"""The five RPTQ workloads this library is tested and measured on, and their byte counts.

Sizes follow OPT hidden widths (768, 4096, 9216, 12288) and an attention K/V cache.
Values not fixed by the workload descriptions are readings, marked `# reading`.
"""
from __future__ import annotations

from dataclasses import dataclass, field

ESIZE = {"f32": 4, "f16": 2, "bf16": 2}


@dataclass(frozen=True)
class KV:
    B: int
    H: int
    S: int
    D: int
    dtype: str
    g: int
    iters: int
    bits: int
    outlier_frac: float = 0.01
    outlier_factor: float = 100.0

    @property
    def channels(self) -> int:
        return self.H * self.D

    @property
    def elems(self) -> int:
        return self.B * self.H * self.S * self.D


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    # activation path (None for a KV-only workload)
    T: int = 0
    C: int = 0
    dtype: str = "bf16"
    T_cal: int = 0            # 0: calibrate on the runtime batch itself
    g: int = 0
    iters: int = 0
    bits: int = 4
    outlier_frac: float = 0.01
    outlier_factor: float = 100.0
    kv: KV | None = None
    eps: float = 1e-5         # reading: PyTorch's LayerNorm default
    notes: tuple = field(default_factory=tuple)

    @property
    def has_act(self) -> bool:
        return self.T > 0


WORKLOADS = {
    "tiny-768": Workload(
        "tiny-768", seed=0, T=512, C=768, dtype="f32", T_cal=0, g=8, iters=10, bits=4),
    "opt6.7b-4096": Workload(
        "opt6.7b-4096", seed=1, T=2048, C=4096, dtype="f16", T_cal=128 * 2048, g=32, iters=20,
        bits=4),
    "kv-4096": Workload(
        "kv-4096", seed=2,
        kv=KV(B=16, H=32, S=2048, D=128, dtype="f16", g=32, iters=20, bits=3),  # iters: reading
        notes=("iters=20 is a reading (not stated for the K/V workload)",)),
    "opt66b-9216": Workload(
        "opt66b-9216", seed=3, T=16384, C=9216, dtype="bf16", T_cal=128 * 2048, g=64, iters=30,
        bits=3, outlier_frac=0.005, outlier_factor=200.0),
    "opt175b-12288": Workload(
        "opt175b-12288", seed=4, T=32768, C=12288, dtype="bf16", T_cal=128 * 2048, g=64,
        iters=50, bits=3,
        kv=KV(B=8, H=96, S=2048, D=128, dtype="bf16", g=64, iters=50, bits=3),  # g, iters, dtype: reading
        notes=("K/V g=64, iters=50 and bf16 are readings",)),
}

ORDER = ["tiny-768", "opt6.7b-4096", "kv-4096", "opt66b-9216", "opt175b-12288"]


# ---- algorithmic bytes (what a kernel must move at minimum; small per-channel tables excluded)

def bytes_calib(T: int, C: int, dtype: str) -> int:
    """Calibration min/max: read the [T, C] tensor once (the 8*C output bytes are negligible)."""
    return T * C * ESIZE[dtype]


def bytes_ln_quant(T: int, C: int, dtype: str, bits: int, ln_out: bool = False) -> int:
    """Fused LN + reorder + cluster quant: read x, write packed codes (and the dense LN output)."""
    b = T * C * ESIZE[dtype] + T * C * bits // 8
    if ln_out:
        b += T * C * ESIZE[dtype]
    return b


def bytes_ln_quant_plan(C: int) -> int:
    """The LayerNorm plan of one calibration: read gamma, beta, R, col_cluster (4 bytes each per
    channel), write the offset and two coefficients per channel."""
    return 16 * C + 12 * C


def bytes_kv_quant(n_elems: int, dtype: str, bits: int, tensors: int = 2) -> int:
    """K and V quant: read each element, write its packed code."""
    return tensors * (n_elems * ESIZE[dtype] + n_elems * bits // 8)


def bytes_dequant(n_elems: int, out_dtype: str, bits: int) -> int:
    return n_elems * bits // 8 + n_elems * ESIZE[out_dtype]


def kv_cache_bytes(layers: int, batch: int, seq: int, hidden: int, bits: int) -> int:
    """Size of a K+V cache: two tensors of layers x batch x seq x hidden values of `bits` bits."""
    return 2 * layers * batch * seq * hidden * bits // 8


def bytes_kv_append(B: int, H: int, D: int, dtype: str, bits: int) -> int:
    """One decode step's append: read one new token of K and of V, write its packed codes."""
    return 2 * (B * H * D * ESIZE[dtype] + B * H * D * bits // 8)


def bytes_kv_attention(B: int, H: int, L: int, D: int, bits: int) -> int:
    """Decode attention over L positions: read the packed K and V rows once, the fp32 query,
    write the fp32 output."""
    return 2 * B * H * L * D * bits // 8 + 2 * B * H * D * 4


def bytes_explicit_reorder(T: int, C: int, dtype: str, bits: int) -> int:
    """The unfused pipeline: read x, write the fp32 LayerNorm output, read it and write the fp32
    reordered copy, read that and write the packed codes."""
    n = T * C
    return n * ESIZE[dtype] + 4 * n * 4 + n * bits // 8


# ---- the reordered linear layer after the LayerNorm (a tensor-core contraction, not HBM-bound)
LINEAR_TOKENS = 2048  # one 2048-token micro-batch of the step's activation codes


def linear_shape(w: "Workload"):
    """(tokens, C, N) of the layer the step runs on the activation codes: the first
    min(T, 2048) tokens through the fused Q/K/V projection of the model (N = 3 C)."""
    return min(w.T, LINEAR_TOKENS), w.C, 3 * w.C


def flops_linear(T: int, C: int, N: int) -> int:
    """Multiply-adds of the layer, counted as 2 operations each."""
    return 2 * T * C * N


def bytes_linear_prepare(N: int, C: int) -> int:
    """Offline operand preparation: read the 4-bit weight codes, write the fp16 operand and the
    per-row bias and scale."""
    return N * C // 2 + N * C * 2 + 2 * N * 4
