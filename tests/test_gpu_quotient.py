"""The K/V quantizer's division, exhaustively: for every finite bf16 and fp16 value x and a
spread of cluster scales s, the quotient the kernels form (RN(1/s), then one fused
multiply-add correction; P. Markstein, 2000; at a 2^-24 scale so that no product overflows)
equals the IEEE round-to-nearest fp32 x / s, bit for bit, infinities included, wherever |x| and
|x / s| are at least 2^-100.  Code decisions rest on it: exact half-integer quotients (frequent
for raw 16-bit cache values) must round half-to-even like the oracle.  Below 2^-100 the
correction's residual can be subnormal and the last bit may differ, but the quotient is then far
below 1/2: the test asks for the same rounded integer there.  Scales outside [2^-24, 2^102]
take the IEEE division itself."""
import numpy as np
import pytest
import torch

from post_activation_quantization_b200 import rptq
from tests.gpu_common import DEV

pytestmark = pytest.mark.gpu

SCALES = [1.0, 0.5, 3.0, 7.0, 0.1, 1 / 3, 13.333333, 2.857143, 1e-3, 37.5, 1234.5678, 6.1035e-05, 1e-6,
          0.7, 1.4285715, 9.99, 2.0 ** -20, 1e30, 1e-30]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from post_activation_quantization_b200 import build
    build.build()
    rptq.lib()


def _all_finite(kind):
    bits = np.arange(65536, dtype=np.uint32)
    if kind == "bf16":
        v = (bits << 16).view(np.float32)
    else:
        v = bits.astype(np.uint16).view(np.float16).astype(np.float32)
    return v[np.isfinite(v)]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("s", SCALES)
def test_quotient_is_ieee_division(kind, s):
    x = _all_finite(kind)
    s32 = np.float32(s)
    with np.errstate(over="ignore"):
        want = x / s32  # IEEE fp32 division, round to nearest even
    for n in (len(x), len(x) - 1):  # even: the packed form throughout; odd: the last value scalar
        got = rptq.rptq_testing_kv_quotient(torch.from_numpy(x[:n]).to(DEV), float(s32)).cpu().numpy()
        w = want[:n]
        xs = x[:n]
        exact = (np.abs(xs) >= 2.0 ** -100) & (np.abs(w) >= 2.0 ** -100)
        assert np.array_equal(got[exact].view(np.uint32), w[exact].view(np.uint32)), (
            f"{kind} s={s}: {(got[exact].view(np.uint32) != w[exact].view(np.uint32)).sum()} quotients differ")
        assert np.array_equal(np.rint(got[~exact]), np.rint(w[~exact]))
