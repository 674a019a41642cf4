// kv_quant.cu -- per-cluster quantization of the attention K/V cache.
//
// RPTQ article (基于重排序的新量化方法RPTQ…), results paragraph: the W4A4KV / W4A3KV / W3A3KV
// settings quantize the key and value caches alone, with the same per-cluster asymmetric
// quantizer as the activations (text after Fig. 2; quantization-basics article, section 1.3).
//
// The cache keeps its [B, H, S, D] layout; channel c = h*D + d carries the cluster id of
// channel c.  A CTA handles one (b, h) pair of one tensor: all its S rows share the same D
// channels, so every thread loads the coefficients of its DPT consecutive channels once
//     A_d = 1 / (s_k * qmax),  B_d = z_k / qmax        (u = sat(x*A_d + B_d), code = rint(u*qmax))
// and then streams rows: 16-byte loads, codes accumulated in registers (the rounding constant
// 1.5*2^23 leaves each code in the low bits of a float; a shifted sum of those bit patterns
// minus a known constant is the packed word), and whole-word stores of the packed codes.
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace rptq {

// Correctly rounded x / s from r = RN(1/s): q0 = RN(x r), the residual x - q0 s is exact in
// one fused multiply-add, and q0 + residual * r rounds to RN(x / s) (P. Markstein, "IA-64 and
// Elementary Functions", 2000, division by a reciprocal with one correction).  Quotients that
// are exact half-integers therefore stay exact and round half-to-even like the reference.
__device__ __forceinline__ float div_rn(float x, float s, float r)
{
    const float q0 = x * r;
    const float res = fmaf(-q0, s, x);
    return fmaf(res, r, q0);
}

template <typename T, int BITS, int DPT>
__global__ void __launch_bounds__(256)
    kv_quant_kernel(const T *__restrict__ k, const T *__restrict__ v, int H, int64_t S, int D,
                    const int32_t *__restrict__ ck, const float *__restrict__ sk,
                    const int32_t *__restrict__ zk, const int32_t *__restrict__ cv,
                    const float *__restrict__ sv, const int32_t *__restrict__ zv, int g,
                    uint8_t *__restrict__ kq, uint8_t *__restrict__ vq, int *err)
{
    constexpr int VEC = Elem<T>::VEC;
    constexpr int NLD = DPT / VEC;  // 16-byte loads per row and thread
    constexpr int NG = DPT / 8;     // packed 8-code groups per row and thread
    constexpr int QMAX = (1 << BITS) - 1;
    constexpr uint32_t MAGIC_BITS = 0x4B400000u;
    constexpr int U = 4;            // rows whose loads are in flight together
    const bool is_v = blockIdx.y == 1;
    const T *src = is_v ? v : k;
    uint8_t *dst = is_v ? vq : kq;
    const int32_t *cl = is_v ? cv : ck;
    const float *sc = is_v ? sv : sk;
    const int32_t *zp = is_v ? zv : zk;
    if (src == nullptr) return;

    const int bh = blockIdx.x;  // b*H + h
    const int h = bh % H;
    const int TPR = D / DPT;    // threads per row
    const int RPI = blockDim.x / TPR;
    const int tl = threadIdx.x % TPR, rr = threadIdx.x / TPR;
    if (rr >= RPI) return;
    const int d0 = tl * DPT;

    // per-channel divisor s (negated), its reciprocal r, and the code-domain clamp [-z, qmax - z]
    f32x2 ns2[DPT / 2], r2[DPT / 2];
    float lo_[DPT], hi_[DPT];
    uint32_t bias[NG];  // sum_i (MAGIC_BITS - z_i) << (BITS*i): removes the rounding constant
    bool small_z = true;  // |z| < 2^21 keeps q + 1.5*2^23 inside one binade (exact rounding)
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) bias[gi] = 0;
#pragma unroll
    for (int i = 0; i < DPT; i += 2) {
        float sv2[2], rv2[2];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            int kc = cl[h * D + d0 + i + h2];
            if (kc < 0 || kc >= g) {
                raise_error(err, RPTQ_DEVERR_CLUSTER_ID);
                kc = 0;
            }
            sv2[h2] = sc[kc];
            rv2[h2] = __frcp_rn(sv2[h2]);
            const int z = zp[kc];
            lo_[i + h2] = (float)(-z);
            hi_[i + h2] = (float)(QMAX - z);
            bias[(i + h2) / 8] += (MAGIC_BITS - (uint32_t)z) << (BITS * ((i + h2) % 8));
            small_z &= (z > -(1 << 21)) && (z < (1 << 21));
        }
        ns2[i / 2] = mk2(-sv2[0], -sv2[1]);
        r2[i / 2] = mk2(rv2[0], rv2[1]);
    }
    const f32x2 magic2 = mk2(MAGIC_RINT, MAGIC_RINT);
    const int64_t pitch = (int64_t)D * BITS / 8;
    const T *base = src + (int64_t)bh * S * D + d0;
    uint8_t *obase = dst + (int64_t)bh * S * pitch + (int64_t)tl * (DPT * BITS / 8);

    for (int64_t s0 = rr; s0 < S; s0 += (int64_t)U * RPI) {
        uint4 xb[U][NLD];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t row = s0 + (int64_t)u * RPI;
#pragma unroll
            for (int l = 0; l < NLD; ++l)
                xb[u][l] = row < S ? ldg_stream(base + row * D + l * VEC) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t row = s0 + (int64_t)u * RPI;
            if (row >= S) break;
            uint32_t grp[NG];
            if (small_z) {
#pragma unroll
                for (int gi = 0; gi < NG; ++gi) {
                    uint32_t acc = 0;
#pragma unroll
                    for (int j = 0; j < 8; j += 2) {
                        const int i = gi * 8 + j;
                        // correctly rounded x/s for two channels (reciprocal + one correction)
                        const f32x2 x2 = pair_of<T>(xb[u][i / VEC], (i % VEC) / 2);
                        const f32x2 q0 = mul2(x2, r2[i / 2]);
                        const f32x2 q1 = fma2(fma2(q0, ns2[i / 2], x2), r2[i / 2], q0);
                        // clamp(rint(q) + z) == rint(clamp(q, -z, qmax - z)) + z
                        const f32x2 qc = mk2(fminf(fmaxf(lo2(q1), lo_[i]), hi_[i]),
                                             fminf(fmaxf(hi2(q1), lo_[i + 1]), hi_[i + 1]));
                        const f32x2 b2 = add2(qc, magic2);
                        acc += __float_as_uint(lo2(b2)) << (BITS * j);
                        acc += __float_as_uint(hi2(b2)) << (BITS * (j + 1));
                    }
                    grp[gi] = acc - bias[gi];
                }
            } else {  // a huge zero point: integer rounding and clamping
#pragma unroll
                for (int gi = 0; gi < NG; ++gi) {
                    uint32_t acc = 0;
                    for (int j = 0; j < 8; ++j) {
                        const int i = gi * 8 + j;
                        const float xf = Elem<T>::get(xb[u][i / VEC], i % VEC);
                        const float si = (i & 1) ? -hi2(ns2[i / 2]) : -lo2(ns2[i / 2]);
                        const float ri = (i & 1) ? hi2(r2[i / 2]) : lo2(r2[i / 2]);
                        const float q = rintf(div_rn(xf, si, ri));
                        const float c = fminf(fmaxf(q, lo_[i]), hi_[i]) - lo_[i];
                        acc |= (uint32_t)c << (BITS * j);
                    }
                    grp[gi] = acc;
                }
            }
            uint8_t *o = obase + row * pitch;
            if constexpr (BITS == 4) {
                if constexpr (NG == 2)
                    *reinterpret_cast<uint2 *>(o) = make_uint2(grp[0], grp[1]);
                else
                    *reinterpret_cast<uint32_t *>(o) = grp[0];
            } else {
                if constexpr (NG == 2) {  // 6 bytes at an even offset: three 2-byte stores
                    uint16_t *o16 = reinterpret_cast<uint16_t *>(o);
                    o16[0] = (uint16_t)grp[0];
                    o16[1] = (uint16_t)((grp[0] >> 16) | (grp[1] << 8));
                    o16[2] = (uint16_t)(grp[1] >> 8);
                } else {
                    o[0] = (uint8_t)grp[0];
                    o[1] = (uint8_t)(grp[0] >> 8);
                    o[2] = (uint8_t)(grp[0] >> 16);
                }
            }
        }
    }
}

template <typename T, int BITS, int DPT>
static cudaError_t launch_kv_t(const KvArgs &a)
{
    // D <= 2048 (checked by the caller) keeps threads-per-row D / DPT <= 256
    const int threads = 256;
    const dim3 grid((unsigned)(a.B * a.H), 2);
    kv_quant_kernel<T, BITS, DPT><<<grid, threads, 0, a.stream>>>(
        (const T *)a.k, (const T *)a.v, a.H, a.S, a.D, a.ck, a.sk, a.zk, a.cv, a.sv, a.zv, a.g, a.kq,
        a.vq, a.err);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_kv_d(const KvArgs &a)
{
    if (a.D % 16 == 0) return a.bits == 4 ? launch_kv_t<T, 4, 16>(a) : launch_kv_t<T, 3, 16>(a);
    return a.bits == 4 ? launch_kv_t<T, 4, 8>(a) : launch_kv_t<T, 3, 8>(a);
}

cudaError_t launch_kv_quant(const KvArgs &a)
{
    if (a.S == 0 || a.B == 0 || a.H == 0) return cudaSuccess;
    switch (a.dtype) {
    case RPTQ_F32: return launch_kv_d<float>(a);
    case RPTQ_F16: return launch_kv_d<__half>(a);
    default: return launch_kv_d<__nv_bfloat16>(a);
    }
}

}  // namespace rptq
