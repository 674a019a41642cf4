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

template <typename T, int BITS>
__global__ void __launch_bounds__(256)
    kv_quant_kernel(const T *__restrict__ k, const T *__restrict__ v, int H, int64_t S, int D,
                    const int32_t *__restrict__ ck, const float *__restrict__ sk,
                    const int32_t *__restrict__ zk, const int32_t *__restrict__ cv,
                    const float *__restrict__ sv, const int32_t *__restrict__ zv, int g,
                    uint8_t *__restrict__ kq, uint8_t *__restrict__ vq, int *err)
{
    constexpr int VEC = Elem<T>::VEC;
    constexpr int NLD = 8 / VEC;  // 16-byte loads per 8 channels
    constexpr int QMAX = (1 << BITS) - 1;
    constexpr uint32_t MAGIC_BITS = 0x4B400000u;
    const bool is_v = blockIdx.y == 1;
    const T *src = is_v ? v : k;
    uint8_t *dst = is_v ? vq : kq;
    const int32_t *cl = is_v ? cv : ck;
    const float *sc = is_v ? sv : sk;
    const int32_t *zp = is_v ? zv : zk;
    if (src == nullptr) return;

    const int bh = blockIdx.x;  // b*H + h
    const int h = bh % H;
    const int TPR = D / 8;      // threads per row, 8 channels each
    const int RPI = blockDim.x / TPR;
    const int tl = threadIdx.x % TPR, rr = threadIdx.x / TPR;
    const bool active = rr < RPI;
    const int d0 = tl * 8;

    // per-channel divisor, its reciprocal and the code-domain clamp [-z, qmax - z]
    float s8[8], r8[8], lo8[8], hi8[8];
    uint32_t bias = 0;  // sum_i (MAGIC_BITS - z_i) << (BITS*i): removes the rounding constant
    bool small_z = true;  // |z| < 2^21 keeps q + 1.5*2^23 inside one binade (exact rounding)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int kc = active ? cl[h * D + d0 + i] : 0;
        if (kc < 0 || kc >= g) {
            raise_error(err, RPTQ_DEVERR_CLUSTER_ID);
            kc = 0;
        }
        s8[i] = sc[kc];
        r8[i] = __frcp_rn(s8[i]);
        const int z = zp[kc];
        lo8[i] = (float)(-z);
        hi8[i] = (float)(QMAX - z);
        bias += (MAGIC_BITS - (uint32_t)z) << (BITS * i);
        small_z &= (z > -(1 << 21)) && (z < (1 << 21));
    }
    const int64_t pitch = (int64_t)D * BITS / 8;
    const T *base = src + (int64_t)bh * S * D + d0;
    uint8_t *obase = dst + (int64_t)bh * S * pitch;
    // A warp covers whole consecutive rows (or a run of one row) when TPR divides 32 or 32
    // divides TPR: its 3-byte groups then form one contiguous run that lanes store as words.
    const bool contiguous = (32 % TPR == 0) || (TPR % 32 == 0);
    const int lane = threadIdx.x & 31;

    const int64_t iters = active ? (S - rr + RPI - 1) / RPI : 0;
    const int64_t trips = (S + RPI - 1) / RPI;  // the same for every lane (shuffles below)
    constexpr int U = 4;                         // rows whose loads are in flight together
    for (int64_t it0 = 0; it0 < trips; it0 += U) {
        uint4 xb[U][NLD];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t s_row = rr + (it0 + u) * RPI;
            const bool valid = it0 + u < iters && s_row < S;
#pragma unroll
            for (int l = 0; l < NLD; ++l)
                xb[u][l] = valid ? ldg_stream(base + s_row * D + l * VEC) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        if (it0 + u >= trips) break;
        const int64_t it = it0 + u;
        const int64_t s_row = rr + it * RPI;
        const bool valid = it < iters && s_row < S;
        const uint4 *xv = xb[u];
        uint32_t grp;  // codes of the 8 channels, packed
        if (small_z) {
            uint32_t acc = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float xf = Elem<T>::get(xv[i / VEC], i % VEC);
                float q = div_rn(xf, s8[i], r8[i]);
                q = fminf(fmaxf(q, lo8[i]), hi8[i]);  // clamp(rint(q) + z) == rint(clamp(q)) + z
                acc += __float_as_uint(q + MAGIC_RINT) << (BITS * i);
            }
            grp = acc - bias;
        } else {  // a huge zero point: integer rounding and clamping
            grp = 0;
            for (int i = 0; i < 8; ++i) {
                const float xf = Elem<T>::get(xv[i / VEC], i % VEC);
                const float q = rintf(div_rn(xf, s8[i], r8[i]));
                const float c = fminf(fmaxf(q, lo8[i]), hi8[i]) - lo8[i];
                grp |= (uint32_t)c << (BITS * i);
            }
        }
        uint8_t *o = obase + s_row * pitch + (int64_t)tl * BITS;  // this thread's group
        if constexpr (BITS == 4) {
            if (valid) *reinterpret_cast<uint32_t *>(o) = grp;
        } else if (contiguous) {
            // The warp's groups form one run starting at lane 0's group; its valid lanes are a
            // prefix of the warp (rows beyond S come last).  Lane w < 24 writes bytes [4w, 4w+4)
            // of the run: a whole word when the run start is 4-byte aligned and the word is
            // complete, single bytes otherwise.
            const unsigned long long a0 = __shfl_sync(FULL, reinterpret_cast<unsigned long long>(o), 0);
            const int nbytes = 3 * __popc(__ballot_sync(FULL, valid));
            const int w = lane, a = (4 * w) / 3, off = (4 * w) % 3;
            const uint32_t ga = __shfl_sync(FULL, grp, a < 32 ? a : 31);
            const uint32_t gb = __shfl_sync(FULL, grp, a + 1 < 32 ? a + 1 : 31);
            const uint32_t lo = (ga & 0xffffffu) | (gb << 24), hi = (gb & 0xffffffu) >> 8;
            const uint32_t word = __funnelshift_r(lo, hi, 8 * off);
            uint8_t *run = reinterpret_cast<uint8_t *>(a0);
            if (w < 24 && 4 * w < nbytes) {
                if ((a0 & 3ull) == 0 && 4 * w + 4 <= nbytes) {
                    *reinterpret_cast<uint32_t *>(run + 4 * w) = word;
                } else {
                    for (int b = 0; b < 4 && 4 * w + b < nbytes; ++b) run[4 * w + b] = (uint8_t)(word >> (8 * b));
                }
            }
        } else if (valid) {
            o[0] = (uint8_t)grp;
            o[1] = (uint8_t)(grp >> 8);
            o[2] = (uint8_t)(grp >> 16);
        }
    }
    }
}

template <typename T, int BITS>
static cudaError_t launch_kv_b(const KvArgs &a)
{
    // D <= 2048 (checked by the caller) keeps threads-per-row D / 8 <= 256
    const int threads = 256;
    const dim3 grid((unsigned)(a.B * a.H), 2);
    kv_quant_kernel<T, BITS><<<grid, threads, 0, a.stream>>>(
        (const T *)a.k, (const T *)a.v, a.H, a.S, a.D, a.ck, a.sk, a.zk, a.cv, a.sv, a.zv, a.g, a.kq,
        a.vq, a.err);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_kv_d(const KvArgs &a)
{
    return a.bits == 4 ? launch_kv_b<T, 4>(a) : launch_kv_b<T, 3>(a);
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
