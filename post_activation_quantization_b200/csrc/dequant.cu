// dequant.cu -- dequantization value = s_k * (q - z_k) (quantization-basics article,
// section 1.3: the real value is the scale times the code minus the zero point).
//
// The code q becomes an exact float without a conversion instruction: the bit pattern
// 0x4B000000 | q is the float 2^23 + q, and 2^23 + z is exact for |z| < 2^23 - 16, so
// (2^23 + q) - (2^23 + z) = q - z exactly and one multiply by s gives the same fp32 value as
// s * (float)(q - z).  A thread whose columns include a larger |z| converts with an integer ->
// float conversion instead (same result).  Each thread owns DPT consecutive channels (32 when
// the row length allows, else 8) and keeps their (s, 2^23 + z) in registers across rows.
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace rptq {

template <typename T> struct Store;
template <> struct Store<float> {
    template <int N> __device__ static void put(float *dst, const float (&v)[N])
    {
#pragma unroll
        for (int i = 0; i < N; i += 4)
            *reinterpret_cast<float4 *>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    }
};
template <> struct Store<__nv_bfloat16> {
    template <int N> __device__ static void put(__nv_bfloat16 *dst, const float (&v)[N])
    {
#pragma unroll
        for (int i = 0; i < N; i += 8) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const __nv_bfloat162 p = __floats2bfloat162_rn(v[i + 2 * j], v[i + 2 * j + 1]);
                w[j] = *reinterpret_cast<const uint32_t *>(&p);
            }
            *reinterpret_cast<uint4 *>(dst + i) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
};
template <> struct Store<__half> {
    template <int N> __device__ static void put(__half *dst, const float (&v)[N])
    {
#pragma unroll
        for (int i = 0; i < N; i += 8) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const __half2 p = __floats2half2_rn(v[i + 2 * j], v[i + 2 * j + 1]);
                w[j] = *reinterpret_cast<const uint32_t *>(&p);
            }
            *reinterpret_cast<uint4 *>(dst + i) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
};

// Read the packed codes of DPT consecutive positions (DPT*BITS/8 bytes) as 8-code groups.
template <int BITS, int DPT>
__device__ __forceinline__ void load_groups(const uint8_t *p, uint32_t (&grp)[DPT / 8])
{
    if constexpr (BITS == 4) {
        if constexpr (DPT == 32) {
            const uint4 q = *reinterpret_cast<const uint4 *>(p);
            grp[0] = q.x;
            grp[1] = q.y;
            grp[2] = q.z;
            grp[3] = q.w;
        } else {
            grp[0] = *reinterpret_cast<const uint32_t *>(p);
        }
    } else {
        if constexpr (DPT == 32) {
            const uint32_t *p32 = reinterpret_cast<const uint32_t *>(p);
            const uint32_t w0 = p32[0], w1 = p32[1], w2 = p32[2];
            grp[0] = w0 & 0xffffffu;
            grp[1] = (w0 >> 24) | ((w1 & 0xffffu) << 8);
            grp[2] = (w1 >> 16) | ((w2 & 0xffu) << 16);
            grp[3] = w2 >> 8;
        } else {
            grp[0] = (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16);
        }
    }
}

// rows of `width` channels; the channel of position p in a row is chan0 + p (its cluster is
// cluster[chan0 + p]).  Used for both layouts: ROWS (chan0 = 0, width = C) and BHSD (one (b,h)
// pair per blockIdx.x, chan0 = h*D, width = D).
template <typename T, int BITS, int DPT>
__global__ void __launch_bounds__(256, 2)
    dequant_kernel(const uint8_t *__restrict__ codes, int64_t rows, int width, int rows_per_bh, int H,
                   const int32_t *__restrict__ cluster, const float *__restrict__ scale,
                   const int32_t *__restrict__ zero, int g, T *__restrict__ out, int *err)
{
    constexpr int NGRP = DPT / 8;
    constexpr uint32_t QMASK = (1u << BITS) - 1;
    const int TPR = width / DPT;
    // BHSD: blockIdx.x = b*H + h and the CTA walks the S rows of that pair;
    // ROWS: blockIdx.y selects a column block, the CTA walks rows with stride gridDim.x.
    const bool bhsd = rows_per_bh > 0;
    int tl, rr, RPI;
    int64_t r0, r1, rstep;
    int chan0;
    if (bhsd) {
        tl = threadIdx.x % TPR;
        rr = threadIdx.x / TPR;
        RPI = blockDim.x / TPR;
        if (rr >= RPI) return;
        const int bh = blockIdx.x;
        chan0 = (bh % H) * width;
        r0 = (int64_t)bh * rows_per_bh + rr;
        r1 = (int64_t)(bh + 1) * rows_per_bh;
        rstep = RPI;
    } else {
        tl = blockIdx.y * blockDim.x + threadIdx.x;
        if (tl >= TPR) return;
        chan0 = 0;
        r0 = blockIdx.x;
        r1 = rows;
        rstep = gridDim.x;
    }
    const int p0 = tl * DPT;
    float sc[DPT], zf[DPT];
    bool exact = true;
#pragma unroll
    for (int i = 0; i < DPT; ++i) {
        int k = cluster[chan0 + p0 + i];
        if (k < 0 || k >= g) {
            raise_error(err, RPTQ_DEVERR_CLUSTER_ID);
            k = 0;
        }
        sc[i] = scale[k];
        const int z = zero[k];
        const bool ok = (z > -(1 << 23) + 16) && (z < (1 << 23) - 16);
        exact &= ok;
        zf[i] = (float)((1 << 23) + (ok ? z : 0));
    }
    const int64_t pitch = (int64_t)width * BITS / 8;
    const uint8_t *cbase = codes + (int64_t)tl * (DPT * BITS / 8);
    T *obase = out + p0;
    if (exact) {
        constexpr int U = 4;  // rows of codes in flight per thread
        for (int64_t rb = r0; rb < r1; rb += (int64_t)U * rstep) {
            uint32_t grp[U][NGRP];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t r = rb + (int64_t)u * rstep;
                if (r < r1)
                    load_groups<BITS, DPT>(cbase + r * pitch, grp[u]);
                else
#pragma unroll
                    for (int i = 0; i < NGRP; ++i) grp[u][i] = 0;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t r = rb + (int64_t)u * rstep;
                if (r >= r1) break;
#pragma unroll
                for (int c8 = 0; c8 < NGRP; ++c8) {
                    float v[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint32_t q = (grp[u][c8] >> (BITS * i)) & QMASK;
                        v[i] = sc[8 * c8 + i] * (__uint_as_float(0x4B000000u | q) - zf[8 * c8 + i]);
                    }
                    Store<T>::template put<8>(obase + r * width + 8 * c8, v);
                }
            }
        }
    } else {  // some |z| too large for the exact float form: integer subtraction, then convert
        for (int64_t r = r0; r < r1; r += rstep) {
            uint32_t grp[NGRP];
            load_groups<BITS, DPT>(cbase + r * pitch, grp);
            for (int c8 = 0; c8 < NGRP; ++c8) {
                float v[8];
                for (int i = 0; i < 8; ++i) {
                    const uint32_t q = (grp[c8] >> (BITS * i)) & QMASK;
                    int k = cluster[chan0 + p0 + 8 * c8 + i];
                    k = (k < 0 || k >= g) ? 0 : k;
                    v[i] = scale[k] * (float)((int)q - zero[k]);
                }
                Store<T>::template put<8>(obase + r * width + 8 * c8, v);
            }
        }
    }
}

template <typename T, int BITS, int DPT>
static cudaError_t launch_dq_t(const DequantArgs &a)
{
    if (a.layout == RPTQ_LAYOUT_BHSD) {
        const dim3 grid((unsigned)(a.n0 * a.n1));
        dequant_kernel<T, BITS, DPT><<<grid, 256, 0, a.stream>>>(a.codes, a.n0 * a.n1 * a.S, a.D, (int)a.S,
                                                                  a.n1, a.cluster, a.scale, a.zero, a.g,
                                                                  (T *)a.out, a.err);
    } else {
        const int TPR = a.n1 / DPT;
        const int threads = std::min(256, (TPR + 31) / 32 * 32);
        const int gy = (TPR + threads - 1) / threads;
        const int64_t want = (int64_t)a.num_sms * 8 / gy + 1;
        const int64_t gx = std::max<int64_t>(1, std::min<int64_t>(a.n0, want));
        dequant_kernel<T, BITS, DPT><<<dim3((unsigned)gx, gy), threads, 0, a.stream>>>(
            a.codes, a.n0, a.n1, 0, 1, a.cluster, a.scale, a.zero, a.g, (T *)a.out, a.err);
    }
    return cudaGetLastError();
}

template <typename T, int BITS>
static cudaError_t launch_dq_b(const DequantArgs &a)
{
    const int width = a.layout == RPTQ_LAYOUT_BHSD ? a.D : a.n1;
    if (width % 32 == 0) return launch_dq_t<T, BITS, 32>(a);
    return launch_dq_t<T, BITS, 8>(a);
}

template <typename T>
static cudaError_t launch_dq_d(const DequantArgs &a)
{
    return a.bits == 4 ? launch_dq_b<T, 4>(a) : launch_dq_b<T, 3>(a);
}

cudaError_t launch_dequant(const DequantArgs &a)
{
    const int64_t rows = a.layout == RPTQ_LAYOUT_BHSD ? a.n0 * a.n1 * a.S : a.n0;
    if (rows == 0) return cudaSuccess;
    switch (a.out_dtype) {
    case RPTQ_F32: return launch_dq_d<float>(a);
    case RPTQ_F16: return launch_dq_d<__half>(a);
    default: return launch_dq_d<__nv_bfloat16>(a);
    }
}

}  // namespace rptq
