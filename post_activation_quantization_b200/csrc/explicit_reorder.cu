// explicit_reorder.cu -- the unfused pipeline that RPTQ's fused LayerNorm avoids, kept as a
// measurement baseline (include/rptq_baseline.h).
//
// RPTQ article (基于重排序的新量化方法RPTQ…), the paragraph before Fig. 3's text: reordering the
// activation channels explicitly at run time moves every channel and costs time and memory; the
// text after Fig. 3: RPTQ changes the LayerNorm so that it writes its output already in cluster
// order, and no reordered copy is ever made.  This file makes that copy on purpose, three kernels
// and two fp32 intermediates in HBM:
//   1. LayerNorm:  y[t, c]  = LN(x[t])[c]                 (read x, write y, original order)
//   2. reorder:    yr[t, j] = y[t, R[j]]                   (read y, write yr, cluster order)
//   3. quantize:   code[t, j] = clamp(rint(yr / s_k) + z_k, 0, qmax), k = col_cluster[j]
//                                                          (read yr, write the packed codes)
// The intermediates are fp32, so the codes are those of the fused kernel's definition (the
// quantizer sees the fp32 LayerNorm value).  Each kernel is a plain streaming kernel with
// coalesced 16-byte accesses; the reorder stages a row in shared memory and gathers from there.
#include <algorithm>

#include "launch.h"
#include "row_pipeline.cuh"

namespace rptq {

constexpr int XR_THREADS = 512;

// 1. LayerNorm of one row per CTA iteration; the row is staged in shared memory as fp32
//    (C floats), statistics two-pass (mean, then the deviations), y written with 16-byte stores.
template <typename T>
__global__ void __launch_bounds__(XR_THREADS)
    xr_layernorm_kernel(const T *__restrict__ x, int64_t T_, int C, const float *__restrict__ gamma,
                        const float *__restrict__ beta, float eps, float *__restrict__ y)
{
    extern __shared__ __align__(16) float row[];
    __shared__ float red[8 * 32];
    constexpr int VEC = Elem<T>::VEC;
    const int tid = threadIdx.x, NCH = C / VEC;
    for (int64_t t = blockIdx.x; t < T_; t += gridDim.x) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x + t * (int64_t)C);
        float s = 0.f;
        for (int ch = tid; ch < NCH; ch += XR_THREADS) {
            const uint4 v = ldg_stream(src + ch);
            float f[VEC];
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                f[e] = Elem<T>::get(v, e);
                s += f[e];
            }
            // whole 16-byte stores: a warp writes contiguous bytes, no bank conflict
#pragma unroll
            for (int e = 0; e < VEC; e += 4)
                reinterpret_cast<float4 *>(row)[(ch * VEC + e) / 4] = make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
        }
        float v8[8] = {s, 0, 0, 0, 0, 0, 0, 0};
        cta_sum8(v8, red);
        float hi, rstd, nmr;
        row_moments(row, C, v8[0], eps, red, hi, rstd, nmr);
        float4 *dst = reinterpret_cast<float4 *>(y + t * (int64_t)C);
        for (int c4 = tid; c4 < C / 4; c4 += XR_THREADS) {
            const float4 xv = reinterpret_cast<const float4 *>(row)[c4];
            const float4 gv = __ldg(reinterpret_cast<const float4 *>(gamma) + c4);
            const float4 bv = __ldg(reinterpret_cast<const float4 *>(beta) + c4);
            float4 o;
            o.x = fmaf(fmaf(xv.x - hi, rstd, nmr), gv.x, bv.x);
            o.y = fmaf(fmaf(xv.y - hi, rstd, nmr), gv.y, bv.y);
            o.z = fmaf(fmaf(xv.z - hi, rstd, nmr), gv.z, bv.z);
            o.w = fmaf(fmaf(xv.w - hi, rstd, nmr), gv.w, bv.w);
            dst[c4] = o;
        }
        __syncthreads();  // the row buffer and red are reused by the next row
    }
}

// 2. The explicit reorder: yr[t, j] = y[t, R[j]].  R is read into shared memory once per CTA;
//    each row of y is staged in shared memory (16-byte loads), then gathered in stored order
//    with 16-byte stores.
__global__ void __launch_bounds__(XR_THREADS)
    xr_reorder_kernel(const float *__restrict__ y, int64_t T_, int C, const int32_t *__restrict__ R,
                      float *__restrict__ yr, int *err)
{
    extern __shared__ __align__(16) float sm[];
    float *row = sm;                                            // C floats
    int32_t *rs = reinterpret_cast<int32_t *>(sm + C);          // C ints
    const int tid = threadIdx.x;
    for (int j = tid; j < C; j += XR_THREADS) {
        int c = R[j];
        if (c < 0 || c >= C) {
            raise_error(err, RPTQ_DEVERR_REORDER);
            c = 0;
        }
        rs[j] = c;
    }
    __syncthreads();
    for (int64_t t = blockIdx.x; t < T_; t += gridDim.x) {
        const float4 *src = reinterpret_cast<const float4 *>(y + t * (int64_t)C);
        for (int c4 = tid; c4 < C / 4; c4 += XR_THREADS) reinterpret_cast<float4 *>(row)[c4] = ldg_f4(src + c4);
        __syncthreads();
        float4 *dst = reinterpret_cast<float4 *>(yr + t * (int64_t)C);
        for (int j4 = tid; j4 < C / 4; j4 += XR_THREADS) {
            const int4 r = reinterpret_cast<const int4 *>(rs)[j4];
            dst[j4] = make_float4(row[r.x], row[r.y], row[r.z], row[r.w]);
        }
        __syncthreads();
    }
}

// 3. Per-cluster quantization of the reordered rows: a thread packs 8 consecutive stored
//    columns (one 3- or 4-byte group).  The cluster table (s, RN(1/s), z) is staged in shared
//    memory; the quotient is the correctly rounded y / s from the reciprocal and one fused
//    multiply-add correction (the K/V quantizer's method; the IEEE division for scales outside
//    [2^-24, 2^102] or |y| < 2^-100, where that correction's residual could be subnormal), and
//    clamp(rint(q) + z, 0, qmax) follows the definition.
template <int BITS>
__global__ void __launch_bounds__(256)
    xr_quant_kernel(const float *__restrict__ yr, int64_t T_, int C, const int32_t *__restrict__ col_cluster,
                    const float *__restrict__ scale, const int32_t *__restrict__ zero, int g,
                    uint8_t *__restrict__ codes, int *err)
{
    constexpr float QMAX = (float)((1 << BITS) - 1);
    __shared__ float4 tab[RPTQ_MAX_CLUSTERS];  // (s, RN(1/s), z, fast)
    for (int k = threadIdx.x; k < g; k += blockDim.x) {
        const float sk = scale[k];
        const bool fast = sk >= 0x1p-24f && sk <= 0x1p+102f;
        tab[k] = make_float4(sk, __frcp_rn(sk), (float)zero[k], fast ? 1.f : 0.f);
    }
    __syncthreads();
    const int groups = C / 8;
    const int64_t total = T_ * groups;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / groups;
        const int gi = (int)(i - t * groups);
        const float4 *src = reinterpret_cast<const float4 *>(yr + t * (int64_t)C + gi * 8);
        const float4 a = ldg_f4(src), b = ldg_f4(src + 1);
        const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        const int4 k0 = __ldg(reinterpret_cast<const int4 *>(col_cluster + gi * 8));
        const int4 k1 = __ldg(reinterpret_cast<const int4 *>(col_cluster + gi * 8) + 1);
        const int kk[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
        uint32_t w = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            int k = kk[e];
            if (k < 0 || k >= g) {
                raise_error(err, RPTQ_DEVERR_CLUSTER_ID);
                k = 0;
            }
            const float4 c = tab[k];
            float q;
            if (c.w != 0.f && fabsf(v[e]) >= 0x1p-100f) {
                const float q0 = v[e] * c.y;
                q = fmaf(fmaf(-q0, c.x, v[e]), c.y, q0);
            } else {
                q = __fdiv_rn(v[e], c.x);
            }
            // rint(q) + z is exact while |q| < 2^23; beyond, the clamp decides by the sign alone
            const float qc = fminf(fmaxf(rintf(q) + c.z, 0.f), QMAX);
            w |= (uint32_t)qc << (BITS * e);
        }
        uint8_t *dst = codes + t * (int64_t)(C * BITS / 8) + gi * BITS;
        if constexpr (BITS == 4) {
            *reinterpret_cast<uint32_t *>(dst) = w;
        } else {
            dst[0] = (uint8_t)w;
            dst[1] = (uint8_t)(w >> 8);
            dst[2] = (uint8_t)(w >> 16);
        }
    }
}

cudaError_t launch_explicit_reorder(const XrArgs &a)
{
    if (a.T == 0) return cudaSuccess;
    const int64_t grid_rows = std::min<int64_t>(a.T, (int64_t)a.num_sms * 4);
    // 1. LayerNorm
    {
        const size_t smem = (size_t)a.C * 4;
        const void *kern = a.dtype == RPTQ_F32   ? (const void *)xr_layernorm_kernel<float>
                           : a.dtype == RPTQ_F16 ? (const void *)xr_layernorm_kernel<__half>
                                                 : (const void *)xr_layernorm_kernel<__nv_bfloat16>;
        cudaError_t e = kernel_smem(kern, smem);
        if (e != cudaSuccess) return e;
        void *args[] = {(void *)&a.x, (void *)&a.T, (void *)&a.C, (void *)&a.gamma, (void *)&a.beta, (void *)&a.eps,
                        (void *)&a.y};
        e = cudaLaunchKernel(kern, dim3((unsigned)grid_rows), dim3(XR_THREADS), args, smem, a.stream);
        if (e != cudaSuccess) return e;
    }
    // 2. explicit reorder
    {
        const size_t smem = (size_t)a.C * 8;
        cudaError_t e = kernel_smem((const void *)xr_reorder_kernel, smem);
        if (e != cudaSuccess) return e;
        xr_reorder_kernel<<<(unsigned)grid_rows, XR_THREADS, smem, a.stream>>>(a.y, a.T, a.C, a.R, a.yr, a.err);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // 3. quantize + pack
    const int64_t total = a.T * (a.C / 8);
    const unsigned grid = (unsigned)std::min<int64_t>((total + 255) / 256, (int64_t)a.num_sms * 16);
    if (a.bits == 4)
        xr_quant_kernel<4><<<grid, 256, 0, a.stream>>>(a.yr, a.T, a.C, a.col_cluster, a.scale, a.zero, a.g, a.codes,
                                                       a.err);
    else
        xr_quant_kernel<3><<<grid, 256, 0, a.stream>>>(a.yr, a.T, a.C, a.col_cluster, a.scale, a.zero, a.g, a.codes,
                                                       a.err);
    return cudaGetLastError();
}

}  // namespace rptq
