// kv_attention.cu -- one decode step of attention reading the packed K/V caches directly.
//
// RPTQ article (基于重排序的新量化方法RPTQ…), results paragraph (the K and V caches quantized per
// cluster: W4A4KV / W4A3KV / W3A3KV) and closing memory paragraph (at large batch x sequence the
// cache dominates memory): the consumer of the quantized cache never materialises K or V in 16
// or 32 bits; every code is dequantized in registers as it is read,
//     value = s_k * (q - z_k)     (quantization-basics article, section 1.3; fp32, one rounding,
//                                  the same value rptq_dequant writes),
// and used at once.  For each (b, h) and the query q[b, h, :]:
//     score_s = scale * sum_d q_d K[s, d],  p = softmax(score over s < L),  out_d = sum_s p_s V[s, d].
//
// One CTA per (b, h).  A position's row is D codes; D/8 lanes share it, each lane owning 8
// channels (its q values and the 8 channels' s and z stay in registers), so a warp reads
// 32/(D/8) rows per step, contiguous in the cache.  Pass 1 writes the L scores to shared memory
// (8-lane-group shuffles reduce a row's dot product), the CTA reduces their maximum and the sum
// of exp(score - max), and pass 2 accumulates p_s V_s per lane over its share of the positions,
// then across position slots and warps.
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace rptq {

constexpr int KVA_THREADS = 256;

// The 8 codes of channels 8*c8 .. 8*c8+7 of one packed row: 4-bit as one 32-bit word, 3-bit as
// the little-endian 24-bit group (three byte loads: a 3-bit row need not be word aligned).
template <int BITS>
__device__ __forceinline__ uint32_t codes8(const uint8_t *row, int c8)
{
    if constexpr (BITS == 4) {
        return __ldg(reinterpret_cast<const uint32_t *>(row) + c8);
    } else {
        const uint8_t *p = row + 3 * c8;
        return (uint32_t)__ldg(p) | ((uint32_t)__ldg(p + 1) << 8) | ((uint32_t)__ldg(p + 2) << 16);
    }
}

// sum over the lanes of one group of LPP consecutive lanes (LPP a power of two, <= 32)
__device__ __forceinline__ float group_sum(float v, int LPP)
{
    for (int o = LPP >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    return v;
}

template <int BITS>
__global__ void __launch_bounds__(KVA_THREADS)
    kv_attention_kernel(const float *__restrict__ q, int H, int D, const uint8_t *__restrict__ kq,
                        const uint8_t *__restrict__ vq, int64_t S_max, int L, const int32_t *__restrict__ ck,
                        const float *__restrict__ sk, const int32_t *__restrict__ zk, const int32_t *__restrict__ cv,
                        const float *__restrict__ sv, const int32_t *__restrict__ zv, int g, float scale,
                        float *__restrict__ out, int *err)
{
    constexpr uint32_t MASK = (1u << BITS) - 1u;
    extern __shared__ __align__(16) float p[];  // L scores, then the weights
    __shared__ float red[KVA_THREADS / 32];
    __shared__ float part[KVA_THREADS / 32][256];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = KVA_THREADS / 32;
    const int LPP = D / 8;                      // lanes per position row (a power of two)
    const int PPW = 32 / LPP;                   // rows per warp step
    const int slot = lane / LPP, c8 = lane % LPP;
    const int bh = blockIdx.x, h = bh % H;
    const int64_t pitch = (int64_t)D * BITS / 8;
    const uint8_t *krow0 = kq + (int64_t)bh * S_max * pitch;
    const uint8_t *vrow0 = vq + (int64_t)bh * S_max * pitch;

    // the lane's 8 channels: query values and the K and V quantization parameters
    float qv[8], ks[8], kzf[8], vs[8], vzf[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int d = c8 * 8 + j, c = h * D + d;
        qv[j] = q[(int64_t)bh * D + d];
        int a = ck[c], b = cv[c];
        if (a < 0 || a >= g || b < 0 || b >= g) {
            raise_error(err, RPTQ_DEVERR_CLUSTER_ID);
            a = a < 0 || a >= g ? 0 : a;
            b = b < 0 || b >= g ? 0 : b;
        }
        ks[j] = sk[a];
        kzf[j] = (float)zk[a];
        vs[j] = sv[b];
        vzf[j] = (float)zv[b];
    }

    // pass 1: scores.  (q - z) as a float is exact for |q - z| < 2^24, and s * (q - z) rounds
    // once, as rptq_dequant does; the dot product of a row: 8 fused multiply-adds per lane, then
    // the group's shuffle tree
    float mloc = -INFINITY;
    for (int s0 = warp * PPW; s0 < L; s0 += nwarps * PPW) {
        const int s = s0 + slot;
        float acc = 0.f;
        if (s < L) {
            const uint32_t w = codes8<BITS>(krow0 + (int64_t)s * pitch, c8);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float kval = ks[j] * ((float)((w >> (BITS * j)) & MASK) - kzf[j]);
                acc = fmaf(qv[j], kval, acc);
            }
        }
        acc = group_sum(acc, LPP) * scale;
        if (s < L && c8 == 0) {
            p[s] = acc;
            mloc = fmaxf(mloc, acc);
        }
    }
    // CTA maximum
    for (int o = 16; o > 0; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(FULL, mloc, o));
    if (lane == 0) red[warp] = mloc;
    __syncthreads();
    float mx = red[0];
    for (int w = 1; w < nwarps; ++w) mx = fmaxf(mx, red[w]);
    __syncthreads();  // red is reused below
    // exp(score - max) in place and its CTA sum
    float sl = 0.f;
    for (int s = tid; s < L; s += KVA_THREADS) {
        const float e = expf(p[s] - mx);
        p[s] = e;
        sl += e;
    }
    for (int o = 16; o > 0; o >>= 1) sl += __shfl_xor_sync(FULL, sl, o);
    if (lane == 0) red[warp] = sl;
    __syncthreads();
    float tot = 0.f;
    for (int w = 0; w < nwarps; ++w) tot += red[w];
    const float inv = 1.0f / tot;

    // pass 2: out_d = sum_s p_s V[s, d]: each lane over the positions of its slot
    float o8[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) o8[j] = 0.f;
    for (int s0 = warp * PPW; s0 < L; s0 += nwarps * PPW) {
        const int s = s0 + slot;
        if (s < L) {
            const uint32_t w = codes8<BITS>(vrow0 + (int64_t)s * pitch, c8);
            const float ps = p[s] * inv;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float vval = vs[j] * ((float)((w >> (BITS * j)) & MASK) - vzf[j]);
                o8[j] = fmaf(ps, vval, o8[j]);
            }
        }
    }
    // across the warp's position slots (lanes with the same c8), then across warps
#pragma unroll
    for (int j = 0; j < 8; ++j)
        for (int o = LPP; o < 32; o <<= 1) o8[j] += __shfl_xor_sync(FULL, o8[j], o);
    if (slot == 0) {
#pragma unroll
        for (int j = 0; j < 8; ++j) part[warp][c8 * 8 + j] = o8[j];
    }
    __syncthreads();
    for (int d = tid; d < D; d += KVA_THREADS) {
        float v = 0.f;
        for (int w = 0; w < nwarps; ++w) v += part[w][d];
        out[(int64_t)bh * D + d] = v;
    }
}

cudaError_t launch_kv_attention(const KvAttnArgs &a)
{
    if (a.B == 0) return cudaSuccess;
    const size_t smem = (size_t)a.L * sizeof(float);
    const float scale = a.scale > 0.f ? a.scale : 1.0f / sqrtf((float)a.D);
    auto kern = a.bits == 4 ? kv_attention_kernel<4> : kv_attention_kernel<3>;
    cudaError_t e = kernel_smem((const void *)kern, smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)((int64_t)a.B * a.H), KVA_THREADS, smem, a.stream>>>(
        a.q, a.H, a.D, a.kq, a.vq, a.S_max, (int)a.L, a.ck, a.sk, a.zk, a.cv, a.sv, a.zv, a.g, scale, a.out,
        a.err);
    return cudaGetLastError();
}

}  // namespace rptq
