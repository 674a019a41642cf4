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
// One CTA per (b, h).  A lane owns CPL consecutive channels of a row (32, or all D when D < 32)
// and reads their codes with one aligned vector load (12 bytes for 3-bit, 16 for 4-bit codes);
// D / CPL lanes share a row, so a warp covers 32 / (D / CPL) rows per step, contiguous in the
// cache.  A code becomes a float by OR-ing it into 2^23 (the float 2^23 + q), and
// (2^23 + q) - (2^23 + z) = q - z exactly, so the dequantized products cost two packed fp32
// operations per pair of codes:
//   score = scale * sum_d (q_d s_d) (q_sd - z_d)          (pass 1, per row; then softmax)
//   out_d = s_d * sum_s e_s (q_sd - z_d) / sum_s e_s      (pass 2, e_s = exp(score_s - max))
// (the products with s_d differ from rounding each dequantized value first by at most one
// rounding each; the bound the tests use includes it).
// Pass 1 writes the scores of the (b, h) to shared memory; the CTA reduces their maximum and
// the sum of the exponentials; pass 2 accumulates per lane over its share of the positions,
// then across the row slots of a warp and the warps.  At entry one bulk L2 prefetch per cache
// pulls the CTA's K and V rows (contiguous) towards the SM.
// Measured at batch 8 x 96 heads x 2048 positions, D = 128, 3-bit (152 MB of codes): 0.142 ms
// with KVA_UNROLL = 8 rows in flight per warp (0.148 ms with 4; 16 needs 180 registers and runs
// at 0.226 ms).  ncu: about 6 instructions per code, 42 % issue-active: neither issue nor HBM
// (12 % of its bandwidth) is the bound; fewer instructions per code (codes masked in place at
// their bit position) and four independent accumulators in pass 1 measured no faster, more
// loads in flight did.  Splitting the positions of a (b, h) over a thread-block cluster
// (combining max, sum and partial outputs through distributed shared memory) measured slower:
// 2 CTAs 0.174 ms, 4 CTAs 0.244 ms.
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace rptq {

constexpr int KVA_THREADS = 256;
constexpr int KVA_UNROLL = 8;  // row steps per warp iteration, their loads issued first
constexpr uint32_t KVA_MAGIC = 0x4B000000u;  // the float 2^23

// The codes of channels CPL*cc .. CPL*cc + CPL - 1 of a packed row, as the little-endian bit
// string w[0], w[1], ...
template <int BITS, int CPL>
struct RowCodes {
    static constexpr int NW = (CPL * BITS + 31) / 32;
    uint32_t w[NW];
    __device__ __forceinline__ void load(const uint8_t *row, int cc)
    {
        const uint8_t *p = row + cc * (CPL * BITS / 8);
        if constexpr (BITS == 4 && CPL == 32) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p));
            w[0] = v.x, w[1] = v.y, w[2] = v.z, w[3] = v.w;
        } else if constexpr (BITS == 4 && CPL == 16) {
            const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p));
            w[0] = v.x, w[1] = v.y;
        } else if constexpr (BITS == 4 || (BITS == 3 && CPL == 32)) {  // whole words
#pragma unroll
            for (int i = 0; i < NW; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t *>(p) + i);
        } else if constexpr (CPL == 16) {  // 3-bit, 6 bytes at an even offset
            const uint16_t *h = reinterpret_cast<const uint16_t *>(p);
            w[0] = (uint32_t)__ldg(h) | ((uint32_t)__ldg(h + 1) << 16);
            w[1] = (uint32_t)__ldg(h + 2);
        } else {  // 3-bit, 3 bytes
            w[0] = (uint32_t)__ldg(p) | ((uint32_t)__ldg(p + 1) << 8) | ((uint32_t)__ldg(p + 2) << 16);
        }
    }
    // code j as the float 2^23 + code
    __device__ __forceinline__ float f(int j) const
    {
        constexpr uint32_t MASK = (1u << BITS) - 1u;
        const int bit = BITS * j, i = bit >> 5, sh = bit & 31;
        uint32_t v;
        if (sh + BITS <= 32 || i + 1 >= NW)
            v = w[i] >> sh;
        else
            v = __funnelshift_r(w[i], w[i + 1], sh);
        return __uint_as_float((v & MASK) | KVA_MAGIC);
    }
};

template <int BITS, int CPL>
__global__ void __launch_bounds__(KVA_THREADS)
    kv_attention_kernel(const float *__restrict__ q, int H, int D, const uint8_t *__restrict__ kq,
                        const uint8_t *__restrict__ vq, int64_t S_max, int L, const int32_t *__restrict__ ck,
                        const float *__restrict__ sk, const int32_t *__restrict__ zk, const int32_t *__restrict__ cv,
                        const float *__restrict__ sv, const int32_t *__restrict__ zv, int g, float scale,
                        float *__restrict__ out, int *err)
{
    constexpr int NP = CPL / 2;  // pairs of channels per lane
    extern __shared__ __align__(16) float e[];  // the L scores, then exp(score - max)
    __shared__ float red[KVA_THREADS / 32];
    __shared__ float part[KVA_THREADS / 32][256];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = KVA_THREADS / 32;
    const int LPP = D / CPL;       // lanes per row
    const int RPW = 32 / LPP;      // rows per warp step
    const int slot = lane / LPP, cc = lane % LPP;
    const int bh = blockIdx.x, h = bh % H;
    const int n = L;
    const int64_t pitch = (int64_t)D * BITS / 8;
    const uint8_t *krow0 = kq + (int64_t)bh * S_max * pitch;
    const uint8_t *vrow0 = vq + (int64_t)bh * S_max * pitch;
    // the CTA's K and V rows are contiguous: one bulk L2 prefetch each, so that the row loads
    // below find them in L2 (whole 16-byte units inside the block)
    if (tid == 0 && n > 0) {
        const uint64_t kb = reinterpret_cast<uint64_t>(krow0), vb = reinterpret_cast<uint64_t>(vrow0);
        const uint64_t bytes = (uint64_t)n * pitch;
        const uint64_t k0 = (kb + 15) & ~15ull, k1 = (kb + bytes) & ~15ull;
        const uint64_t v0 = (vb + 15) & ~15ull, v1 = (vb + bytes) & ~15ull;
        if (k1 > k0) prefetch_l2(reinterpret_cast<const void *>(k0), (uint32_t)(k1 - k0));
        if (v1 > v0) prefetch_l2(reinterpret_cast<const void *>(v0), (uint32_t)(v1 - v0));
    }

    // pass 1 coefficients of the lane's channels: a_d = scale * q_d * s_d and -(2^23 + z_d)
    f32x2 a2[NP], nz2[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        float av[2], zv2[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int d = cc * CPL + 2 * i + t, c = h * D + d;
            int k = ck[c];
            if (k < 0 || k >= g) {
                raise_error(err, RPTQ_DEVERR_CLUSTER_ID);
                k = 0;
            }
            av[t] = q[(int64_t)bh * D + d] * sk[k] * scale;
            zv2[t] = -(8388608.0f + (float)zk[k]);
        }
        a2[i] = mk2(av[0], av[1]);
        nz2[i] = mk2(zv2[0], zv2[1]);
    }
    // KVA_UNROLL row steps per iteration: their loads are all issued before any arithmetic, so
    // a warp keeps several rows in flight
    const int step = nwarps * RPW;
    float mloc = -INFINITY;
    for (int s0 = warp * RPW; s0 < n; s0 += KVA_UNROLL * step) {
        RowCodes<BITS, CPL> rc[KVA_UNROLL];
#pragma unroll
        for (int u = 0; u < KVA_UNROLL; ++u) {
            const int s = s0 + u * step + slot;
            if (s < n) rc[u].load(krow0 + (int64_t)s * pitch, cc);
        }
#pragma unroll
        for (int u = 0; u < KVA_UNROLL; ++u) {
            const int s = s0 + u * step + slot;
            f32x2 acc = mk2(0.f, 0.f);
            if (s < n) {
#pragma unroll
                for (int i = 0; i < NP; ++i)
                    acc = fma2(a2[i], add2(mk2(rc[u].f(2 * i), rc[u].f(2 * i + 1)), nz2[i]), acc);
            }
            float sc = lo2(acc) + hi2(acc);
            for (int o = LPP >> 1; o > 0; o >>= 1) sc += __shfl_xor_sync(FULL, sc, o);
            if (s < n && cc == 0) {
                e[s] = sc;
                mloc = fmaxf(mloc, sc);
            }
        }
    }
    for (int o = 16; o > 0; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(FULL, mloc, o));
    if (lane == 0) red[warp] = mloc;
    __syncthreads();
    float mx = red[0];
    for (int w = 1; w < nwarps; ++w) mx = fmaxf(mx, red[w]);
    __syncthreads();  // red is reused below
    float sl = 0.f;
    for (int s = tid; s < n; s += KVA_THREADS) {
        const float ev = expf(e[s] - mx);
        e[s] = ev;
        sl += ev;
    }
    for (int o = 16; o > 0; o >>= 1) sl += __shfl_xor_sync(FULL, sl, o);
    if (lane == 0) red[warp] = sl;
    __syncthreads();
    float tot = 0.f;
    for (int w = 0; w < nwarps; ++w) tot += red[w];

    // pass 2: acc_d = sum_s e_s (q_sd - z_d) over the lane's positions
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        float zv2[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int c = h * D + cc * CPL + 2 * i + t;
            int k = cv[c];
            if (k < 0 || k >= g) {
                raise_error(err, RPTQ_DEVERR_CLUSTER_ID);
                k = 0;
            }
            zv2[t] = -(8388608.0f + (float)zv[k]);
        }
        nz2[i] = mk2(zv2[0], zv2[1]);
        a2[i] = mk2(0.f, 0.f);  // now the accumulators
    }
    for (int s0 = warp * RPW; s0 < n; s0 += KVA_UNROLL * step) {
        RowCodes<BITS, CPL> rc[KVA_UNROLL];
#pragma unroll
        for (int u = 0; u < KVA_UNROLL; ++u) {
            const int s = s0 + u * step + slot;
            if (s < n) rc[u].load(vrow0 + (int64_t)s * pitch, cc);
        }
#pragma unroll
        for (int u = 0; u < KVA_UNROLL; ++u) {
            const int s = s0 + u * step + slot;
            if (s < n) {
                const f32x2 p2 = mk2(e[s], e[s]);
#pragma unroll
                for (int i = 0; i < NP; ++i)
                    a2[i] = fma2(p2, add2(mk2(rc[u].f(2 * i), rc[u].f(2 * i + 1)), nz2[i]), a2[i]);
            }
        }
    }
    // across the warp's row slots (lanes with the same cc), then across warps
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        float x0 = lo2(a2[i]), x1 = hi2(a2[i]);
        for (int o = LPP; o < 32; o <<= 1) {
            x0 += __shfl_xor_sync(FULL, x0, o);
            x1 += __shfl_xor_sync(FULL, x1, o);
        }
        if (slot == 0) {
            part[warp][cc * CPL + 2 * i] = x0;
            part[warp][cc * CPL + 2 * i + 1] = x1;
        }
    }
    __syncthreads();
    const float inv = 1.0f / tot;
    for (int d = tid; d < D; d += KVA_THREADS) {
        float v = 0.f;
        for (int w = 0; w < nwarps; ++w) v += part[w][d];
        int k = cv[h * D + d];
        k = (k < 0 || k >= g) ? 0 : k;
        out[(int64_t)bh * D + d] = sv[k] * v * inv;
    }
}

cudaError_t launch_kv_attention(const KvAttnArgs &a)
{
    if (a.B == 0) return cudaSuccess;
    const size_t smem = (size_t)a.L * sizeof(float);
    const float scale = a.scale > 0.f ? a.scale : 1.0f / sqrtf((float)a.D);
    auto pick = [&](auto k3, auto k4) { return a.bits == 4 ? k4 : k3; };
    const void *kern = a.D >= 32 ? (const void *)pick(kv_attention_kernel<3, 32>, kv_attention_kernel<4, 32>)
                       : a.D == 16 ? (const void *)pick(kv_attention_kernel<3, 16>, kv_attention_kernel<4, 16>)
                                   : (const void *)pick(kv_attention_kernel<3, 8>, kv_attention_kernel<4, 8>);
    cudaError_t e = kernel_smem(kern, smem);
    if (e != cudaSuccess) return e;
    int L = (int)a.L;
    void *args[] = {(void *)&a.q, (void *)&a.H, (void *)&a.D, (void *)&a.kq, (void *)&a.vq, (void *)&a.S_max,
                    (void *)&L, (void *)&a.ck, (void *)&a.sk, (void *)&a.zk, (void *)&a.cv, (void *)&a.sv,
                    (void *)&a.zv, (void *)&a.g, (void *)&scale, (void *)&a.out, (void *)&a.err};
    return cudaLaunchKernel(kern, dim3((unsigned)((int64_t)a.B * a.H)), dim3(KVA_THREADS), args, smem, a.stream);
}

}  // namespace rptq
