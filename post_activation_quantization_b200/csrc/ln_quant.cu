// ln_quant.cu -- reorder-fused LayerNorm + per-cluster asymmetric quantization.
//
// RPTQ article (基于重排序的新量化方法RPTQ…), text after Fig. 3: the LayerNorm is changed so
// that it emits activations already in cluster order, so no reordered copy of the activation
// tensor is ever stored; text after Fig. 2: one scale s and zero point z per cluster.
// Quantization-basics article, sections 1.1 (static range, clamp) and 1.3 (q = round(y/s)+z).
//
// Fast kernel (codes only, C % 32 == 0): see row_pipeline.cuh for the row staging.  When shared
// memory cannot hold eight ring rows next to a separate code buffer (large C), the code buffer of
// a quad lives in that quad's own four ring slots, which are free once the rows sit in registers;
// they are refilled after the pack, and the eight-row ring still keeps a whole quad in flight.
// Per quad
// of four tokens a thread holds its chunks of x in registers, computes the LayerNorm
// statistics, and for each of its channels c turns the four tokens' values into four codes
//     u = sat(((x - mean) * rstd) * A_c + B_c),  code = rint(u * qmax)
// with A_c = gamma_c / (s_k * qmax), B_c = (beta_c / s_k + z_k) / qmax, k the cluster of c
// (this is clamp(rint(y/s_k) + z_k, 0, qmax) with y the LayerNorm output, in fp32).  The four
// codes form one 32-bit word that is stored at the channel's STORED position R^-1(c) in a
// shared code buffer: the reorder happens in that single shared-memory store, and because the
// word carries four tokens a random position costs a quarter of a byte-wise scatter.  After a
// barrier each thread reads 32 consecutive stored positions (4 tokens each), packs them into
// 3- or 4-bit codes in registers and writes whole words of the packed rows.
//
// Simple kernel (any C % 8 == 0, dense LayerNorm output and/or codes): one CTA per token row,
// the row in shared memory as fp32, a two-pass LayerNorm, a gather through R per stored
// column, the quantizer written as clamp(rint(y / s) + z) with an IEEE divide.
#include <algorithm>

#include "launch.h"
#include "row_pipeline.cuh"

namespace rptq {

// ------------------------------------------------------------------------------------------
// Pieces shared by the two fast kernels.

// Per-channel tables: postab[c] = code-buffer offset of channel c's stored column, and the
// thread's affine coefficients pA, pB for its chunks (tid + k*NT).
template <typename T, int BITS, int CPT, typename P>
__device__ __forceinline__ void quant_tables(const int32_t *R, const int32_t *col_cluster, const float *scale,
                                             const int32_t *zero, const float *gamma, const float *beta, int g, int C,
                                             P *postab, uint32_t pbase, float (&pA)[CPT][Elem<T>::VEC],
                                             float (&pB)[CPT][Elem<T>::VEC], int *err)
{
    // postab[c] = pbase + code-buffer offset of channel c's stored column (P = uint16_t: the
    // offset alone; P = uint32_t: the shared-memory address of the word)
    constexpr int VEC = Elem<T>::VEC;
    constexpr float QMAX = (float)((1 << BITS) - 1);
    const int tid = threadIdx.x, NT = blockDim.x, NCH = C / VEC;
    for (int c = tid; c < C; c += NT) postab[c] = (P)pbase;
    __syncthreads();
    for (int j = tid; j < C; j += NT) {
        const int c = R[j];
        if (c >= 0 && c < C)
            postab[c] = (P)(pbase + codebuf_offset((uint32_t)j));
        else
            raise_error(err, RPTQ_DEVERR_REORDER);
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < CPT; ++k) {
        const int ch = tid + k * NT;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            pA[k][e] = 0.f;
            pB[k][e] = 0.f;
            if (ch < NCH) {
                const int c = ch * VEC + e;
                const int j = (int)codebuf_index((uint32_t)postab[c] - pbase);
                int kc = col_cluster[j];
                if (kc < 0 || kc >= g) {
                    raise_error(err, RPTQ_DEVERR_CLUSTER_ID);
                    kc = 0;
                }
                const double s = (double)scale[kc];
                pA[k][e] = (float)((double)gamma[c] / (s * (double)QMAX));
                pB[k][e] = (float)(((double)beta[c] / s + (double)zero[kc]) / (double)QMAX);
            }
        }
    }
}

// The same tables for the direct kernel, built with coalesced loads: one pass over the stored
// columns j (R and col_cluster read as int4) records each channel's code-buffer address and
// cluster; a per-cluster table holds 1 / (s qmax) and z / qmax in fp64, so a channel's
// coefficients are one multiply and one fused multiply-add (A = gamma / (s qmax),
// B = beta / (s qmax) + z / qmax).  Needs C % 4 == 0 and 16-byte aligned R, col_cluster,
// gamma and beta.
template <typename T, int BITS, int CPT>
__device__ __forceinline__ void quant_tables_direct(const int32_t *R, const int32_t *col_cluster, const float *scale,
                                                    const int32_t *zero, const float *gamma, const float *beta,
                                                    int g, int C, uint32_t *postab, uint16_t *ctab, double *ctl,
                                                    uint32_t pbase, float (&pA)[CPT][Elem<T>::VEC],
                                                    float (&pB)[CPT][Elem<T>::VEC], int *err)
{
    constexpr int VEC = Elem<T>::VEC;
    constexpr double QMAX = (double)((1 << BITS) - 1);
    // every thread's share of R and col_cluster (int4 j4 = tid + u*NT; NT*CPT chunks cover the
    // row, so NR int4 per thread suffice) is loaded first; thread 0 also pulls gamma and beta
    // into L2 for the loads after the scatter
    constexpr int NR = CPT * VEC / 4;
    const int tid = threadIdx.x, NT = blockDim.x, NCH = C / VEC, C4 = C / 4;
    if (tid == 0) {
        prefetch_l2(gamma, (uint32_t)C * 4u);
        prefetch_l2(beta, (uint32_t)C * 4u);
    }
    const int4 *R4 = reinterpret_cast<const int4 *>(R);
    const int4 *K4 = reinterpret_cast<const int4 *>(col_cluster);
    int4 r[NR], kk[NR];
#pragma unroll
    for (int u = 0; u < NR; ++u) {
        const int j4 = tid + u * NT;
        r[u] = j4 < C4 ? R4[j4] : make_int4(-1, -1, -1, -1);
        kk[u] = j4 < C4 ? K4[j4] : make_int4(0, 0, 0, 0);
    }
    for (int c = tid; c < C; c += NT) {
        postab[c] = pbase;
        ctab[c] = 0;
    }
    for (int k = tid; k < g; k += NT) {
        const double s = (double)scale[k] * QMAX;
        ctl[2 * k] = 1.0 / s;
        ctl[2 * k + 1] = (double)zero[k] / QMAX;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < NR; ++u) {
        const int j4 = tid + u * NT;
        if (j4 >= C4) continue;
        const int rv[4] = {r[u].x, r[u].y, r[u].z, r[u].w}, kv[4] = {kk[u].x, kk[u].y, kk[u].z, kk[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int c = rv[i], k = kv[i];
            if (c >= 0 && c < C) {
                postab[c] = pbase + codebuf_offset((uint32_t)(4 * j4 + i));
                ctab[c] = (uint16_t)((k >= 0 && k < g) ? k : 0);
            } else {
                raise_error(err, RPTQ_DEVERR_REORDER);
            }
            if (k < 0 || k >= g) raise_error(err, RPTQ_DEVERR_CLUSTER_ID);
        }
    }
    __syncthreads();
    // gamma, beta of the thread's chunks as 16-byte loads, all in flight before the arithmetic
    float4 gm[CPT][VEC / 4], bt[CPT][VEC / 4];
#pragma unroll
    for (int kc = 0; kc < CPT; ++kc) {
        const int ch = tid + kc * NT;
#pragma unroll
        for (int q = 0; q < VEC / 4; ++q) {
            gm[kc][q] = ch < NCH ? __ldg(reinterpret_cast<const float4 *>(gamma + ch * VEC) + q) : make_float4(0, 0, 0, 0);
            bt[kc][q] = ch < NCH ? __ldg(reinterpret_cast<const float4 *>(beta + ch * VEC) + q) : make_float4(0, 0, 0, 0);
        }
    }
#pragma unroll
    for (int kc = 0; kc < CPT; ++kc) {
        const int ch = tid + kc * NT;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            const float4 g4 = gm[kc][e / 4], b4 = bt[kc][e / 4];
            const float gv = (e & 3) == 0 ? g4.x : (e & 3) == 1 ? g4.y : (e & 3) == 2 ? g4.z : g4.w;
            const float bv = (e & 3) == 0 ? b4.x : (e & 3) == 1 ? b4.y : (e & 3) == 2 ? b4.z : b4.w;
            pA[kc][e] = 0.f;
            pB[kc][e] = 0.f;
            if (ch < NCH) {
                const int k = ctab[ch * VEC + e];
                const double inv = ctl[2 * k];
                pA[kc][e] = (float)((double)gv * inv);
                pB[kc][e] = (float)fma((double)bv, inv, ctl[2 * k + 1]);
            }
        }
    }
}

// The same per-thread state from a plan written by ln_quant_plan_kernel (one entry per channel:
// code-buffer offset, A, B; computed once per calibration, which is the offline LayerNorm
// rewrite): each thread reads only its own channels' entries, coalesced 16-byte loads, and
// keeps its offsets in its own slots of the shared position table.  An offset is clamped into the
// code buffer and 4-byte aligned, so even a damaged plan cannot store outside it.
template <typename T, int CPT>
__device__ __forceinline__ void load_plan(const void *plan, int C, int NCH, int NT, uint32_t *postab, uint32_t pbase,
                                          float (&pA)[CPT][Elem<T>::VEC], float (&pB)[CPT][Elem<T>::VEC])
{
    constexpr int VEC = Elem<T>::VEC, V4 = VEC / 4;
    const uint4 *P = static_cast<const uint4 *>(plan);
    const float4 *PA = reinterpret_cast<const float4 *>(static_cast<const uint32_t *>(plan) + C);
    const float4 *PB = PA + C / 4;
    const uint32_t lim = 4u * (uint32_t)C - 4u;
    const int tid = threadIdx.x;
#pragma unroll
    for (int kc = 0; kc < CPT; ++kc) {
        const int ch = tid + kc * NT;
#pragma unroll
        for (int q = 0; q < V4; ++q) {
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
            if (ch < NCH) {
                uint4 pp = __ldg(P + ch * V4 + q);
                pp.x = pbase + (min(pp.x, lim) & ~3u);
                pp.y = pbase + (min(pp.y, lim) & ~3u);
                pp.z = pbase + (min(pp.z, lim) & ~3u);
                pp.w = pbase + (min(pp.w, lim) & ~3u);
                reinterpret_cast<uint4 *>(postab)[ch * V4 + q] = pp;
                a = __ldg(PA + ch * V4 + q);
                b = __ldg(PB + ch * V4 + q);
            }
            pA[kc][4 * q + 0] = a.x, pA[kc][4 * q + 1] = a.y, pA[kc][4 * q + 2] = a.z, pA[kc][4 * q + 3] = a.w;
            pB[kc][4 * q + 0] = b.x, pB[kc][4 * q + 1] = b.y, pB[kc][4 * q + 2] = b.z, pB[kc][4 * q + 3] = b.w;
        }
    }
}

// The plan: for every stored column j, channel c = R[j] of cluster k = col_cluster[j] gets
// offset codebuf_offset(j), A = gamma_c / (s_k qmax) and B = beta_c / (s_k qmax) + z_k / qmax,
// with the fp64 arithmetic of quant_tables_direct (so both paths give the same coefficients).
// The plan is zeroed first; an R entry outside [0, C) is skipped, a cluster id outside [0, g)
// uses cluster 0; both set the error word.
template <int BITS>
__global__ void __launch_bounds__(256)
    ln_quant_plan_kernel(const float *__restrict__ gamma, const float *__restrict__ beta, const int32_t *__restrict__ R,
                         const int32_t *__restrict__ col_cluster, const float *__restrict__ scale,
                         const int32_t *__restrict__ zero, int C, int g, uint32_t *__restrict__ pos,
                         float *__restrict__ A, float *__restrict__ B, int *err)
{
    constexpr double QMAX = (double)((1 << BITS) - 1);
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < C; j += gridDim.x * blockDim.x) {
        const int c = R[j];
        int k = col_cluster[j];
        if (k < 0 || k >= g) {
            raise_error(err, RPTQ_DEVERR_CLUSTER_ID);
            k = 0;
        }
        if (c < 0 || c >= C) {
            raise_error(err, RPTQ_DEVERR_REORDER);
            continue;
        }
        const double inv = 1.0 / ((double)scale[k] * QMAX);
        pos[c] = codebuf_offset((uint32_t)j);
        A[c] = (float)((double)gamma[c] * inv);
        B[c] = (float)fma((double)beta[c], inv, (double)zero[k] / QMAX);
    }
}

// Codes of the quad's four tokens for every channel of the thread -> one word per channel at
// its stored position in the code buffer.  The normalised value of x is fmaf(x - sub[r], rstd[r],
// nmr[r]) (sub = 0 except for rows with a large offset, see quad_stats); x - sub is formed by the
// widening mixed-precision add, so both kinds of row share this code and cost no extra
// instruction.  NT_: the CTA's thread count when known at compile time (0: blockDim.x).
template <typename T, int BITS, int CPT, bool ABS>
__device__ __forceinline__ void quant_scatter(const uint4 (&xr)[4][CPT], const float (&rstd)[4], const float (&nmr)[4],
                                              const float (&sub)[4],
                                              const float (&pA)[CPT][Elem<T>::VEC],
                                              const float (&pB)[CPT][Elem<T>::VEC], const void *postab,
                                              uint8_t *codebuf, int NCH, uint32_t boff = 0, int NT_ = 0)
{
    // ABS: postab holds 32-bit shared-memory addresses (stored directly, no extraction);
    // otherwise 16-bit offsets into codebuf, two per word
    constexpr int VEC = Elem<T>::VEC;
    constexpr float QMAX = (float)((1 << BITS) - 1);
    const int tid = threadIdx.x, NT = NT_ ? NT_ : (int)blockDim.x;
    const f32x2 rs01 = mk2(rstd[0], rstd[1]), rs23 = mk2(rstd[2], rstd[3]);
    const f32x2 nm01 = mk2(nmr[0], nmr[1]), nm23 = mk2(nmr[2], nmr[3]);
    const float ms[4] = {-sub[0], -sub[1], -sub[2], -sub[3]};
    const f32x2 qm2 = mk2(QMAX, QMAX), mg2 = mk2(MAGIC_RINT, MAGIC_RINT);
#pragma unroll
    for (int k = 0; k < CPT; ++k) {
        const int ch = tid + k * NT;
        if (ch >= NCH) continue;
        uint32_t pw[ABS ? VEC : VEC / 2];
        if constexpr (ABS) {
            const uint4 *p4 = reinterpret_cast<const uint4 *>(static_cast<const uint32_t *>(postab) + ch * VEC);
#pragma unroll
            for (int i = 0; i < VEC / 4; ++i) {
                const uint4 p = p4[i];
                pw[4 * i] = p.x, pw[4 * i + 1] = p.y, pw[4 * i + 2] = p.z, pw[4 * i + 3] = p.w;
            }
        } else if constexpr (VEC == 8) {
            const uint4 p = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(postab) + ch * 8);
            pw[0] = p.x, pw[1] = p.y, pw[2] = p.z, pw[3] = p.w;
        } else {
            const uint2 p = *reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(postab) + ch * 4);
            pw[0] = p.x, pw[1] = p.y;
        }
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            // normalised values of channel e for tokens (0,1) and (2,3), two lanes at a time
            const f32x2 x01 = mk2(elem_plus<T>(xr[0][k], e, ms[0]), elem_plus<T>(xr[1][k], e, ms[1]));
            const f32x2 x23 = mk2(elem_plus<T>(xr[2][k], e, ms[2]), elem_plus<T>(xr[3][k], e, ms[3]));
            const f32x2 t01 = fma2(x01, rs01, nm01);
            const f32x2 t23 = fma2(x23, rs23, nm23);
            const float A = pA[k][e], Bc = pB[k][e];
            // u = sat(y / (s qmax) + z / qmax); code = rint(u qmax) (the 1.5*2^23 rounding add)
            const f32x2 u01 = mk2(fma_sat(lo2(t01), A, Bc), fma_sat(hi2(t01), A, Bc));
            const f32x2 u23 = mk2(fma_sat(lo2(t23), A, Bc), fma_sat(hi2(t23), A, Bc));
            const f32x2 b01 = fma2(u01, qm2, mg2), b23 = fma2(u23, qm2, mg2);
            const uint32_t word = prmt(prmt(__float_as_uint(lo2(b01)), __float_as_uint(hi2(b01)), 0x0040),
                                       prmt(__float_as_uint(lo2(b23)), __float_as_uint(hi2(b23)), 0x0040), 0x5410);
            if constexpr (ABS) {
                asm volatile("st.shared.b32 [%0], %1;" ::"r"(pw[e] + boff), "r"(word) : "memory");
            } else {
                const uint32_t pos = (e & 1) ? (pw[e >> 1] >> 16) : (pw[e >> 1] & 0xffffu);
                *reinterpret_cast<uint32_t *>(codebuf + pos) = word;
            }
        }
    }
}

// Pack 32 stored positions x 4 tokens per thread from the code buffer and write whole words of
// rows 4*gq .. 4*gq + nrows - 1.
template <int BITS>
__device__ __forceinline__ void pack_store(const uint8_t *codebuf, uint8_t *codes, int64_t gq, int64_t pitch, int nrows,
                                           int NU, int NT_ = 0)
{
    const int NT = NT_ ? NT_ : (int)blockDim.x;
    for (int u = threadIdx.x; u < NU; u += NT) {
        uint32_t o[4][4];  // [group m of 8 positions][token r]
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            uint32_t w[8];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t slot = 8u * u + ((2 * m + h) ^ (u & 7));
                const uint4 q = *reinterpret_cast<const uint4 *>(codebuf + (slot << 4));
                w[4 * h + 0] = q.x;
                w[4 * h + 1] = q.y;
                w[4 * h + 2] = q.z;
                w[4 * h + 3] = q.w;
            }
            if constexpr (BITS == 4)
                pack8x4_a4(w, o[m]);
            else
                pack8x4_a3(w, o[m]);
        }
        uint8_t *dst = codes + 4 * gq * pitch + (BITS == 4 ? 16 : 12) * (int64_t)u;
#pragma unroll
        for (int r = 0; r < 4; ++r, dst += pitch) {
            if (r >= nrows) break;
            if constexpr (BITS == 4) {
                *reinterpret_cast<uint4 *>(dst) = make_uint4(o[0][r], o[1][r], o[2][r], o[3][r]);
            } else {
                uint32_t *d32 = reinterpret_cast<uint32_t *>(dst);
                d32[0] = o[0][r] | (o[1][r] << 24);
                d32[1] = (o[1][r] >> 8) | (o[2][r] << 16);
                d32[2] = (o[2][r] >> 16) | (o[3][r] << 8);
            }
        }
    }
}

// ------------------------------------------------------------------------------------------
// Fast kernel, rows staged through the shared-memory ring (row_pipeline.cuh).
template <typename T, int BITS, int CPT>
__global__ void __launch_bounds__(512, 1)
    ln_quant_fast_kernel(const T *__restrict__ x, int64_t T_, int C, const float *__restrict__ gamma,
                         const float *__restrict__ beta, float eps, const int32_t *__restrict__ R,
                         const int32_t *__restrict__ col_cluster, const float *__restrict__ scale,
                         const int32_t *__restrict__ zero, int g, uint8_t *__restrict__ codes, int NS,
                         int alias, int *err)
{
    constexpr int VEC = Elem<T>::VEC;
    extern __shared__ __align__(128) uint8_t smem[];
    const int NCH = C / VEC;
    const uint32_t rowbytes = (uint32_t)C * sizeof(T);
    const size_t cb_bytes = alias ? 0 : (size_t)C * 4;
    const QuadSmem L = quad_smem_layout(NS, rowbytes, cb_bytes + (size_t)C * 2 + 2 * 8 * 32 * 4);
    uint8_t *codebuf = smem + L.extra_off;                                    // 4*C bytes (own)
    uint16_t *postab = reinterpret_cast<uint16_t *>(smem + L.extra_off + cb_bytes);  // 2*C bytes
    float *red = reinterpret_cast<float *>(postab + C);                      // 8*32 floats
    float *red2 = red + 8 * 32;

    __shared__ int s_abort;
    QuadRows<T, CPT> pipe{x, T_, C, NCH, NS, rowbytes, smem, smem_u32(smem + L.bar_off), err, &s_abort};
    pipe.start();
    float pA[CPT][VEC], pB[CPT][VEC];
    quant_tables<T, BITS, CPT>(R, col_cluster, scale, zero, gamma, beta, g, C, postab, 0u, pA, pB, err);

    const int64_t pitch = (int64_t)C * BITS / 8;
    const int NU = C >> 5;  // 32-position pack units
    int64_t lq = 0;
    for (int64_t gq = blockIdx.x; 4 * gq < T_; gq += gridDim.x, ++lq) {
        const int nrows = (int)(T_ - 4 * gq < 4 ? T_ - 4 * gq : 4);
        uint4 xr[4][CPT];
        pipe.load(nrows, xr);
        float rstd[4], nmr[4], sub[4];
        quad_stats<T, CPT>(xr, C, NCH, eps, red, red2, pipe, lq, rstd, nmr, sub, !alias);
        if (pipe.aborted()) {  // a row never arrived (the error word is set): stop, no refill
            pipe.drain(lq);
            return;
        }
        if (alias) codebuf = smem + (size_t)pipe.slot * rowbytes;  // this quad's slots
        quant_scatter<T, BITS, CPT, false>(xr, rstd, nmr, sub, pA, pB, postab, codebuf, NCH);
        __syncthreads();
        pack_store<BITS>(codebuf, codes, gq, pitch, nrows, NU);
        if (alias) {  // the quad's slots held its codes until now
            __syncthreads();
            pipe.refill(lq);
        }
        pipe.advance();
    }
}

// Direct kernel: rows go from global memory straight to registers (coalesced 16-byte loads),
// with the DRAM stream kept ahead by bulk L2 prefetches of whole quads (four contiguous rows,
// one instruction, two quads ahead); the next quad's loads are issued as soon as the current
// quad's rows are dead (after the scatter), so they fly during the pack.  Shared memory holds
// only the code buffer and the tables (the stored positions as 32-bit shared addresses).
struct NoRefill {
    __device__ __forceinline__ void refill(int64_t) const {}
};

template <typename T, int CPT>
__device__ __forceinline__ void load_quad_direct(const T *x, int64_t T_, int C, int64_t gq, bool exact,
                                                 uint4 (&xr)[4][CPT], int NT_ = 0)
{
    constexpr int VEC = Elem<T>::VEC;
    const int tid = threadIdx.x, NT = NT_ ? NT_ : (int)blockDim.x, NCH = C / VEC;
    const T *src = x + 4 * gq * (int64_t)C + tid * VEC;
    if (exact && 4 * gq + 4 <= T_) {  // a full quad and every chunk inside the row: no predicates
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int k = 0; k < CPT; ++k) xr[r][k] = ldg_stream(src + (int64_t)r * C + k * NT * VEC);
        return;
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int64_t row = 4 * gq + r;
#pragma unroll
        for (int k = 0; k < CPT; ++k) {
            const int ch = tid + k * NT;
            xr[r][k] = (row < T_ && ch < NCH) ? ldg_stream(src + (int64_t)r * C + k * NT * VEC) : make_uint4(0, 0, 0, 0);
        }
    }
}

__device__ __forceinline__ void prefetch_quad_l2(const void *x, int64_t T_, uint32_t rowbytes, int64_t gq)
{
    if (threadIdx.x == 0 && 4 * gq < T_) {
        const int64_t n = (T_ - 4 * gq < 4 ? T_ - 4 * gq : 4) * (int64_t)rowbytes;
        prefetch_l2(static_cast<const uint8_t *>(x) + 4 * gq * (int64_t)rowbytes, (uint32_t)n);
    }
}

// code buffer 4C | positions 4C | reductions 2 KB | cluster table 16 g | channel clusters 2C
__host__ __device__ inline size_t direct_smem_bytes(int C, int g)
{
    return (size_t)C * 10 + 2 * 8 * 32 * 4 + (size_t)g * 16;
}
// DB: the second code buffer (4C) after the tables, at a 16-byte boundary
__host__ __device__ inline size_t direct_db_off(int C, int g) { return (direct_smem_bytes(C, g) + 15) & ~(size_t)15; }

// MAXT bounds the threads per CTA and so the registers per thread: 512 (128 registers) or 384
// (168 registers, for 4 chunks per thread, or 3 chunks when 384 threads cover the row).
// DB: two code buffers used in turn, so a quad's pack runs after the NEXT quad's statistics
// barrier (which already orders every thread's scatter before it) and one CTA barrier per quad
// remains: stats(q) [barrier] -> scatter(q) into buffer q%2 -> loads of q+1 -> pack(q-1) from
// buffer (q-1)%2.  The scatter of q+1 rewrites buffer (q-1)%2 only after the barrier of q+1,
// which every thread reaches after its pack(q-1).
// CC: the channel count fixed at compile time (0: the runtime argument).  With it the thread
// count (CC / VEC / CPT, the exact split) and every loop bound, row pitch and load offset are
// constants, which removes most of the per-quad address, bound and branch instructions; the
// launcher instantiates it for the common hidden sizes.
// PLAN: the per-channel offsets and coefficients come from a plan (load_plan) instead of being
// built by every CTA from R, col_cluster, s, z, gamma and beta (quant_tables_direct).
template <typename T, int BITS, int CPT, int MAXT, bool DB, bool PLAN, int CC = 0>
__global__ void __launch_bounds__(MAXT, 1)
    ln_quant_direct_kernel(const T *__restrict__ x, int64_t T_, int C_, const float *__restrict__ gamma,
                           const float *__restrict__ beta, float eps, const int32_t *__restrict__ R,
                           const int32_t *__restrict__ col_cluster, const float *__restrict__ scale,
                           const int32_t *__restrict__ zero, int g, uint8_t *__restrict__ codes,
                           const void *__restrict__ plan, int *err)
{
    constexpr int VEC = Elem<T>::VEC;
    extern __shared__ __align__(128) uint8_t smem[];
    const int C = CC ? CC : C_;
    const int NT = CC ? CC / VEC / CPT : (int)blockDim.x;
    const int NCH = C / VEC;
    const uint32_t rowbytes = (uint32_t)C * sizeof(T);
    uint8_t *codebuf = smem;                                                    // 4*C bytes
    uint32_t *postab = reinterpret_cast<uint32_t *>(smem + (size_t)C * 4);     // 4*C bytes
    float *red = reinterpret_cast<float *>(postab + C);                        // 8*32 floats
    float *red2 = red + 8 * 32;
    double *ctl = reinterpret_cast<double *>(red2 + 8 * 32);                   // 2*g doubles
    uint16_t *ctab = reinterpret_cast<uint16_t *>(ctl + 2 * g);                // C u16
    const int64_t G = gridDim.x;
    const bool exact = NCH == CPT * NT;  // the chunks split evenly over the threads
    float pA[CPT][VEC], pB[CPT][VEC];
    uint4 xr[4][CPT];
    prefetch_quad_l2(x, T_, rowbytes, blockIdx.x);
    if constexpr (PLAN) {
        // The first quads of all CTAs have DRAM to themselves while the plan loads; the second
        // quads are asked for only after: with both prefetched at once the first quad of the
        // last CTAs arrived later (measured at C = 9216: 72.4 -> 70.3 us).
        load_plan<T, CPT>(plan, C, NCH, NT, postab, smem_u32(codebuf), pA, pB);
        load_quad_direct<T, CPT>(x, T_, C, blockIdx.x, exact, xr, NT);
        prefetch_quad_l2(x, T_, rowbytes, blockIdx.x + G);
    } else {
        prefetch_quad_l2(x, T_, rowbytes, blockIdx.x + G);
        quant_tables_direct<T, BITS, CPT>(R, col_cluster, scale, zero, gamma, beta, g, C, postab, ctab, ctl,
                                          smem_u32(codebuf), pA, pB, err);
        load_quad_direct<T, CPT>(x, T_, C, blockIdx.x, exact, xr, NT);  // the L2 prefetch above is in flight
    }

    const int64_t pitch = (int64_t)C * BITS / 8;
    const int NU = C >> 5;
    const NoRefill none;
    uint8_t *codebuf1 = smem + direct_db_off(C, g);  // DB only
    const uint32_t boff = smem_u32(codebuf1) - smem_u32(codebuf);
    int64_t pgq = -1;  // DB: the quad whose codes wait in the other buffer
    int prows = 0, it = 0;
    for (int64_t gq = blockIdx.x; 4 * gq < T_; gq += G) {
        const int nrows = (int)(T_ - 4 * gq < 4 ? T_ - 4 * gq : 4);
        float rstd[4], nmr[4], sub[4];
        const uint32_t off = (DB && (it & 1)) ? boff : 0u;
        quad_stats<T, CPT>(xr, C, NCH, eps, red, red2, none, 0, rstd, nmr, sub, false, NT);
        quant_scatter<T, BITS, CPT, true>(xr, rstd, nmr, sub, pA, pB, postab, codebuf, NCH, off, NT);
        // the rows are dead: next quad's loads fly during the pack, and one more quad to L2
        load_quad_direct<T, CPT>(x, T_, C, gq + G, exact, xr, NT);
        prefetch_quad_l2(x, T_, rowbytes, gq + 2 * G);
        if constexpr (DB) {
            if (pgq >= 0) pack_store<BITS>((it & 1) ? codebuf : codebuf1, codes, pgq, pitch, prows, NU, NT);
            pgq = gq;
            prows = nrows;
            ++it;
        } else {
            __syncthreads();
            pack_store<BITS>(codebuf, codes, gq, pitch, nrows, NU, NT);
            // the next quad's scatter overwrites the code buffer only after the barrier inside
            // its LayerNorm statistics, which every thread reaches after this pack
        }
    }
    if (DB && pgq >= 0) {  // the last quad (number it - 1) and its buffer
        __syncthreads();
        pack_store<BITS>((it & 1) ? codebuf : codebuf1, codes, pgq, pitch, prows, NU, NT);
    }
}

// ------------------------------------------------------------------------------------------
template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v)
{
    return __bfloat162float(v);
}
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v)
{
    return __float2bfloat16_rn(v);
}

template <typename T>
__global__ void __launch_bounds__(256)
    ln_quant_simple_kernel(const T *__restrict__ x, int64_t T_, int C, const float *__restrict__ gamma,
                           const float *__restrict__ beta, float eps, const int32_t *__restrict__ R,
                           const int32_t *__restrict__ col_cluster, const float *__restrict__ scale,
                           const int32_t *__restrict__ zero, int g, int bits, uint8_t *__restrict__ codes,
                           T *__restrict__ ln_out, int *err)
{
    extern __shared__ __align__(16) uint8_t smem[];
    float *xs = reinterpret_cast<float *>(smem);              // C floats
    uint8_t *qb = smem + (size_t)C * 4;                        // C bytes
    __shared__ float red[8 * 8];
    const int tid = threadIdx.x, NT = blockDim.x;
    const int qmax = (1 << bits) - 1;
    const int64_t pitch = (int64_t)C * bits / 8;
    for (int64_t t = blockIdx.x; t < T_; t += gridDim.x) {
        const T *xr = x + t * (int64_t)C;
        float s = 0.f;
        for (int c = tid; c < C; c += NT) {
            const float v = to_f32<T>(xr[c]);
            xs[c] = v;
            s += v;
        }
        float v8[8] = {s, 0, 0, 0, 0, 0, 0, 0};
        cta_sum8(v8, red);
        float hi, rstd, nmr;
        row_moments(xs, C, v8[0], eps, red, hi, rstd, nmr);
        for (int j = tid; j < C; j += NT) {
            int c = R[j];
            if (c < 0 || c >= C) {
                raise_error(err, RPTQ_DEVERR_REORDER);
                c = 0;
            }
            int k = col_cluster[j];
            if (k < 0 || k >= g) {
                raise_error(err, RPTQ_DEVERR_CLUSTER_ID);
                k = 0;
            }
            const float y = fmaf(fmaf(xs[c] - hi, rstd, nmr), gamma[c], beta[c]);
            if (ln_out) ln_out[t * (int64_t)C + j] = from_f32<T>(y);
            if (codes) {
                const float q = rintf(__fdiv_rn(y, scale[k])) + (float)zero[k];
                qb[j] = (uint8_t)fminf(fmaxf(q, 0.f), (float)qmax);
            }
        }
        __syncthreads();
        if (codes) {
            uint8_t *dst = codes + t * pitch;
            for (int grp = tid; grp < C / 8; grp += NT) {
                const uint8_t *q = qb + 8 * grp;
                if (bits == 4) {
                    uint32_t wv = 0;
                    for (int i = 0; i < 8; ++i) wv |= (uint32_t)(q[i] & 15) << (4 * i);
                    *reinterpret_cast<uint32_t *>(dst + 4 * grp) = wv;
                } else {
                    uint32_t wv = 0;
                    for (int i = 0; i < 8; ++i) wv |= (uint32_t)(q[i] & 7) << (3 * i);
                    dst[3 * grp + 0] = (uint8_t)wv;
                    dst[3 * grp + 1] = (uint8_t)(wv >> 8);
                    dst[3 * grp + 2] = (uint8_t)(wv >> 16);
                }
            }
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------------------------------
// Host launchers
// ------------------------------------------------------------------------------------------

// The direct kernel for (C, thread split, DB, PLAN); the hidden sizes of OPT-6.7B, -66B and
// -175B with 16-bit inputs are compiled for their exact thread split (the plan below picks
// 512 x 1, 384 x 3 and 384 x 4 chunks).
template <typename T, int BITS, int CPT, int MAXT, bool PLAN>
static const void *direct_kernel_for(int C, int NT, bool db)
{
    const void *kern = db ? (const void *)ln_quant_direct_kernel<T, BITS, CPT, MAXT, true, PLAN>
                          : (const void *)ln_quant_direct_kernel<T, BITS, CPT, MAXT, false, PLAN>;
    if constexpr (sizeof(T) == 2 && CPT == 1 && MAXT == 512) {
        if (C == 4096 && NT == 4096 / 8)
            kern = db ? (const void *)ln_quant_direct_kernel<T, BITS, 1, 512, true, PLAN, 4096>
                      : (const void *)ln_quant_direct_kernel<T, BITS, 1, 512, false, PLAN, 4096>;
    }
    if constexpr (sizeof(T) == 2 && CPT == 3 && MAXT == 384) {
        if (C == 9216 && NT == 9216 / 8 / 3)
            kern = db ? (const void *)ln_quant_direct_kernel<T, BITS, 3, 384, true, PLAN, 9216>
                      : (const void *)ln_quant_direct_kernel<T, BITS, 3, 384, false, PLAN, 9216>;
    }
    if constexpr (sizeof(T) == 2 && CPT == 4 && MAXT == 384) {
        if (C == 12288 && NT == 12288 / 8 / 4)
            kern = db ? (const void *)ln_quant_direct_kernel<T, BITS, 4, 384, true, PLAN, 12288>
                      : (const void *)ln_quant_direct_kernel<T, BITS, 4, 384, false, PLAN, 12288>;
    }
    return kern;
}

template <typename T, int BITS, int CPT, int MAXT>
static cudaError_t launch_direct_t(const LnQuantArgs &a, int NT)
{
    // two code buffers (one barrier per quad) whenever they fit: with the thread split fixed at
    // compile time, bf16 A3 measured 0.685 -> 0.706 of the HBM copy rate at C = 12288 (one
    // buffer was faster there with a runtime split) and 0.59 -> 0.62 at C = 9216
    const int g = a.plan ? 0 : a.g;  // a planned launch keeps no cluster table in shared memory
    const size_t db_smem = direct_db_off(a.C, g) + (size_t)4 * a.C;
    const bool db = db_smem <= (size_t)a.max_smem;
    const size_t smem = db ? db_smem : direct_smem_bytes(a.C, g);
    const void *kern = a.plan ? direct_kernel_for<T, BITS, CPT, MAXT, true>(a.C, NT, db)
                              : direct_kernel_for<T, BITS, CPT, MAXT, false>(a.C, NT, db);
    cudaError_t e = kernel_smem(kern, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = kernel_occupancy(&per_sm, kern, NT, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t quads = (a.T + 3) / 4;
    const int64_t grid = std::min<int64_t>(quads, (int64_t)per_sm * a.num_sms);
    void *args[] = {(void *)&a.x,     (void *)&a.T,     (void *)&a.C,     (void *)&a.gamma, (void *)&a.beta,
                    (void *)&a.eps,   (void *)&a.R,     (void *)&a.col_cluster, (void *)&a.scale,
                    (void *)&a.zero,  (void *)&a.g,     (void *)&a.codes, (void *)&a.plan,  (void *)&a.err};
    return cudaLaunchKernel(kern, dim3((unsigned)grid), dim3(NT), args, smem, a.stream);
}

template <typename T, int BITS, int CPT>
static cudaError_t launch_fast_t(const LnQuantArgs &a, int NT, int NS, int alias)
{
    const uint32_t rowbytes = (uint32_t)a.C * sizeof(T);
    const QuadSmem L = quad_smem_layout(NS, rowbytes, (alias ? 0 : (size_t)a.C * 4) + (size_t)a.C * 2 + 2 * 8 * 32 * 4);
    auto kern = ln_quant_fast_kernel<T, BITS, CPT>;
    cudaError_t e = kernel_smem((const void *)kern, L.total);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = kernel_occupancy(&per_sm, (const void *)kern, NT, L.total);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t quads = (a.T + 3) / 4;
    const int64_t grid = std::min<int64_t>(quads, (int64_t)per_sm * a.num_sms);
    kern<<<(unsigned)grid, NT, L.total, a.stream>>>((const T *)a.x, a.T, a.C, a.gamma, a.beta, a.eps,
                                                    a.R, a.col_cluster, a.scale, a.zero, a.g,
                                                    a.codes, NS, alias, a.err);
    return cudaGetLastError();
}

template <typename T, int BITS>
static cudaError_t launch_fast_b(const LnQuantArgs &a, int CPT, int NT, int NS, int alias)
{
    if (alias == 2) {
        switch (CPT) {
        case 1: return launch_direct_t<T, BITS, 1, 512>(a, NT);
        case 2: return launch_direct_t<T, BITS, 2, 512>(a, NT);
        case 3: return NT <= 384 ? launch_direct_t<T, BITS, 3, 384>(a, NT) : launch_direct_t<T, BITS, 3, 512>(a, NT);
        case 4: return launch_direct_t<T, BITS, 4, 384>(a, NT);
        default: return cudaErrorInvalidValue;
        }
    }
    switch (CPT) {
    case 1: return launch_fast_t<T, BITS, 1>(a, NT, NS, alias);
    case 2: return launch_fast_t<T, BITS, 2>(a, NT, NS, alias);
    case 3: return launch_fast_t<T, BITS, 3>(a, NT, NS, alias);
    default: return cudaErrorInvalidValue;
    }
}

template <typename T>
static cudaError_t launch_fast_d(const LnQuantArgs &a, int CPT, int NT, int NS, int alias)
{
    return a.bits == 4 ? launch_fast_b<T, 4>(a, CPT, NT, NS, alias) : launch_fast_b<T, 3>(a, CPT, NT, NS, alias);
}

// Plan of the fast kernels for (C, dtype): threads, chunks per thread and, for the ring kernel,
// ring depth and code-buffer placement (*alias = 0: own buffer, 1: in the quad's slots);
// *alias = 2 selects the direct kernel (no ring; allow_direct: R and col_cluster are 16-byte
// aligned for its vector loads).  Returns false when the shape needs the simple kernel.
bool ln_quant_fast_plan(int C, int esize, int max_smem, bool allow_direct, int *CPT, int *NT, int *NS, int *alias)
{
    if (C % 32 != 0) return false;
    const int VEC = 16 / esize;
    const int NCH = C / VEC;
    int cpt = 0, nt = 0;
    for (int k = 1; k <= 3; ++k) {
        const int n = ((NCH + k - 1) / k + 31) / 32 * 32;
        if (n <= 512) {
            cpt = k;
            nt = n;
            break;
        }
    }
    if (allow_direct && direct_smem_bytes(C, RPTQ_MAX_CLUSTERS) <= (size_t)max_smem) {  // direct kernel
        // 320..384 threads x 3 chunks, or 256..384 threads x 4 chunks, when that splits the row
        // exactly (every thread also packs one 32-position unit), else the ring kernel's choice
        // of up to 512 threads
        int dc = cpt, dn = nt;
        if (NCH % (3 * 32) == 0 && NCH / 3 <= 384 && NCH / 3 >= 320) {
            dc = 3;
            dn = NCH / 3;
        } else if (NCH % (4 * 32) == 0 && NCH / 4 <= 384 && NCH / 4 >= 256) {
            dc = 4;
            dn = NCH / 4;
        }
        if (!dc) return false;
        *CPT = dc;
        *NT = dn;
        *NS = 0;
        *alias = 2;
        return true;
    }
    if (!cpt) return false;
    const uint32_t rowbytes = (uint32_t)C * esize;
    const size_t tables = (size_t)C * 2 + 2 * 8 * 32 * 4;
    auto fits = [&](int ns, bool al) {
        return quad_smem_layout(ns, rowbytes, (al ? 0 : (size_t)C * 4) + tables).total <= (size_t)max_smem;
    };
    // preference: 8 ring rows with a separate code buffer, then 8 rows with the code buffer in
    // the quad's own slots, then fewer rows
    int ns = 0, al = 0;
    if (fits(8, false)) {
        ns = 8;
    } else if (fits(8, true)) {
        ns = 8;
        al = 1;
    } else {
        for (int n = 7; n >= 4 && !ns; --n)
            if (fits(n, false)) ns = n;
    }
    if (!ns) return false;
    *CPT = cpt;
    *NT = nt;
    *NS = ns;
    *alias = al;
    return true;
}

template <typename T>
static cudaError_t launch_simple_t(const LnQuantArgs &a)
{
    const size_t smem = (size_t)a.C * 5;
    auto kern = ln_quant_simple_kernel<T>;
    cudaError_t e = kernel_smem((const void *)kern, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = kernel_occupancy(&per_sm, (const void *)kern, 256, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t grid = std::min<int64_t>(a.T, (int64_t)per_sm * a.num_sms);
    kern<<<(unsigned)grid, 256, smem, a.stream>>>((const T *)a.x, a.T, a.C, a.gamma, a.beta, a.eps, a.R,
                                                  a.col_cluster, a.scale, a.zero, a.g, a.bits, a.codes,
                                                  (T *)a.ln_out, a.err);
    return cudaGetLastError();
}

cudaError_t launch_ln_quant_plan(const float *gamma, const float *beta, const int32_t *R, const int32_t *col_cluster,
                                 const float *scale, const int32_t *zero, int C, int g, int bits, void *plan,
                                 int *err, cudaStream_t stream)
{
    cudaError_t e = cudaMemsetAsync(plan, 0, (size_t)C * 12, stream);
    if (e != cudaSuccess) return e;
    uint32_t *pos = static_cast<uint32_t *>(plan);
    float *A = reinterpret_cast<float *>(pos + C), *B = A + C;
    const unsigned grid = (unsigned)((C + 255) / 256);
    if (bits == 4)
        ln_quant_plan_kernel<4><<<grid, 256, 0, stream>>>(gamma, beta, R, col_cluster, scale, zero, C, g, pos, A, B, err);
    else
        ln_quant_plan_kernel<3><<<grid, 256, 0, stream>>>(gamma, beta, R, col_cluster, scale, zero, C, g, pos, A, B, err);
    return cudaGetLastError();
}

// Whether (C, dtype) runs on the direct kernel, the only one that takes a plan.
bool ln_quant_plan_supported(int C, int esize, int max_smem)
{
    int CPT = 0, NT = 0, NS = 0, alias = 0;
    return ln_quant_fast_plan(C, esize, max_smem, true, &CPT, &NT, &NS, &alias) && alias == 2;
}

cudaError_t launch_ln_quant(const LnQuantArgs &a, int force_simple)
{
    if (a.T == 0) return cudaSuccess;
    const int esize = a.dtype == RPTQ_F32 ? 4 : 2;
    int CPT = 0, NT = 0, NS = 0, alias = 0;
    const bool vec_tables = (uintptr_t)a.R % 16 == 0 && (uintptr_t)a.col_cluster % 16 == 0 &&
                            (uintptr_t)a.gamma % 16 == 0 && (uintptr_t)a.beta % 16 == 0;
    const bool fast = !force_simple && a.ln_out == nullptr && a.codes != nullptr &&
                      ln_quant_fast_plan(a.C, esize, a.max_smem, vec_tables || a.plan, &CPT, &NT, &NS, &alias);
    if (a.plan && !(fast && alias == 2)) return cudaErrorInvalidValue;  // checked by the caller
    if (fast) {
        switch (a.dtype) {
        case RPTQ_F32: return launch_fast_d<float>(a, CPT, NT, NS, alias);
        case RPTQ_F16: return launch_fast_d<__half>(a, CPT, NT, NS, alias);
        default: return launch_fast_d<__nv_bfloat16>(a, CPT, NT, NS, alias);
        }
    }
    switch (a.dtype) {
    case RPTQ_F32: return launch_simple_t<float>(a);
    case RPTQ_F16: return launch_simple_t<__half>(a);
    default: return launch_simple_t<__nv_bfloat16>(a);
    }
}

}  // namespace rptq
