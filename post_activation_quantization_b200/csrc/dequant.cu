// dequant.cu -- dequantization value = s_k * (q - z_k) (quantization-basics article,
// section 1.3: the real value is the scale times the code minus the zero point).
//
// The code q becomes an exact float without a conversion instruction: the bit pattern
// 0x4B000000 | q is the float 2^23 + q, and 2^23 + z is exact for |z| < 2^23 - 16, so
// (2^23 + q) - (2^23 + z) = q - z exactly and one multiply by s gives the same fp32 value as
// s * (float)(q - z).  A thread whose channels include a larger |z| converts with an integer ->
// float conversion instead (same result).
//
// Span kernels (the common shapes): a lane owns groups of 8 consecutive channels, and the 32
// lanes of a warp own 32 consecutive groups, so every warp-wide 16-byte store covers 512
// contiguous bytes of the output (whole 128-byte lines).  The 8 packed codes of a lane are 4
// bytes (A4: one word per lane) or 3 bytes (A3: 24 lanes load the warp's 96 bytes as words and
// each lane assembles its 3 bytes with two shuffles and a funnel shift).  Rows layout: warp w
// of a CTA owns the 256-channel spans w, w + WR, w + 2 WR, ... of every row it walks, with
// their (s, 2^23 + z) in registers.  BHSD layout: a warp covers 256 / D consecutive rows per
// store, so a lane's channel position is fixed; warps take contiguous ranges of (h, b, chunk)
// units.  Other shapes use the general kernel (DPT consecutive channels per thread).
//
// Ring kernel (BHSD layout, 16-bit output, shapes that pass kv_ring_shape_ok): the stage
// decomposition of kv_stream.cuh run in reverse.  A stage is 32 KB of output (2048 pieces of 8
// channels) and 2048*BITS contiguous bytes of codes; thread 0 streams the codes into a ring of
// shared slots, every thread decodes its eight pieces into one of two 32 KB staging buffers, and
// thread 0 writes the stage with one bulk copy.
#include <algorithm>

#include "kv_stream.cuh"
#include "launch.h"

namespace rptq {

// Output stores are streaming (st.global.cs): the dequantised tensor is not read again by this
// library, and evict-first stores measured 79% -> 84% of the HBM copy rate on the row layout.
template <typename T> struct Store;
template <> struct Store<float> {
    template <int N> __device__ static void put(float *dst, const float (&v)[N])
    {
#pragma unroll
        for (int i = 0; i < N; i += 4)
            __stcs(reinterpret_cast<float4 *>(dst + i), make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]));
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
            __stcs(reinterpret_cast<uint4 *>(dst + i), make_uint4(w[0], w[1], w[2], w[3]));
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
            __stcs(reinterpret_cast<uint4 *>(dst + i), make_uint4(w[0], w[1], w[2], w[3]));
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

// ---------------------------------------------------------------------------------------------
// span kernels
template <int BITS>
__device__ __forceinline__ uint32_t span_load(const uint8_t *span, int lane)
{
    // A4: 128 bytes, word `lane`; A3: 96 bytes, words 0..23 (lanes 24..31 load nothing)
    if constexpr (BITS == 4) return ldg_stream32(span + 4 * lane);
    return lane < 24 ? ldg_stream32(span + 4 * lane) : 0u;
}
// the same when only the first `valid` bytes of the span exist (a partial last span)
template <int BITS>
__device__ __forceinline__ uint32_t span_load_partial(const uint8_t *span, int lane, int valid)
{
    uint32_t v = 0;
    for (int b = 0; b < 4; ++b)
        if (4 * lane + b < valid) v |= (uint32_t)span[4 * lane + b] << (8 * b);
    return v;
}
template <int BITS>
__device__ __forceinline__ uint32_t span_codes(uint32_t w, int lane)
{
    if constexpr (BITS == 4) return w;
    const int b = 3 * lane, i0 = b >> 2;
    const uint32_t lo = __shfl_sync(FULL, w, i0), hi = __shfl_sync(FULL, w, (i0 + 1) & 31);
    return __funnelshift_r(lo, hi, 8 * (b & 3)) & 0xffffffu;
}

// 8 values s * (q - z) of one group; nzf = -(2^23 + z) (exact path) and the scales
template <typename T, int BITS>
__device__ __forceinline__ void decode_store(uint32_t grp, const float (&sc)[8], const float (&nzf)[8], T *dst)
{
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const uint32_t q0 = (grp >> (BITS * i)) & ((1u << BITS) - 1), q1 = (grp >> (BITS * (i + 1))) & ((1u << BITS) - 1);
        const f32x2 x = add2(mk2(__uint_as_float(0x4B000000u | q0), __uint_as_float(0x4B000000u | q1)),
                             mk2(nzf[i], nzf[i + 1]));
        const f32x2 y = mul2(x, mk2(sc[i], sc[i + 1]));
        v[i] = lo2(y);
        v[i + 1] = hi2(y);
    }
    Store<T>::template put<8>(dst, v);
}
// the same through an integer subtraction (any z); channels c0 .. c0+7
template <typename T, int BITS>
__device__ __forceinline__ void decode_store_slow(uint32_t grp, const float (&sc)[8], const int32_t *cluster, int c0,
                                               const int32_t *zero, int g, T *dst)
{
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int k = cluster[c0 + i];
        k = (k < 0 || k >= g) ? 0 : k;
        v[i] = sc[i] * (float)((int)((grp >> (BITS * i)) & ((1u << BITS) - 1)) - zero[k]);
    }
    Store<T>::template put<8>(dst, v);
}

__device__ __forceinline__ int checked_cluster(const int32_t *cluster, int c, int g, int *err)
{
    int k = cluster[c];
    if (k < 0 || k >= g) {
        raise_error(err, RPTQ_DEVERR_CLUSTER_ID);
        k = 0;
    }
    return k;
}

// Rows layout, C % 256 == 0: CTA = WR warps, warp w owns spans w + WR*i (i < NSPAN) of every row.
// SPLIT: the row's spans are split into `parts` column ranges of WR * NSPAN spans, CTA b taking
// range b % parts of every (gridDim / parts)-th row, so that rows too wide for one CTA of one
// span per warp still get several resident CTAs per SM.
template <typename T, int BITS, int NSPAN, bool SPLIT>
__global__ void __launch_bounds__(NSPAN <= 2 ? 1024 : 512)
    dequant_rows_span(const uint8_t *__restrict__ codes, int64_t rows, int C, const int32_t *__restrict__ cluster,
                      const float *__restrict__ scale, const int32_t *__restrict__ zero, int g, T *__restrict__ out,
                      int *err, int parts)
{
    constexpr int U = 4;  // rows in flight
    const int lane = threadIdx.x & 31, WR = blockDim.x >> 5;
    const int w = (threadIdx.x >> 5) + (SPLIT ? (int)(blockIdx.x % parts) * WR * NSPAN : 0);
    const int64_t pitch = (int64_t)C * BITS / 8;
    float sc[NSPAN][8], nzf[NSPAN][8];
    bool exact = true;
#pragma unroll
    for (int i = 0; i < NSPAN; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int c = (w + WR * i) * 256 + 8 * lane + e;
            const int k = checked_cluster(cluster, c, g, err);
            sc[i][e] = scale[k];
            const int z = zero[k];
            const bool ok = z > -(1 << 23) + 16 && z < (1 << 23) - 16;
            exact &= ok;
            nzf[i][e] = -(float)((1 << 23) + (ok ? z : 0));
        }
    exact = __all_sync(FULL, exact);  // the shuffles below need the whole warp on one path
    const int64_t step = SPLIT ? gridDim.x / parts : gridDim.x;
    for (int64_t r0 = SPLIT ? blockIdx.x / parts : blockIdx.x; r0 < rows; r0 += U * step) {
        uint32_t wv[U][NSPAN];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t r = r0 + u * step;
#pragma unroll
            for (int i = 0; i < NSPAN; ++i)
                wv[u][i] = r < rows ? span_load<BITS>(codes + r * pitch + (int64_t)(w + WR * i) * (32 * BITS), lane) : 0u;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t r = r0 + u * step;
#pragma unroll
            for (int i = 0; i < NSPAN; ++i) {
                const uint32_t grp = span_codes<BITS>(wv[u][i], lane);
                T *dst = out + r * C + (w + WR * i) * 256 + 8 * lane;
                if (r < rows) {
                    if (exact)
                        decode_store<T, BITS>(grp, sc[i], nzf[i], dst);
                    else
                        decode_store_slow<T, BITS>(grp, sc[i], cluster, (w + WR * i) * 256 + 8 * lane, zero, g, dst);
                }
            }
        }
    }
}

// Eight fp32 values -> one 16-byte chunk of 16-bit values (round to nearest even).
template <typename T> __device__ __forceinline__ uint4 pack8(const float (&v)[8]);
template <> __device__ __forceinline__ uint4 pack8<__nv_bfloat16>(const float (&v)[8])
{
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 p = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
        w[j] = *reinterpret_cast<const uint32_t *>(&p);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}
template <> __device__ __forceinline__ uint4 pack8<__half>(const float (&v)[8])
{
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const __half2 p = __floats2half2_rn(v[2 * j], v[2 * j + 1]);
        w[j] = *reinterpret_cast<const uint32_t *>(&p);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// ring depth of the (small) code stages: measured at [8, 96, 2048, 128] 3-bit -> bf16, a depth
// of 2 streams at 82% of the HBM copy rate, depths 3, 6 and 8 at 79%
constexpr int DQR_NS = 2;
template <int BITS>
constexpr size_t dq_ring_smem() { return (size_t)DQR_NS * KVR_PIECES * BITS + 2 * (size_t)KVR_STAGE + 8 * DQR_NS; }

template <typename T, int BITS>
__global__ void __launch_bounds__(KVR_THREADS, 2)
    dequant_bhsd_ring(const uint8_t *__restrict__ codes, int B, int H, int SPB, int D,
                      const int32_t *__restrict__ cluster, const float *__restrict__ scale,
                      const int32_t *__restrict__ zero, int g, T *__restrict__ out, int *err)
{
    constexpr uint32_t CBYTES = KVR_PIECES * BITS;  // codes of one stage
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_abort;
    uint8_t *stage = smem;                                  // 2 x 32 KB of output
    uint8_t *ring = smem + 2 * (size_t)KVR_STAGE;           // DQR_NS x CBYTES of codes
    const uint32_t bar0 = smem_u32(ring + (size_t)DQR_NS * CBYTES);
    const int tid = threadIdx.x;
    const int64_t total = (int64_t)B * H * SPB;
    const int64_t j0 = total * blockIdx.x / gridDim.x, j1 = total * (blockIdx.x + 1) / gridDim.x;
    const int n = (int)(j1 - j0);
    if (n <= 0) return;
    KvStagePos prod;  // thread 0: the next stage whose codes to load
    auto issue = [&](uint32_t s) {
        mbar_expect_tx(bar0 + 8u * s, CBYTES);
        bulk_g2s(smem_u32(ring + (size_t)s * CBYTES), codes + prod.mem_index(H, SPB) * CBYTES, CBYTES, bar0 + 8u * s);
        prod.advance(B, H, SPB);
    };
    if (tid == 0) {
        s_abort = 0;
        for (int s = 0; s < DQR_NS; ++s) mbar_init(bar0 + 8u * s, 1);
        fence_mbar_init();
        prod.set(j0, total, B, SPB);
        for (int s = 0; s < DQR_NS && s < n; ++s) issue((uint32_t)s);
    }
    __syncthreads();
    KvStagePos cur;
    cur.set(j0, total, B, SPB);
    const int col = tid & ((D >> 3) - 1);  // the thread's 8-channel group in every piece
    float sc[8], nzf[8];
    bool exact = true;
    int cur_h = -1;
    uint32_t slot = 0, phase = 0;
    for (int i = 0; i < n; ++i) {
        if (cur.h != cur_h) {
            exact = true;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int k = checked_cluster(cluster, cur.h * D + col * 8 + e, g, err);
                sc[e] = scale[k];
                const int z = zero[k];
                const bool ok = z > -(1 << 23) + 16 && z < (1 << 23) - 16;
                exact &= ok;
                nzf[e] = -(float)((1 << 23) + (ok ? z : 0));
            }
            cur_h = cur.h;
        }
        if (!mbar_wait_bounded(bar0 + 8u * slot, phase, err)) s_abort = 1;
        const uint8_t *cs = ring + (size_t)slot * CBYTES;
        uint4 *dst = reinterpret_cast<uint4 *>(stage + (size_t)(i & 1) * KVR_STAGE);
#pragma unroll
        for (int k = 0; k < KVR_PPT; ++k) {
            const int p = tid + k * KVR_THREADS;
            uint32_t grp;
            if constexpr (BITS == 4) {
                grp = *reinterpret_cast<const uint32_t *>(cs + 4 * p);
            } else {  // 3 bytes at 3p: the aligned word holding the first, the next one only
                      // when the bytes cross into it (never past the slot), and a funnel shift
                const uint32_t *w = reinterpret_cast<const uint32_t *>(cs) + ((3 * p) >> 2);
                const uint32_t sh = (uint32_t)((3 * p) & 3) * 8u;
                grp = __funnelshift_r(w[0], sh > 8u ? w[1] : 0u, sh) & 0xffffffu;
            }
            float v[8];
            if (exact) {
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const uint32_t q0 = (grp >> (BITS * e)) & ((1u << BITS) - 1), q1 = (grp >> (BITS * (e + 1))) & ((1u << BITS) - 1);
                    const f32x2 x = add2(mk2(__uint_as_float(0x4B000000u | q0), __uint_as_float(0x4B000000u | q1)),
                                         mk2(nzf[e], nzf[e + 1]));
                    const f32x2 y = mul2(x, mk2(sc[e], sc[e + 1]));
                    v[e] = lo2(y);
                    v[e + 1] = hi2(y);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int kc = checked_cluster(cluster, cur.h * D + col * 8 + e, g, err);
                    v[e] = sc[e] * (float)((int)((grp >> (BITS * e)) & ((1u << BITS) - 1)) - zero[kc]);
                }
            }
            dst[p] = pack8<T>(v);
        }
        // the previous stage's output copy has finished reading its buffer, which the stage after
        // this one rewrites
        if (tid == 0) bulk_wait_read<0>();
        __syncthreads();  // codes slot read, the stage's output complete
        if (s_abort) break;
        if (tid == 0) {
            fence_proxy_async_smem();
            bulk_s2g(reinterpret_cast<uint8_t *>(out) + cur.mem_index(H, SPB) * KVR_STAGE, smem_u32(dst), KVR_STAGE);
            bulk_commit();
            if (i + DQR_NS < n) issue(slot);
        }
        cur.advance(B, H, SPB);
        if (++slot == DQR_NS) {
            slot = 0;
            phase ^= 1u;
        }
    }
    if (tid == 0) bulk_wait_all();
}

// BHSD layout, D % 8 == 0 and (D/8) divides 32.  A span is the RPW = 256/D consecutive rows one
// warp-wide store covers; a work unit is up to 32 spans of one (b, h) block; units are ordered
// (h, b, chunk) and every warp of a one-wave grid takes a contiguous range of them.  A lane's
// channel position p is fixed; its 8 (s, 2^23 + z) are reloaded when the head changes.
constexpr int DQ_SPANS_PER_UNIT = 32;

template <typename T, int BITS>
__global__ void __launch_bounds__(256)
    dequant_bhsd_span(const uint8_t *__restrict__ codes, int B, int H, int S, int D, const int32_t *__restrict__ cluster,
                      const float *__restrict__ scale, const int32_t *__restrict__ zero, int g, T *__restrict__ out,
                      int *err)
{
    constexpr int U = 4;
    const int lane = threadIdx.x & 31;
    const int G8 = D >> 3, RPW = 32 / G8;
    const int p = 8 * (lane % G8), lrow = lane / G8;
    const int nspan = (S + RPW - 1) / RPW;  // spans per (b, h)
    const int nchunk = (nspan + DQ_SPANS_PER_UNIT - 1) / DQ_SPANS_PER_UNIT;
    // units in (h, b, chunk) order; warp gw takes the contiguous range [u0, u1), so it crosses
    // at most a few heads and reloads its coefficients only then
    const int64_t units = (int64_t)H * B * nchunk, TW = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t u0 = units * gw / TW, u1 = units * (gw + 1) / TW;
    int64_t hb = u0 / nchunk;
    int chunk = (int)(u0 - hb * nchunk);
    int h = (int)(hb / B), b = (int)(hb - (int64_t)h * B);
    float sc[8], nzf[8];
    bool exact = true;
    int cur_h = -1;
    for (int64_t un = u0; un < u1; ++un) {
        if (h != cur_h) {
            exact = true;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int k = checked_cluster(cluster, h * D + p + e, g, err);
                sc[e] = scale[k];
                const int z = zero[k];
                const bool ok = z > -(1 << 23) + 16 && z < (1 << 23) - 16;
                exact &= ok;
                nzf[e] = -(float)((1 << 23) + (ok ? z : 0));
            }
            exact = __all_sync(FULL, exact);
            cur_h = h;
        }
        const int64_t bh = (int64_t)b * H + h;
        const int sp0 = chunk * DQ_SPANS_PER_UNIT, sp1 = min(nspan, sp0 + DQ_SPANS_PER_UNIT);
        const int64_t blk = bh * S;  // first row of this (b, h)
        if (sp1 - sp0 == DQ_SPANS_PER_UNIT && (int64_t)sp1 * RPW <= S) {
            // a whole unit: 32 full spans, contiguous codes and output from the unit's base
            const uint8_t *cu = codes + (blk + (int64_t)sp0 * RPW) * D * BITS / 8;
            T *ou = out + (blk + (int64_t)sp0 * RPW + lrow) * D + p;
#pragma unroll 1
            for (int sp = 0; sp < DQ_SPANS_PER_UNIT; sp += 2 * U) {
                uint32_t wv[2 * U];
#pragma unroll
                for (int u = 0; u < 2 * U; ++u) wv[u] = span_load<BITS>(cu + (sp + u) * (32 * BITS), lane);
#pragma unroll
                for (int u = 0; u < 2 * U; ++u) {
                    const uint32_t grp = span_codes<BITS>(wv[u], lane);
                    T *dst = ou + (int64_t)(sp + u) * 256;
                    if (exact)
                        decode_store<T, BITS>(grp, sc, nzf, dst);
                    else
                        decode_store_slow<T, BITS>(grp, sc, cluster, h * D + p, zero, g, dst);
                }
            }
        } else
        for (int sp = sp0; sp < sp1; sp += U) {
            uint32_t wv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int spu = sp + u;
                const int nrow = min(RPW, S - spu * RPW);
                const uint8_t *src = codes + (blk + (int64_t)spu * RPW) * D * BITS / 8;
                wv[u] = spu >= sp1 ? 0u
                        : nrow == RPW ? span_load<BITS>(src, lane)
                                      : span_load_partial<BITS>(src, lane, nrow * D * BITS / 8);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int spu = sp + u;
                const uint32_t grp = span_codes<BITS>(wv[u], lane);
                const int row = spu * RPW + lrow;
                if (spu < sp1 && row < S) {
                    T *dst = out + (blk + row) * D + p;
                    if (exact)
                        decode_store<T, BITS>(grp, sc, nzf, dst);
                    else
                        decode_store_slow<T, BITS>(grp, sc, cluster, h * D + p, zero, g, dst);
                }
            }
        }
        if (++chunk == nchunk) {  // next unit
            chunk = 0;
            if (++b == B) {
                b = 0;
                ++h;
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

template <typename T, int BITS, int NSPAN, bool SPLIT>
static cudaError_t launch_rows_span(const DequantArgs &a, int WR, int parts, int per_sm)
{
    const int threads = WR * 32;
    const int64_t ctas = std::max<int64_t>(1, std::min<int64_t>(a.n0, (int64_t)a.num_sms * per_sm / parts));
    dequant_rows_span<T, BITS, NSPAN, SPLIT><<<(unsigned)(ctas * parts), threads, 0, a.stream>>>(
        a.codes, a.n0, a.n1, a.cluster, a.scale, a.zero, a.g, (T *)a.out, a.err, parts);
    return cudaGetLastError();
}

template <typename T, int BITS>
static cudaError_t launch_dq_ring(const DequantArgs &a)
{
    const int SPB = (int)(a.S / kv_ring_rows(a.D));
    auto kern = dequant_bhsd_ring<T, BITS>;
    const size_t smem = dq_ring_smem<BITS>();
    cudaError_t e = kernel_smem((const void *)kern, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = kernel_occupancy(&per_sm, (const void *)kern, KVR_THREADS, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t total = a.n0 * a.n1 * SPB;
    const int64_t grid = std::min<int64_t>((int64_t)per_sm * a.num_sms, total);
    kern<<<(unsigned)grid, KVR_THREADS, smem, a.stream>>>(a.codes, (int)a.n0, a.n1, SPB, a.D, a.cluster, a.scale,
                                                          a.zero, a.g, (T *)a.out, a.err);
    return cudaGetLastError();
}

template <typename T, int BITS>
static cudaError_t launch_dq_b(const DequantArgs &a)
{
    const bool aligned = ((uintptr_t)a.codes % 4 == 0) && ((uintptr_t)a.out % 16 == 0);
    if constexpr (sizeof(T) == 2)  // bulk copies: both bases 16-byte aligned (checked by the caller)
        if (a.layout == RPTQ_LAYOUT_BHSD && a.n0 <= 0x7fffffff && kv_ring_shape_ok((int)a.n0, a.n1, a.S, a.D, 2))
            return launch_dq_ring<T, BITS>(a);
    if (a.layout == RPTQ_LAYOUT_BHSD) {
        // word loads need every (b, h) block of codes to start on a 4-byte boundary
        const bool blocks4 = ((int64_t)a.S * a.D * BITS / 8) % 4 == 0;
        if (aligned && blocks4 && a.D % 8 == 0 && 32 % (a.D / 8) == 0 && a.D <= 256) {
            int per_sm = 1;
            if (kernel_occupancy(&per_sm, (const void *)dequant_bhsd_span<T, BITS>, 256, 0) !=
                    cudaSuccess ||
                per_sm < 1)
                per_sm = 1;
            const int64_t rpw = 32 / (a.D / 8), nspan = (a.S + rpw - 1) / rpw;
            const int64_t units = a.n0 * a.n1 * ((nspan + DQ_SPANS_PER_UNIT - 1) / DQ_SPANS_PER_UNIT);
            const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((int64_t)a.num_sms * per_sm, (units + 7) / 8));
            dequant_bhsd_span<T, BITS><<<(unsigned)grid, 256, 0, a.stream>>>(
                a.codes, (int)a.n0, a.n1, (int)a.S, a.D, a.cluster, a.scale, a.zero, a.g, (T *)a.out, a.err);
            return cudaGetLastError();
        }
    } else if (aligned && a.n1 % 256 == 0) {
        const int spans = a.n1 / 256;  // 256-channel spans per row, at most 64
        // a CTA takes spans / parts spans of a row, NSPAN per warp: the first split (fewest
        // parts, then fewest spans per warp) that keeps at least 24 warps resident on an SM,
        // else the split with the most
        const void *whole[5] = {nullptr, (const void *)dequant_rows_span<T, BITS, 1, false>,
                                (const void *)dequant_rows_span<T, BITS, 2, false>,
                                (const void *)dequant_rows_span<T, BITS, 3, false>,
                                (const void *)dequant_rows_span<T, BITS, 4, false>};
        const void *split[3] = {nullptr, (const void *)dequant_rows_span<T, BITS, 1, true>,
                                (const void *)dequant_rows_span<T, BITS, 2, true>};
        int bp = 0, bn = 0, bwarps = 0, bper = 0;
        for (int parts = 1; parts <= 4; ++parts)
            for (int n = 1; n <= (parts == 1 ? 4 : 2); ++n) {
                if (spans % (parts * n) != 0) continue;
                const int wr = spans / (parts * n);
                if (wr * 32 > (n <= 2 ? 1024 : 512) || wr < std::min(4, spans)) continue;
                int per_sm = 0;
                if (kernel_occupancy(&per_sm, parts == 1 ? whole[n] : split[n], wr * 32, 0) != cudaSuccess) per_sm = 0;
                if (per_sm * wr > bwarps && bwarps < 24) {
                    bp = parts, bn = n, bwarps = per_sm * wr, bper = per_sm;
                }
            }
        if (bn) {
            const int wr = spans / (bp * bn);
            if (bp > 1)
                return bn == 1 ? launch_rows_span<T, BITS, 1, true>(a, wr, bp, bper)
                               : launch_rows_span<T, BITS, 2, true>(a, wr, bp, bper);
            if (bn == 1) return launch_rows_span<T, BITS, 1, false>(a, wr, 1, bper);
            if (bn == 2) return launch_rows_span<T, BITS, 2, false>(a, wr, 1, bper);
            if (bn == 3) return launch_rows_span<T, BITS, 3, false>(a, wr, 1, bper);
            return launch_rows_span<T, BITS, 4, false>(a, wr, 1, bper);
        }
    }
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
