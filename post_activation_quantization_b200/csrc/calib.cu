// calib.cu -- calibration statistics: per-channel max and min over calibration tokens.
//
// RPTQ article (基于重排序的新量化方法RPTQ…), text after Fig. 2 (run calibration data through
// the model and record each activation channel's max and min) and the Fig. 1 caption (one
// (max, min) point per channel).  The statistic is taken on the tensor that is later
// quantized: LayerNorm(x) for the activation path, the raw tensor for the K/V path.
//
// Raw mode: a CTA owns 32 chunk columns (512 bytes of every row, one 16-byte chunk per lane)
// and a contiguous row range; its eight warps stride over the rows, keep running max/min in
// registers (packed half2/bfloat162 max/min for 16-bit inputs, which are exact), combine
// through shared memory and fold into the outputs with integer atomics (exact and
// order-independent, so the result equals a sequential CPU max/min bit for bit).
//
// LayerNorm mode: the row pipeline of row_pipeline.cuh (bulk-copied token rows, fp32
// LayerNorm statistics).  For every owned channel a thread keeps the running max and min of
// the normalised value t = (x - mean) * rstd over its quads; the affine part y = t*gamma+beta is
// monotone in t, so max y = fmaf(max t, gamma, beta) for gamma >= 0 (and the min of t for
// gamma < 0) is the same value as taking the max of the per-token fmaf results.
#include <algorithm>

#include "kv_stream.cuh"
#include "launch.h"
#include "row_pipeline.cuh"

namespace rptq {

__global__ void calib_init_kernel(float *ch_max, float *ch_min, int C)
{
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c < C) {
        ch_max[c] = -INFINITY;
        ch_min[c] = INFINITY;
    }
}

// ---- raw mode ------------------------------------------------------------------------------
template <typename T> struct RawAcc;
template <> struct RawAcc<float> {
    float mx[4], mn[4];
    __device__ void init()
    {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            mx[i] = -INFINITY;
            mn[i] = INFINITY;
        }
    }
    __device__ void add(const uint4 &v)
    {
        const float f[4] = {__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z),
                            __uint_as_float(v.w)};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            mx[i] = fmaxf(mx[i], f[i]);
            mn[i] = fminf(mn[i], f[i]);
        }
    }
    __device__ float get_max(int e) const { return mx[e]; }
    __device__ float get_min(int e) const { return mn[e]; }
};
template <typename H2> struct RawAcc16 {
    H2 mx[4], mn[4];
    __device__ void add(const uint4 &v)
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const H2 h = *reinterpret_cast<const H2 *>(&w[i]);
            mx[i] = __hmax2(mx[i], h);
            mn[i] = __hmin2(mn[i], h);
        }
    }
};
template <> struct RawAcc<__nv_bfloat16> : RawAcc16<__nv_bfloat162> {
    __device__ void init()
    {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(-INFINITY, -INFINITY);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(INFINITY, INFINITY);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            mx[i] = lo;
            mn[i] = hi;
        }
    }
    __device__ float get_max(int e) const
    {
        return (e & 1) ? __high2float(mx[e >> 1]) : __low2float(mx[e >> 1]);
    }
    __device__ float get_min(int e) const
    {
        return (e & 1) ? __high2float(mn[e >> 1]) : __low2float(mn[e >> 1]);
    }
};
template <> struct RawAcc<__half> : RawAcc16<__half2> {
    __device__ void init()
    {
        const __half2 lo = __floats2half2_rn(-INFINITY, -INFINITY);
        const __half2 hi = __floats2half2_rn(INFINITY, INFINITY);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            mx[i] = lo;
            mn[i] = hi;
        }
    }
    __device__ float get_max(int e) const
    {
        return (e & 1) ? __high2float(mx[e >> 1]) : __low2float(mx[e >> 1]);
    }
    __device__ float get_min(int e) const
    {
        return (e & 1) ? __high2float(mn[e >> 1]) : __low2float(mn[e >> 1]);
    }
};

template <typename T>
__global__ void __launch_bounds__(256)
    calib_raw_kernel(const T *__restrict__ x, int64_t T_, int C, int64_t rows_per_cta,
                     float *ch_max, float *ch_min)
{
    constexpr int VEC = Elem<T>::VEC;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NCH = C / VEC;
    const int ch = blockIdx.x * 32 + lane;
    const int64_t r0 = (int64_t)blockIdx.y * rows_per_cta;
    const int64_t r1 = r0 + rows_per_cta < T_ ? r0 + rows_per_cta : T_;
    RawAcc<T> acc;
    acc.init();
    if (ch < NCH) {
        const uint4 *base = reinterpret_cast<const uint4 *>(x) + ch;
        int64_t r = r0 + warp;
        // four independent rows in flight per thread
        for (; r + 24 < r1; r += 32) {
            const uint4 a = ldg_stream(base + (r + 0) * NCH);
            const uint4 b = ldg_stream(base + (r + 8) * NCH);
            const uint4 c = ldg_stream(base + (r + 16) * NCH);
            const uint4 d = ldg_stream(base + (r + 24) * NCH);
            acc.add(a);
            acc.add(b);
            acc.add(c);
            acc.add(d);
        }
        for (; r < r1; r += 8) acc.add(ldg_stream(base + r * NCH));
    }
    __shared__ float smx[8][32 * 8], smn[8][32 * 8];
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
        smx[warp][lane * VEC + e] = acc.get_max(e);
        smn[warp][lane * VEC + e] = acc.get_min(e);
    }
    __syncthreads();
    // 32 lanes x VEC channels = 32*VEC columns; thread i < 32*VEC folds column i of the 8 warps
    const int i = threadIdx.x;
    if (i < 32 * VEC) {
        const int c = (blockIdx.x * 32) * VEC + i;
        if (c < C) {
            float m = smx[0][i], n = smn[0][i];
#pragma unroll
            for (int w = 1; w < 8; ++w) {
                m = fmaxf(m, smx[w][i]);
                n = fminf(n, smn[w][i]);
            }
            if (r1 > r0) {
                atomic_max_f32(ch_max + c, m);
                atomic_min_f32(ch_min + c, n);
            }
        }
    }
}

// ---- K/V layout: [B, H, S, D], channel c = h*D + d, statistics over the B*S tokens ------------
// A CTA takes one (b, h) pair and a slice of S; each thread owns 8 consecutive d of one row
// group and strides over the rows; a shared-memory fold over the row groups and integer atomics
// finish the exact max/min.
template <typename T>
__global__ void __launch_bounds__(256)
    kv_calib_kernel(const T *__restrict__ x, int H, int64_t S, int D, int64_t s_per_cta, float *ch_max,
                    float *ch_min)
{
    constexpr int VEC = Elem<T>::VEC;
    constexpr int NLD = 8 / VEC;
    const int bh = blockIdx.x, h = bh % H;
    const int TPR = D / 8, RPI = blockDim.x / TPR;
    const int tl = threadIdx.x % TPR, rr = threadIdx.x / TPR;
    const int64_t s0 = (int64_t)blockIdx.y * s_per_cta;
    const int64_t s1 = s0 + s_per_cta < S ? s0 + s_per_cta : S;
    RawAcc<T> acc[NLD];
#pragma unroll
    for (int l = 0; l < NLD; ++l) acc[l].init();
    if (rr < RPI) {
        const T *base = x + (int64_t)bh * S * D + tl * 8;
        int64_t s = s0 + rr;
        for (; s + 3 * RPI < s1; s += 4 * RPI) {
            uint4 a[4][NLD];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int l = 0; l < NLD; ++l) a[u][l] = ldg_stream(base + (s + u * RPI) * D + l * VEC);
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int l = 0; l < NLD; ++l) acc[l].add(a[u][l]);
        }
        for (; s < s1; s += RPI)
#pragma unroll
            for (int l = 0; l < NLD; ++l) acc[l].add(ldg_stream(base + s * D + l * VEC));
    }
    __shared__ float kmx[256 * 8], kmn[256 * 8];
    if (rr < RPI)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            kmx[rr * D + tl * 8 + i] = acc[i / VEC].get_max(i % VEC);
            kmn[rr * D + tl * 8 + i] = acc[i / VEC].get_min(i % VEC);
        }
    __syncthreads();
    if (s1 <= s0) return;
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
        float m = kmx[d], n = kmn[d];
        for (int r = 1; r < RPI; ++r) {
            m = fmaxf(m, kmx[r * D + d]);
            n = fminf(n, kmn[r * D + d]);
        }
        atomic_max_f32(ch_max + h * D + d, m);
        atomic_min_f32(ch_min + h * D + d, n);
    }
}

// Ring form for 16-bit caches whose shape passes kv_ring_shape_ok (stages of kv_stream.cuh): the
// eight pieces of a stage that a thread reads all hold its channel group, so it keeps one packed
// running max / min.  When the head changes (and at the end) every thread of the CTA flushes:
// the lanes sharing a channel group are folded by shuffles, the warps through a D-wide shared
// buffer (fmx / fmn, integer atomics, exact and order-independent), and the CTA's result goes to
// the outputs with the same integer atomics, one per channel and 32 consecutive channels per warp.
// fmx / fmn hold -inf / +inf on entry and again on return.
template <typename T>
__device__ __forceinline__ void kv_calib_flush(const RawAcc<T> &acc, int h, int D, float *fmx, float *fmn,
                                               float *ch_max, float *ch_min)
{
    const int lane = threadIdx.x & 31, npr = D >> 3, col = threadIdx.x & (npr - 1);
    float m[8], n[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        m[e] = acc.get_max(e);
        n[e] = acc.get_min(e);
    }
    for (int o = npr; o < 32; o <<= 1)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            m[e] = fmaxf(m[e], __shfl_xor_sync(FULL, m[e], o));
            n[e] = fminf(n[e], __shfl_xor_sync(FULL, n[e], o));
        }
    if (lane < npr || npr >= 32)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            atomic_max_f32(fmx + col * 8 + e, m[e]);
            atomic_min_f32(fmn + col * 8 + e, n[e]);
        }
    __syncthreads();
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
        atomic_max_f32(ch_max + h * D + d, fmx[d]);
        atomic_min_f32(ch_min + h * D + d, fmn[d]);
        fmx[d] = -INFINITY;
        fmn[d] = INFINITY;
    }
    __syncthreads();  // the buffer is reset before any thread's next flush
}

constexpr int KVR_BAR_BYTES = 32;  // the ring's KVR_NS mbarriers, rounded up to 16 bytes
static_assert(8 * KVR_NS <= KVR_BAR_BYTES, "ring barriers");

template <typename T>
__global__ void __launch_bounds__(KVR_THREADS, 2)
    kv_calib_ring(const T *__restrict__ x, int B, int H, int SPB, int D, float *ch_max, float *ch_min, int *err)
{
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_abort;
    uint8_t *ring = smem;
    const uint32_t bar0 = smem_u32(smem + (size_t)KVR_NS * KVR_STAGE);
    float *fmx = reinterpret_cast<float *>(smem + (size_t)KVR_NS * KVR_STAGE + KVR_BAR_BYTES), *fmn = fmx + D;
    const int tid = threadIdx.x;
    const int64_t total = (int64_t)B * H * SPB;
    const int64_t j0 = total * blockIdx.x / gridDim.x, j1 = total * (blockIdx.x + 1) / gridDim.x;
    const int n = (int)(j1 - j0);
    if (n <= 0) return;
    KvStagePos prod;  // thread 0: the next stage to load
    auto issue = [&](uint32_t s) {
        const uint8_t *src = reinterpret_cast<const uint8_t *>(x) + prod.mem_index(H, SPB) * KVR_STAGE;
        mbar_expect_tx(bar0 + 8u * s, KVR_STAGE);
        bulk_g2s(smem_u32(ring + (size_t)s * KVR_STAGE), src, KVR_STAGE, bar0 + 8u * s);
        prod.advance(B, H, SPB);
    };
    if (tid == 0) {
        s_abort = 0;
        for (int s = 0; s < KVR_NS; ++s) mbar_init(bar0 + 8u * s, 1);
        fence_mbar_init();
        prod.set(j0, total, B, SPB);
        for (int s = 0; s < KVR_NS && s < n; ++s) issue((uint32_t)s);
    }
    for (int d = tid; d < D; d += KVR_THREADS) {
        fmx[d] = -INFINITY;
        fmn[d] = INFINITY;
    }
    __syncthreads();
    KvStagePos cur;
    cur.set(j0, total, B, SPB);
    RawAcc<T> acc;
    acc.init();
    int acc_h = cur.h;
    uint32_t slot = 0, phase = 0;
    for (int i = 0; i < n; ++i) {
        if (cur.h != acc_h) {  // the same in every thread
            kv_calib_flush<T>(acc, acc_h, D, fmx, fmn, ch_max, ch_min);
            acc.init();
            acc_h = cur.h;
        }
        if (!mbar_wait_bounded(bar0 + 8u * slot, phase, err)) s_abort = 1;
        const uint4 *src = reinterpret_cast<const uint4 *>(ring + (size_t)slot * KVR_STAGE);
        uint4 xb[KVR_PPT];
#pragma unroll
        for (int k = 0; k < KVR_PPT; ++k) xb[k] = src[tid + k * KVR_THREADS];
#pragma unroll
        for (int k = 0; k < KVR_PPT; ++k) acc.add(xb[k]);
        __syncthreads();  // the slot has been read
        if (s_abort) break;
        if (tid == 0 && i + KVR_NS < n) {
            fence_proxy_async_smem();
            issue(slot);
        }
        cur.advance(B, H, SPB);
        if (++slot == KVR_NS) {
            slot = 0;
            phase ^= 1u;
        }
    }
    kv_calib_flush<T>(acc, acc_h, D, fmx, fmn, ch_max, ch_min);
}

// ---- LayerNorm mode ------------------------------------------------------------------------
template <typename T, int CPT>
__global__ void __launch_bounds__(512, 1)
    calib_ln_kernel(const T *__restrict__ x, int64_t T_, int C, const float *__restrict__ gamma,
                    const float *__restrict__ beta, float eps, float *ch_max, float *ch_min, int NS,
                    int *err)
{
    constexpr int VEC = Elem<T>::VEC;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, NT = blockDim.x;
    const int NCH = C / VEC;
    const uint32_t rowbytes = (uint32_t)C * sizeof(T);
    const QuadSmem L = quad_smem_layout(NS, rowbytes, 2 * 8 * 32 * 4);
    float *red = reinterpret_cast<float *>(smem + L.extra_off);
    float *red2 = red + 8 * 32;
    __shared__ int s_abort;
    QuadRows<T, CPT> pipe{x, T_, C, NCH, NS, rowbytes, smem, smem_u32(smem + L.bar_off), err, &s_abort};
    pipe.start();
    __syncthreads();

    float tmax[CPT][VEC], tmin[CPT][VEC];
#pragma unroll
    for (int k = 0; k < CPT; ++k)
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            tmax[k][e] = -INFINITY;
            tmin[k][e] = INFINITY;
        }
    int64_t lq = 0;
    for (int64_t gq = blockIdx.x; 4 * gq < T_; gq += gridDim.x, ++lq) {
        const int nrows = (int)(T_ - 4 * gq < 4 ? T_ - 4 * gq : 4);
        uint4 xr[4][CPT];
        pipe.load(nrows, xr);
        float rstd[4], nmr[4], sub[4];
        const bool offs = quad_stats<T, CPT>(xr, C, NCH, eps, red, red2, pipe, lq, rstd, nmr, sub);
        if (pipe.aborted()) {  // a row never arrived: stop here (the error word is set)
            pipe.drain(lq);
            return;
        }
        if (nrows == 4 && !offs) {  // normalised values of tokens (0, 1) and (2, 3) two lanes at a time
            const f32x2 rs01 = mk2(rstd[0], rstd[1]), rs23 = mk2(rstd[2], rstd[3]);
            const f32x2 nm01 = mk2(nmr[0], nmr[1]), nm23 = mk2(nmr[2], nmr[3]);
#pragma unroll
            for (int k = 0; k < CPT; ++k)
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    const f32x2 t01 = fma2(mk2(Elem<T>::get(xr[0][k], e), Elem<T>::get(xr[1][k], e)), rs01, nm01);
                    const f32x2 t23 = fma2(mk2(Elem<T>::get(xr[2][k], e), Elem<T>::get(xr[3][k], e)), rs23, nm23);
                    tmax[k][e] = max3f(max3f(tmax[k][e], lo2(t01), hi2(t01)), lo2(t23), hi2(t23));
                    tmin[k][e] = min3f(min3f(tmin[k][e], lo2(t01), hi2(t01)), lo2(t23), hi2(t23));
                }
        } else {  // a partial quad, or one with an offset row (x - sub is exact; see quad_stats)
#pragma unroll
            for (int k = 0; k < CPT; ++k)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    if (r >= nrows) break;
#pragma unroll
                    for (int e = 0; e < VEC; ++e) {
                        const float t = fmaf(Elem<T>::get(xr[r][k], e) - sub[r], rstd[r], nmr[r]);
                        tmax[k][e] = fmaxf(tmax[k][e], t);
                        tmin[k][e] = fminf(tmin[k][e], t);
                    }
                }
        }
        pipe.advance();
    }
    if (lq == 0) return;  // this CTA saw no rows
    // The CTA's extremes pass through shared memory so that the atomics of a warp cover 32
    // consecutive channels (from registers, a thread's VEC consecutive channels would spread
    // them VEC words apart over VEC times as many lines).  The ring is idle here: every row
    // copied into it has been read, and its 4 or more rows of C values hold the 2 C floats.
    __syncthreads();
    float *shi = reinterpret_cast<float *>(smem), *slo = shi + C;
#pragma unroll
    for (int k = 0; k < CPT; ++k) {
        const int ch = tid + k * NT;
        if (ch >= NCH) continue;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            const int c = ch * VEC + e;
            const float gm = gamma[c], bt = beta[c];
            shi[c] = fmaf(gm >= 0.f ? tmax[k][e] : tmin[k][e], gm, bt);
            slo[c] = fmaf(gm >= 0.f ? tmin[k][e] : tmax[k][e], gm, bt);
        }
    }
    __syncthreads();
    for (int c = tid; c < C; c += NT) {
        atomic_max_f32(ch_max + c, shi[c]);
        atomic_min_f32(ch_min + c, slo[c]);
    }
}

__device__ __forceinline__ float to_float(float v) { return v; }
__device__ __forceinline__ float to_float(__half v) { return __half2float(v); }
__device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }

// LayerNorm mode, general shapes (any C % 8 == 0 the quad kernel cannot hold in registers):
// one row at a time in shared memory as fp32, two-pass statistics, running max/min of the
// normalised value per channel in shared memory.
template <typename T>
__global__ void __launch_bounds__(256)
    calib_ln_simple_kernel(const T *__restrict__ x, int64_t T_, int C, const float *__restrict__ gamma,
                           const float *__restrict__ beta, float eps, float *ch_max, float *ch_min)
{
    extern __shared__ __align__(16) float csm[];
    float *xs = csm, *tmx = csm + C, *tmn = csm + 2 * (size_t)C;
    __shared__ float red[8 * 8];
    const int tid = threadIdx.x, NT = blockDim.x;
    for (int c = tid; c < C; c += NT) {
        tmx[c] = -INFINITY;
        tmn[c] = INFINITY;
    }
    for (int64_t t = blockIdx.x; t < T_; t += gridDim.x) {
        const T *xr = x + t * (int64_t)C;
        float s = 0.f;
        for (int c = tid; c < C; c += NT) {
            const float v = to_float(xr[c]);
            xs[c] = v;
            s += v;
        }
        float v8[8] = {s, 0, 0, 0, 0, 0, 0, 0};
        cta_sum8(v8, red);
        float hi, rstd, nmr;
        row_moments(xs, C, v8[0], eps, red, hi, rstd, nmr);
        for (int c = tid; c < C; c += NT) {
            const float tv = fmaf(xs[c] - hi, rstd, nmr);
            tmx[c] = fmaxf(tmx[c], tv);
            tmn[c] = fminf(tmn[c], tv);
        }
        __syncthreads();  // xs and red are rewritten by the next row
    }
    if ((int64_t)blockIdx.x >= T_) return;
    for (int c = tid; c < C; c += NT) {
        const float gm = gamma[c], bt = beta[c];
        atomic_max_f32(ch_max + c, fmaf(gm >= 0.f ? tmx[c] : tmn[c], gm, bt));
        atomic_min_f32(ch_min + c, fmaf(gm >= 0.f ? tmn[c] : tmx[c], gm, bt));
    }
}


// ---- host launchers ---------------------------------------------------------------------------

template <typename T>
static cudaError_t launch_raw_t(const CalibArgs &a)
{
    constexpr int VEC = Elem<T>::VEC;
    const int NCH = a.C / VEC;
    const int gx = (NCH + 31) / 32;
    // about 8 CTAs of 256 threads per SM in total, each with at least 64 rows
    int64_t gy = std::max<int64_t>(1, ((int64_t)a.num_sms * 8 + gx - 1) / gx);
    gy = std::min<int64_t>(gy, std::max<int64_t>(1, a.T / 64));
    gy = std::min<int64_t>(gy, 65535);
    const int64_t rows_per_cta = (a.T + gy - 1) / gy;
    gy = (a.T + rows_per_cta - 1) / rows_per_cta;
    calib_raw_kernel<T><<<dim3(gx, (unsigned)gy), 256, 0, a.stream>>>((const T *)a.x, a.T, a.C,
                                                                       rows_per_cta, a.ch_max, a.ch_min);
    return cudaGetLastError();
}

template <typename T, int CPT>
static cudaError_t launch_ln_t(const CalibArgs &a, int NT, int NS)
{
    const uint32_t rowbytes = (uint32_t)a.C * sizeof(T);
    const QuadSmem L = quad_smem_layout(NS, rowbytes, 2 * 8 * 32 * 4);
    auto kern = calib_ln_kernel<T, CPT>;
    cudaError_t e = kernel_smem((const void *)kern, L.total);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = kernel_occupancy(&per_sm, (const void *)kern, NT, L.total);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t quads = (a.T + 3) / 4;
    const int64_t grid = std::min<int64_t>(quads, (int64_t)per_sm * a.num_sms);
    kern<<<(unsigned)grid, NT, L.total, a.stream>>>((const T *)a.x, a.T, a.C, a.gamma, a.beta, a.eps,
                                                    a.ch_max, a.ch_min, NS, a.err);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_ln_simple(const CalibArgs &a)
{
    const size_t smem = (size_t)a.C * 12;
    if (smem > (size_t)a.max_smem) return cudaErrorInvalidValue;
    auto kern = calib_ln_simple_kernel<T>;
    cudaError_t e = kernel_smem((const void *)kern, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = kernel_occupancy(&per_sm, (const void *)kern, 256, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t grid = std::min<int64_t>(a.T, (int64_t)per_sm * a.num_sms);
    kern<<<(unsigned)grid, 256, smem, a.stream>>>((const T *)a.x, a.T, a.C, a.gamma, a.beta, a.eps,
                                                  a.ch_max, a.ch_min);
    return cudaGetLastError();
}

template <typename T, int CPT>
static int ln_calib_per_sm(int NT, size_t smem)
{
    int per_sm = 0;
    if (kernel_smem((const void *)calib_ln_kernel<T, CPT>, smem) !=
            cudaSuccess ||
        kernel_occupancy(&per_sm, (const void *)calib_ln_kernel<T, CPT>, NT, smem) != cudaSuccess)
        return 0;
    return per_sm;
}

template <typename T>
static cudaError_t launch_ln_d(const CalibArgs &a)
{
    constexpr int VEC = Elem<T>::VEC;
    const int NCH = a.C / VEC;
    // fewest chunks per thread that keep the CTA within `lim` threads
    auto pick = [&](int lim, int &cpt, int &nt) {
        cpt = nt = 0;
        for (int k = 1; k <= 4; ++k) {
            const int n = ((NCH + k - 1) / k + 31) / 32 * 32;
            if (n <= lim) {
                cpt = k;
                nt = n;
                return;
            }
        }
    };
    const uint32_t rowbytes = (uint32_t)a.C * sizeof(T);
    int ns = 0;
    for (int s = 8; s >= 4; --s)
        if (quad_smem_layout(s, rowbytes, 2 * 8 * 32 * 4).total <= (size_t)a.max_smem) {
            ns = s;
            break;
        }
    int cpt, nt;
    pick(512, cpt, nt);
    if (!cpt || !ns) return launch_ln_simple<T>(a);
    // Short rows are latency-bound: two CTAs of at most 256 threads (two independent row
    // pipelines per SM) measured 49% -> 74% of the HBM copy rate at C = 4096 (fp16).  Taken only
    // when the occupancy query confirms two CTAs per SM (at 4 chunks per thread the registers
    // allow one, and one 256-thread CTA ran slower than one of 512).
    int c2, n2;
    pick(256, c2, n2);
    if (c2 && c2 < 4) {
        const size_t smem = quad_smem_layout(ns, rowbytes, 2 * 8 * 32 * 4).total;
        const int per_sm = c2 == 1 ? ln_calib_per_sm<T, 1>(n2, smem)
                           : c2 == 2 ? ln_calib_per_sm<T, 2>(n2, smem)
                                     : ln_calib_per_sm<T, 3>(n2, smem);
        if (per_sm >= 2) {
            cpt = c2;
            nt = n2;
        }
    }
    switch (cpt) {
    case 1: return launch_ln_t<T, 1>(a, nt, ns);
    case 2: return launch_ln_t<T, 2>(a, nt, ns);
    case 3: return launch_ln_t<T, 3>(a, nt, ns);
    default: return launch_ln_t<T, 4>(a, nt, ns);
    }
}

cudaError_t launch_calib(const CalibArgs &a)
{
    if (!a.accumulate) {
        calib_init_kernel<<<(a.C + 255) / 256, 256, 0, a.stream>>>(a.ch_max, a.ch_min, a.C);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (a.T == 0) return cudaSuccess;
    if (a.gamma) {
        switch (a.dtype) {
        case RPTQ_F32: return launch_ln_d<float>(a);
        case RPTQ_F16: return launch_ln_d<__half>(a);
        default: return launch_ln_d<__nv_bfloat16>(a);
        }
    }
    switch (a.dtype) {
    case RPTQ_F32: return launch_raw_t<float>(a);
    case RPTQ_F16: return launch_raw_t<__half>(a);
    default: return launch_raw_t<__nv_bfloat16>(a);
    }
}

template <typename T>
static cudaError_t launch_kv_calib_ring(const KvCalibArgs &a)
{
    const int SPB = (int)(a.S / kv_ring_rows(a.D));
    auto kern = kv_calib_ring<T>;
    // the stage ring, its barriers and the CTA's D-wide max / min fold buffer
    const size_t smem = (size_t)KVR_NS * KVR_STAGE + KVR_BAR_BYTES + 8 * (size_t)a.D;
    cudaError_t e = kernel_smem((const void *)kern, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = kernel_occupancy(&per_sm, (const void *)kern, KVR_THREADS, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t total = (int64_t)a.B * a.H * SPB;
    const int64_t grid = std::min<int64_t>((int64_t)per_sm * a.num_sms, total);
    kern<<<(unsigned)grid, KVR_THREADS, smem, a.stream>>>((const T *)a.x, a.B, a.H, SPB, a.D, a.ch_max, a.ch_min,
                                                          a.err);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_kv_calib_t(const KvCalibArgs &a)
{
    if constexpr (sizeof(T) == 2)
        if (kv_ring_shape_ok(a.B, a.H, a.S, a.D, 2)) return launch_kv_calib_ring<T>(a);
    const int nbh = a.B * a.H;
    int64_t gy = std::max<int64_t>(1, ((int64_t)a.num_sms * 6 + nbh - 1) / nbh);
    gy = std::min<int64_t>(gy, std::max<int64_t>(1, a.S / 64));
    gy = std::min<int64_t>(gy, 65535);
    const int64_t per = (a.S + gy - 1) / gy;
    gy = (a.S + per - 1) / per;
    kv_calib_kernel<T><<<dim3((unsigned)nbh, (unsigned)gy), 256, 0, a.stream>>>((const T *)a.x, a.H, a.S, a.D,
                                                                                per, a.ch_max, a.ch_min);
    return cudaGetLastError();
}

cudaError_t launch_kv_calib(const KvCalibArgs &a)
{
    if (!a.accumulate) {
        calib_init_kernel<<<(a.H * a.D + 255) / 256, 256, 0, a.stream>>>(a.ch_max, a.ch_min, a.H * a.D);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (a.B == 0 || a.S == 0) return cudaSuccess;
    switch (a.dtype) {
    case RPTQ_F32: return launch_kv_calib_t<float>(a);
    case RPTQ_F16: return launch_kv_calib_t<__half>(a);
    default: return launch_kv_calib_t<__nv_bfloat16>(a);
    }
}

}  // namespace rptq
