// row_pipeline.cuh -- token-row staging and LayerNorm statistics shared by the fused
// LN-reorder-quant kernel and the LayerNorm-mode calibration kernel.
//
// A CTA owns a fixed set of 16-byte chunks of the channel axis (chunk tid + k*NT, k < CPT) and
// walks token rows four at a time ("quads": rows 4q .. 4q+3 of its grid-stride sequence).
// Rows arrive in a ring of NS shared-memory slots through bulk asynchronous copies (one copy
// per row, issued by thread 0, completion on one mbarrier per slot; never multicast).  Each
// quad is read once into registers; right after the first CTA-wide reduction the four slots
// are refilled with the rows NS positions ahead, so the copies overlap the rest of the quad.
//
// LayerNorm statistics (standard LayerNorm of OPT-style models: mean and biased variance over
// the C channels): single-pass fp32 sums of x and x^2, reduced in a fixed order; a quad with a
// row whose squared mean exceeds its variance (where the single-pass form loses accuracy) is
// recomputed with the two-pass form sum((x - mean)^2).
#pragma once

#include "common.cuh"

namespace rptq {

template <typename T, int CPT>
struct QuadRows {
    static constexpr int VEC = Elem<T>::VEC;

    const T *x;
    int64_t T_;
    int C, NCH, NS;
    uint32_t rowbytes;
    uint8_t *ring;      // NS * rowbytes, 128-byte aligned
    uint32_t bar0;      // shared address of NS consecutive 8-byte mbarriers
    int *err;
    int *abort;         // shared flag: a wait of this CTA ran out (set in load, read after a barrier)
    // ring position of the current quad's first row, kept incrementally (no divisions):
    // slot = (4 lq) mod NS and phase parity = ((4 lq) / NS) mod 2
    uint32_t slot = 0, phase = 0;

    __device__ __forceinline__ int64_t row_of(int64_t local) const
    {
        // local row i -> quad i/4 of this CTA's grid-stride sequence, row i%4 of that quad
        const int64_t q = (int64_t)blockIdx.x + (local >> 2) * (int64_t)gridDim.x;
        return 4 * q + (local & 3);
    }
    // thread 0 only: local row `local` into ring slot `s`
    __device__ __forceinline__ void issue(int64_t local, uint32_t s) const
    {
        const int64_t row = row_of(local);
        if (row >= T_) return;
        const uint32_t bar = bar0 + 8u * s;
        mbar_expect_tx(bar, rowbytes);
        bulk_g2s(smem_u32(ring + (size_t)s * rowbytes), x + row * (int64_t)C, rowbytes, bar);
    }
    // thread 0: barriers + first NS rows.  Caller must __syncthreads() before any wait.
    __device__ __forceinline__ void start() const
    {
        if (threadIdx.x == 0) {
            *abort = 0;
            for (int s = 0; s < NS; ++s) mbar_init(bar0 + 8u * s, 1);
            fence_mbar_init();
            for (int s = 0; s < NS; ++s) issue(s, (uint32_t)s);
        }
    }
    // ring slot and phase parity of row r (< 4) of the current quad
    __device__ __forceinline__ void where(int r, uint32_t &s, uint32_t &ph) const
    {
        s = slot + r;
        ph = phase;
        if (s >= (uint32_t)NS) {
            s -= NS;
            ph ^= 1u;
        }
    }
    // Wait for the current quad (rows < nrows valid) and copy this thread's chunks into registers.
    __device__ __forceinline__ void load(int nrows, uint4 (&xr)[4][CPT]) const
    {
        const int tid = threadIdx.x, NT = blockDim.x;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            uint32_t s, ph;
            where(r, s, ph);
            if (r < nrows && !mbar_wait_bounded(bar0 + 8u * s, ph, err)) *abort = 1;
            const uint4 *src = reinterpret_cast<const uint4 *>(ring + (size_t)s * rowbytes);
#pragma unroll
            for (int k = 0; k < CPT; ++k) {
                const int ch = tid + k * NT;
                xr[r][k] = (r < nrows && ch < NCH) ? src[ch] : make_uint4(0, 0, 0, 0);
            }
        }
    }
    // Whether a wait of the current quad ran out: the same answer in every thread once a barrier
    // separates it from load().  The caller then stops (after drain()) instead of refilling.
    __device__ __forceinline__ bool aborted() const { return *(volatile int *)abort != 0; }
    // thread 0 after an abort: wait (bounded) for the copies still in flight into the ring, the
    // rows of the current quad and the NS - 4 rows after them, so none lands after the CTA exits
    __device__ __forceinline__ void drain(int64_t lq) const
    {
        if (threadIdx.x != 0) return;
        uint32_t s = slot, ph = phase;
        for (int i = 0; i < NS; ++i) {
            if (row_of(4 * lq + i) < T_) mbar_wait_bounded(bar0 + 8u * s, ph, err);
            if (++s == (uint32_t)NS) {
                s = 0;
                ph ^= 1u;
            }
        }
    }
    // thread 0 after the quad's last read of its slots r0 .. r1-1: refill them with the rows NS
    // ahead (nothing once the CTA has aborted)
    __device__ __forceinline__ void refill(int64_t lq, int r0 = 0, int r1 = 4) const
    {
        if (threadIdx.x == 0 && !aborted()) {
            fence_proxy_async_smem();
            for (int r = r0; r < r1; ++r) {
                uint32_t s, ph;
                where(r, s, ph);
                issue(4 * lq + NS + r, s);  // the same slot, NS rows later
            }
        }
    }
    // all threads, at the end of every quad
    __device__ __forceinline__ void advance()
    {
        slot += 4;
        if (slot >= (uint32_t)NS) {
            slot -= NS;
            phase ^= 1u;
        }
    }
};

// LayerNorm statistics of the four rows in xr.  The normalised value of x is
// fmaf(x - sub[r], rstd[r], nmr[r]); returns whether any row of the quad needs the subtraction
// (the same answer in every thread).  A row whose mean is small against its spread
// (mean^2 <= var) takes the single-pass moments, sub = 0 and nmr = -mean*rstd.  Otherwise
// (a large common offset, or a constant row) the single-pass variance cancels and the rounding
// of -mean*rstd alone would move every value of the row together, so the row is redone from
// d = x - m0 (m0 = sum / C, correctly rounded): sum(d) refines the mean to the pair
// sub + lo (sub = fl(m0 + sum(d)/C)), var = sum(d^2)/C - (sum(d)/C)^2, nmr = -lo*rstd; x - sub
// is exact for x near the mean, so the offset never meets a rounding.
// `red`, `red2`: 8*(NT/32) floats each.  With refill_now, calls refill() between its first
// barrier and any later one (the caller refills later when it still uses the quad's ring slots).
// NT_: the CTA's thread count when the caller knows it at compile time (0: blockDim.x).
template <typename T, int CPT, typename Pipe>
__device__ __forceinline__ bool quad_stats(const uint4 (&xr)[4][CPT], int C, int NCH, float eps,
                                           float *red, float *red2, const Pipe &pipe, int64_t lq,
                                           float (&rstd)[4], float (&nmr)[4], float (&sub)[4],
                                           bool refill_now = true, int NT_ = 0)
{
    constexpr int VEC = Elem<T>::VEC;
    const int tid = threadIdx.x, NT = NT_ ? NT_ : (int)blockDim.x;
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
    // chunks beyond the row were loaded as zeros and add nothing
#pragma unroll
    for (int k = 0; k < CPT; ++k)
#pragma unroll
        for (int r = 0; r < 4; ++r) chunk_moments<T>(xr[r][k], v[r], v[4 + r]);
    cta_sum8(v, red, NT >> 5);  // every thread is past its reads of this quad's ring slots
    if (refill_now) pipe.refill(lq);
    const float invC = 1.0f / (float)C;
    float mean[4], var[4];
    bool ill[4], any = false;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        mean[r] = v[r] * invC;
        var[r] = v[4 + r] * invC - mean[r] * mean[r];
        ill[r] = !(mean[r] * mean[r] <= var[r]);
        any |= ill[r];
        sub[r] = 0.f;
    }
    if (any) {
        float m0[4], w[8];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            m0[r] = __fdiv_rn(v[r], (float)C);
            w[r] = 0.f;
            w[4 + r] = 0.f;
        }
#pragma unroll
        for (int k = 0; k < CPT; ++k) {
            if (tid + k * NT < NCH) {
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int e = 0; e < VEC; ++e) {
                        const float d = Elem<T>::get(xr[r][k], e) - m0[r];
                        w[r] += d;
                        w[4 + r] = fmaf(d, d, w[4 + r]);
                    }
            }
        }
        cta_sum8(w, red2, NT >> 5);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            if (!ill[r]) continue;
            const float delta = w[r] * invC;
            const float hi = m0[r] + delta;
            mean[r] = delta - (hi - m0[r]);  // the low part of the mean pair (hi, mean)
            sub[r] = hi;
            var[r] = fmaf(-delta, delta, w[4 + r] * invC);
        }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        rstd[r] = rsqrtf(fmaxf(var[r], 0.f) + eps);
        nmr[r] = -mean[r] * rstd[r];
    }
    return any;
}

// LayerNorm statistics of one row held in shared memory (xs[0..C), every thread of the CTA,
// `sum` = the CTA's reduced sum of the row): the mean as the pair hi + lo (hi = fl(m0 + delta),
// m0 = sum / C, delta = sum(x - m0) / C) and the variance from the same deviations, so
// fmaf(x - hi, rstd, nmr) with nmr = -lo*rstd stays exact for rows with a large common offset.
// `red`: 64 floats, reused after a barrier.
__device__ __forceinline__ void row_moments(const float *xs, int C, float sum, float eps, float *red,
                                            float &hi, float &rstd, float &nmr)
{
    const float m0 = __fdiv_rn(sum, (float)C);
    float sd = 0.f, ss = 0.f;
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        const float d = xs[c] - m0;
        sd += d;
        ss = fmaf(d, d, ss);
    }
    float w8[8] = {sd, ss, 0, 0, 0, 0, 0, 0};
    __syncthreads();  // red is reused
    cta_sum8(w8, red);
    const float delta = w8[0] / (float)C;
    hi = m0 + delta;
    const float lo = delta - (hi - m0);
    const float var = fmaf(-delta, delta, w8[1] / (float)C);
    rstd = rsqrtf(fmaxf(var, 0.f) + eps);
    nmr = -lo * rstd;
}

// Dynamic shared memory of a quad pipeline: ring + extra bytes, with 128-byte alignment.
struct QuadSmem {
    size_t ring_off, extra_off, bar_off, total;
};
__host__ __device__ inline QuadSmem quad_smem_layout(int NS, uint32_t rowbytes, size_t extra)
{
    QuadSmem s;
    auto up = [](size_t v) { return (v + 127) & ~(size_t)127; };
    s.ring_off = 0;
    s.extra_off = up((size_t)NS * rowbytes);
    s.bar_off = up(s.extra_off + extra);
    s.total = s.bar_off + 8 * (size_t)NS;
    return s;
}

}  // namespace rptq
