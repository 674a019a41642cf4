// kv_quant.cu -- per-cluster quantization of the attention K/V cache.
//
// RPTQ article (基于重排序的新量化方法RPTQ…), results paragraph: the W4A4KV / W4A3KV / W3A3KV
// settings quantize the key and value caches alone, with the same per-cluster asymmetric
// quantizer as the activations (text after Fig. 2; quantization-basics article, section 1.3).
//
// The cache keeps its [B, H, S, D] layout; channel c = h*D + d carries the cluster id of
// channel c.  A thread owns DPT consecutive channels of a row; all rows of one (b, h) block share
// the same D channels, so the thread's coefficients (s, 1/s and the code-domain clamp) serve a
// whole run of rows.  Per element: a correctly rounded x / s, the clamp, the rounding constant
// 1.5*2^23 (which leaves the code in the low bits of the float), and a shifted sum of those bit
// patterns minus a known constant is the packed word; rows are stored as whole words.
// Ring kernel (16-bit caches cut into whole 32-KB stages, kv_stream.cuh): the default shape.
// Warp kernel (D/DPT divides 32): a work unit is 64 rows of one (b, h) block; units are ordered
// (h, b, chunk) and every warp of a one-wave grid takes a contiguous range of them, reloading its
// coefficients only when the head changes.  CTA kernel
// (other D): one CTA per (b, h) block.
#include <algorithm>

#include "../../include/rptq_testing.h"
#include "kv_stream.cuh"
#include "launch.h"

namespace rptq {

// Correctly rounded x / s from r = RN(1/s): q0 = RN(x r), the residual x - q0 s is exact in
// one fused multiply-add, and q0 + residual * r rounds to RN(x / s) (P. Markstein, "IA-64 and
// Elementary Functions", 2000, division by a reciprocal with one correction).  Quotients that
// are exact half-integers therefore stay exact and round half-to-even like the reference.  The
// residual is exact as long as it is not subnormal: for |x| >= 2^-100 the quotient of every
// finite bf16 or fp16 x is the IEEE one (checked exhaustively by the tests); below, the code is
// decided by rint of a quotient far below 1/2 and does not depend on its last bit.
// The quantizer forms x / (s 2^24) with s' = s 2^24 and r' = RN(1/s) 2^-24 (powers of two: the
// same significands), so that x r' stays finite for every finite x when s >= 2^-24 (no
// inf - inf in the correction), and scales back by 2^24 inside the rounding fma.
__device__ __forceinline__ f32x2 div_rn2(f32x2 x2, f32x2 ns2, f32x2 r2)
{
    const f32x2 q0 = mul2(x2, r2);
    return fma2(fma2(q0, ns2, x2), r2, q0);
}

constexpr int KV_ROWS_PER_UNIT = 64;
constexpr float KV_QSCALE = 16777216.0f;            // 2^24
constexpr float KV_QSCALE_INV = 5.9604644775390625e-08f;  // 2^-24

// Scales s for which the scaled quotient above is exact (no overflow of x r', no overflow or
// subnormal r'); other clusters take the IEEE division.
__device__ __forceinline__ bool kv_fast_scale(float s) { return s >= 0x1p-24f && s <= 0x1p+102f; }

// Coefficients of a thread's DPT channels (h*D + d0 + i) for one head.
template <int BITS, int DPT>
struct KvCoef {
    static constexpr int NG = DPT / 8;
    static constexpr int QMAX = (1 << BITS) - 1;
    static constexpr uint32_t MAGIC_BITS = 0x4B400000u;
    f32x2 ns2[DPT / 2], r2[DPT / 2];  // -s 2^24 and RN(1/s) 2^-24, two channels per pair
    int32_t lo_[DPT], hi_[DPT];       // clamp of the rounded bit pattern: MAGIC_BITS - z .. + qmax
    uint32_t bias[NG];                // sum_i (MAGIC_BITS - z_i) << (BITS*i): removes the rounding constant
    bool fast;                        // every channel: |z| < 2^21 (q + 1.5*2^23 inside one binade) and a fast scale

    __device__ __forceinline__ void load(const int32_t *cl, const float *sc, const int32_t *zp, int c0, int g,
                                         int *err)
    {
        fast = true;
#pragma unroll
        for (int gi = 0; gi < NG; ++gi) bias[gi] = 0;
#pragma unroll
        for (int i = 0; i < DPT; i += 2) {
            float sv2[2], rv2[2];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                int kc = cl[c0 + i + h2];
                if (kc < 0 || kc >= g) {
                    raise_error(err, RPTQ_DEVERR_CLUSTER_ID);
                    kc = 0;
                }
                const float sv = sc[kc];
                sv2[h2] = sv * KV_QSCALE;
                rv2[h2] = __frcp_rn(sv) * KV_QSCALE_INV;
                const int z = zp[kc];
                lo_[i + h2] = (int32_t)(MAGIC_BITS - (uint32_t)z);
                hi_[i + h2] = (int32_t)(MAGIC_BITS + (uint32_t)QMAX - (uint32_t)z);
                bias[(i + h2) / 8] += (MAGIC_BITS - (uint32_t)z) << (BITS * ((i + h2) % 8));
                fast &= (z > -(1 << 21)) && (z < (1 << 21)) && kv_fast_scale(sv);
            }
            ns2[i / 2] = mk2(-sv2[0], -sv2[1]);
            r2[i / 2] = mk2(rv2[0], rv2[1]);
        }
    }
};

// One code from an IEEE quotient, exactly as the definition: clamp(rint(x / s) + z, 0, qmax)
// (the sum in fp64 is exact for every finite quotient, and an infinite one clamps).
template <int QMAX>
__device__ __forceinline__ uint32_t kv_code_ieee(float x, float s, int z)
{
    const double q = (double)rintf(__fdiv_rn(x, s)) + (double)z;
    return (uint32_t)fmin(fmax(q, 0.0), (double)QMAX);
}

// Codes of one row's DPT channels (x in VEC-element 16-byte chunks) -> NG packed 8-code groups.
template <typename T, int BITS, int DPT>
__device__ __forceinline__ void kv_quant_row(const uint4 *xb, const KvCoef<BITS, DPT> &cf, uint32_t *grp)
{
    constexpr int VEC = Elem<T>::VEC;
    constexpr int NG = DPT / 8;
    const f32x2 magic2 = mk2(MAGIC_RINT, MAGIC_RINT), up2 = mk2(KV_QSCALE, KV_QSCALE);
    if (cf.fast) {
#pragma unroll
        for (int gi = 0; gi < NG; ++gi) {
            uint32_t acc = 0;
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
                const int i = gi * 8 + j;
                // correctly rounded x / (s 2^24) for two channels, then rint(x / s) + 1.5*2^23:
                // the bit pattern is MAGIC_BITS + rint(x / s) while |x / s| < 2^22; beyond, and
                // for an infinite quotient, it falls outside [lo, hi] on the side of its sign,
                // so the integer clamp below is clamp(rint(x/s), -z, qmax - z) + MAGIC_BITS
                const f32x2 x2 = pair_of<T>(xb[i / VEC], (i % VEC) / 2);
                const f32x2 b2 = fma2(div_rn2(x2, cf.ns2[i / 2], cf.r2[i / 2]), up2, magic2);
                const int32_t l0 = min(max((int32_t)__float_as_uint(lo2(b2)), cf.lo_[i]), cf.hi_[i]);
                const int32_t l1 = min(max((int32_t)__float_as_uint(hi2(b2)), cf.lo_[i + 1]), cf.hi_[i + 1]);
                acc += (uint32_t)l0 << (BITS * j);
                acc += (uint32_t)l1 << (BITS * (j + 1));
            }
            grp[gi] = acc - cf.bias[gi];
        }
    } else {  // a huge zero point or an extreme scale: the IEEE division and the definition
#pragma unroll
        for (int gi = 0; gi < NG; ++gi) {
            uint32_t acc = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = gi * 8 + j;
                // s and z back from the coefficients (exact: a power-of-two scale, an integer)
                const float sv = -((i & 1) ? hi2(cf.ns2[i / 2]) : lo2(cf.ns2[i / 2])) * KV_QSCALE_INV;
                const int z = (int)(KvCoef<BITS, DPT>::MAGIC_BITS - (uint32_t)cf.lo_[i]);
                acc |= kv_code_ieee<KvCoef<BITS, DPT>::QMAX>(Elem<T>::get(xb[i / VEC], i % VEC), sv, z) << (BITS * j);
            }
            grp[gi] = acc;
        }
    }
}

template <int BITS, int DPT>
__device__ __forceinline__ void kv_store_row(uint8_t *o, const uint32_t *grp)
{
    constexpr int NG = DPT / 8;
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

struct KvTensors {
    const void *src[2];
    uint8_t *dst[2];
    const int32_t *cl[2];
    const float *sc[2];
    const int32_t *zp[2];
};

// Warp kernel: blockIdx.y = tensor (0 = K, 1 = V); contiguous ranges of (h, b, chunk) units per warp.
template <typename T, int BITS, int DPT>
__global__ void __launch_bounds__(256, 2)
    kv_quant_warp(KvTensors t, int B, int H, int S, int D, int g, int *err)
{
    constexpr int VEC = Elem<T>::VEC;
    constexpr int NLD = DPT / VEC;
    constexpr int NG = DPT / 8;
    constexpr int U = 8;  // warp rows-groups whose loads are in flight together
    const int ti = blockIdx.y;
    const T *src = static_cast<const T *>(t.src[ti]);
    if (src == nullptr) return;
    uint8_t *dst = t.dst[ti];
    const int lane = threadIdx.x & 31;
    const int TPR = D / DPT, RPW = 32 / TPR;  // threads per row, rows per warp step
    const int tl = lane % TPR, lr = lane / TPR, d0 = tl * DPT;
    const int64_t pitch = (int64_t)D * BITS / 8;
    const int nchunk = (S + KV_ROWS_PER_UNIT - 1) / KV_ROWS_PER_UNIT;
    // units in (h, b, chunk) order; warp gw takes the contiguous range [u0, u1), so it crosses
    // at most a few heads and reloads its coefficients only then
    const int64_t units = (int64_t)H * B * nchunk, TW = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t u0 = units * gw / TW, u1 = units * (gw + 1) / TW;
    int64_t hb = u0 / nchunk;  // h * B + b
    int chunk = (int)(u0 - hb * nchunk);
    int h = (int)(hb / B), b = (int)(hb - (int64_t)h * B);
    KvCoef<BITS, DPT> cf;
    int cur_h = -1;
    for (int64_t un = u0; un < u1; ++un) {
        if (h != cur_h) {
            cf.load(t.cl[ti], t.sc[ti], t.zp[ti], h * D + d0, g, err);
            cur_h = h;
        }
        const int64_t bh = (int64_t)b * H + h;
        const int r_lo = chunk * KV_ROWS_PER_UNIT, r_hi = min(S, r_lo + KV_ROWS_PER_UNIT);
        const T *base = src + bh * S * (int64_t)D + d0;
        uint8_t *obase = dst + bh * S * pitch + (int64_t)tl * (DPT * BITS / 8);
        for (int s0 = r_lo + lr; s0 < r_hi; s0 += U * RPW) {
            uint4 xb[U][NLD];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int row = s0 + u * RPW;
#pragma unroll
                for (int l = 0; l < NLD; ++l)
                    xb[u][l] = row < r_hi ? ldg_stream(base + (int64_t)row * D + l * VEC) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int row = s0 + u * RPW;
                if (row >= r_hi) break;
                uint32_t grp[NG];
                kv_quant_row<T, BITS, DPT>(xb[u], cf, grp);
                kv_store_row<BITS, DPT>(obase + (int64_t)row * pitch, grp);
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

// Ring kernel (16-bit caches whose shape passes kv_ring_shape_ok; stages of kv_stream.cuh).
// Each thread turns its eight pieces into codes (piece p's codes sit at p*BITS in the code
// buffer, whatever D is: a stage's codes are 2048*BITS contiguous bytes of the output), and
// thread 0 writes them with one bulk copy from one of two code buffers.
template <int BITS>
constexpr size_t kv_ring_smem() { return (size_t)KVR_NS * KVR_STAGE + 2 * KVR_PIECES * BITS + 8 * KVR_NS; }

template <typename T, int BITS>
__global__ void __launch_bounds__(KVR_THREADS, 2)
    kv_quant_ring(KvTensors t, int nt, int sel0, int sel1, int B, int H, int SPB, int D, int g, int *err)
{
    constexpr uint32_t CBYTES = KVR_PIECES * BITS;  // codes of one stage
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int s_abort;
    uint8_t *ring = smem;
    uint8_t *cbuf = smem + (size_t)KVR_NS * KVR_STAGE;
    const uint32_t bar0 = smem_u32(cbuf + 2 * CBYTES);
    const int tid = threadIdx.x;
    const int64_t per_t = (int64_t)B * H * SPB, total = per_t * nt;
    const int64_t j0 = total * blockIdx.x / gridDim.x, j1 = total * (blockIdx.x + 1) / gridDim.x;
    const int n = (int)(j1 - j0);  // the grid has at least total / 2^31 CTAs
    if (n <= 0) return;
    KvStagePos prod;  // thread 0: the next stage to load
    auto issue = [&](uint32_t s) {
        const int tt = prod.ti ? sel1 : sel0;
        const uint8_t *src = static_cast<const uint8_t *>(t.src[tt]) + prod.mem_index(H, SPB) * KVR_STAGE;
        mbar_expect_tx(bar0 + 8u * s, KVR_STAGE);
        bulk_g2s(smem_u32(ring + (size_t)s * KVR_STAGE), src, KVR_STAGE, bar0 + 8u * s);
        prod.advance(B, H, SPB);
    };
    if (tid == 0) {
        s_abort = 0;
        for (int s = 0; s < KVR_NS; ++s) mbar_init(bar0 + 8u * s, 1);
        fence_mbar_init();
        prod.set(j0, per_t, B, SPB);
        for (int s = 0; s < KVR_NS && s < n; ++s) issue((uint32_t)s);
    }
    __syncthreads();
    KvStagePos cur;
    cur.set(j0, per_t, B, SPB);
    const int col = tid & ((D >> 3) - 1);  // the thread's 8-channel group, the same in every piece
    KvCoef<BITS, 8> cf;
    int cf_key = -1;
    uint32_t slot = 0, phase = 0;
    for (int i = 0; i < n; ++i) {
        const int tt = cur.ti ? sel1 : sel0;
        if (cur.ti * H + cur.h != cf_key) {
            cf.load(t.cl[tt], t.sc[tt], t.zp[tt], cur.h * D + col * 8, g, err);
            cf_key = cur.ti * H + cur.h;
        }
        if (!mbar_wait_bounded(bar0 + 8u * slot, phase, err)) s_abort = 1;
        const uint4 *src = reinterpret_cast<const uint4 *>(ring + (size_t)slot * KVR_STAGE);
        uint4 xb[KVR_PPT];
#pragma unroll
        for (int k = 0; k < KVR_PPT; ++k) xb[k] = src[tid + k * KVR_THREADS];
        uint8_t *cb = cbuf + (i & 1) * CBYTES;
#pragma unroll
        for (int k = 0; k < KVR_PPT; ++k) {
            uint32_t grp[1];
            kv_quant_row<T, BITS, 8>(&xb[k], cf, grp);
            uint8_t *o = cb + (tid + k * KVR_THREADS) * BITS;
            if constexpr (BITS == 4) {
                *reinterpret_cast<uint32_t *>(o) = grp[0];
            } else {
                o[0] = (uint8_t)grp[0];
                o[1] = (uint8_t)(grp[0] >> 8);
                o[2] = (uint8_t)(grp[0] >> 16);
            }
        }
        // the previous stage's code store has finished reading its buffer, which the stage
        // after this one rewrites
        if (tid == 0) bulk_wait_read<0>();
        __syncthreads();  // slot read, codes complete
        if (s_abort) break;
        if (tid == 0) {
            fence_proxy_async_smem();
            bulk_s2g(t.dst[tt] + cur.mem_index(H, SPB) * CBYTES, smem_u32(cb), CBYTES);
            bulk_commit();
            if (i + KVR_NS < n) issue(slot);  // the slot just read, KVR_NS stages later
        }
        cur.advance(B, H, SPB);
        if (++slot == KVR_NS) {
            slot = 0;
            phase ^= 1u;
        }
    }
    if (tid == 0) bulk_wait_all();
}

// CTA kernel: blockIdx.x = b*H + h, blockIdx.y = tensor; the CTA streams all S rows of the block.
template <typename T, int BITS, int DPT>
__global__ void __launch_bounds__(256)
    kv_quant_cta(KvTensors t, int H, int64_t S, int D, int g, int *err)
{
    constexpr int VEC = Elem<T>::VEC;
    constexpr int NLD = DPT / VEC;
    constexpr int NG = DPT / 8;
    constexpr int U = 4;
    const int ti = blockIdx.y;
    const T *src = static_cast<const T *>(t.src[ti]);
    if (src == nullptr) return;
    uint8_t *dst = t.dst[ti];
    const int bh = blockIdx.x, h = bh % H;
    const int TPR = D / DPT;  // threads per row
    const int RPI = blockDim.x / TPR;
    const int tl = threadIdx.x % TPR, rr = threadIdx.x / TPR;
    if (rr >= RPI) return;
    const int d0 = tl * DPT;
    KvCoef<BITS, DPT> cf;
    cf.load(t.cl[ti], t.sc[ti], t.zp[ti], h * D + d0, g, err);
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
            kv_quant_row<T, BITS, DPT>(xb[u], cf, grp);
            kv_store_row<BITS, DPT>(obase + row * pitch, grp);
        }
    }
}

template <typename T, int BITS>
static cudaError_t launch_kv_warp(const KvArgs &a)
{
    constexpr int DPT = 8;
    const KvTensors t{{a.k, a.v}, {a.kq, a.vq}, {a.ck, a.cv}, {a.sk, a.sv}, {a.zk, a.zv}};
    int per_sm = 1;
    if (kernel_occupancy(&per_sm, (const void *)kv_quant_warp<T, BITS, DPT>, 256, 0) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int64_t units = (int64_t)a.B * a.H * ((a.S + KV_ROWS_PER_UNIT - 1) / KV_ROWS_PER_UNIT);
    const int64_t gx = std::max<int64_t>(1, std::min<int64_t>((int64_t)a.num_sms * per_sm / 2, (units + 7) / 8));
    kv_quant_warp<T, BITS, DPT><<<dim3((unsigned)gx, 2), 256, 0, a.stream>>>(t, a.B, a.H, (int)a.S, a.D, a.g, a.err);
    return cudaGetLastError();
}

template <typename T, int BITS, int DPT>
static cudaError_t launch_kv_cta(const KvArgs &a)
{
    // D <= 2048 (checked by the caller) keeps threads-per-row D / DPT <= 256
    const KvTensors t{{a.k, a.v}, {a.kq, a.vq}, {a.ck, a.cv}, {a.sk, a.sv}, {a.zk, a.zv}};
    kv_quant_cta<T, BITS, DPT><<<dim3((unsigned)(a.B * a.H), 2), 256, 0, a.stream>>>(t, a.H, a.S, a.D, a.g, a.err);
    return cudaGetLastError();
}

template <typename T, int BITS>
static cudaError_t launch_kv_ring(const KvArgs &a)
{
    const KvTensors t{{a.k, a.v}, {a.kq, a.vq}, {a.ck, a.cv}, {a.sk, a.sv}, {a.zk, a.zv}};
    int sel[2] = {0, 1}, nt = 0;
    if (a.k) sel[nt++] = 0;
    if (a.v) sel[nt++] = 1;
    const int SPB = (int)(a.S / kv_ring_rows(a.D));
    auto kern = kv_quant_ring<T, BITS>;
    const size_t smem = kv_ring_smem<BITS>();
    cudaError_t e = kernel_smem((const void *)kern, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = kernel_occupancy(&per_sm, (const void *)kern, KVR_THREADS, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t total = (int64_t)a.B * a.H * SPB * nt;
    const int64_t grid = std::min<int64_t>((int64_t)per_sm * a.num_sms, total);
    kern<<<(unsigned)grid, KVR_THREADS, smem, a.stream>>>(t, nt, sel[0], sel[1], a.B, a.H, SPB, a.D, a.g, a.err);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_kv_d(const KvArgs &a)
{
    if constexpr (sizeof(T) == 2)
        if (kv_ring_shape_ok(a.B, a.H, a.S, a.D, 2)) return a.bits == 4 ? launch_kv_ring<T, 4>(a) : launch_kv_ring<T, 3>(a);
    // warp kernel when the 8-channel groups of a row tile a warp evenly (D in 8, 16, ..., 256)
    if (a.D % 8 == 0 && a.D <= 256 && 32 % (a.D / 8) == 0 && a.S <= 0x7fffffffLL)
        return a.bits == 4 ? launch_kv_warp<T, 4>(a) : launch_kv_warp<T, 3>(a);
    if (a.D % 16 == 0) return a.bits == 4 ? launch_kv_cta<T, 4, 16>(a) : launch_kv_cta<T, 3, 16>(a);
    return a.bits == 4 ? launch_kv_cta<T, 4, 8>(a) : launch_kv_cta<T, 3, 8>(a);
}

// ------------------------------------------------------------------------------------------
// Decode-time append: the new tokens [B, H, s_len, D] of one step, quantized exactly as above,
// written at positions s_begin .. s_begin + s_len - 1 of the packed caches [B, H, S_max, D*b/8].
// One thread per 8-channel chunk of a new row (s_len is 1 in decode, so the work is B*H*D/8
// chunks: launch latency and the coefficient gathers dominate, not bandwidth).
template <typename T, int BITS>
__global__ void __launch_bounds__(256)
    kv_append_kernel(KvTensors t, int B, int H, int64_t s_len, int D, int64_t S_max, int64_t s_begin, int g,
                     int *err)
{
    constexpr int VEC = Elem<T>::VEC;
    const int tensor = blockIdx.y;
    if (!t.src[tensor]) return;
    const int cpr = D / 8;  // chunks per row
    const int64_t total = (int64_t)B * H * s_len * cpr;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int c8 = (int)(i % cpr);
        const int64_t row = i / cpr;  // ((b * H + h) * s_len + s)
        const int64_t s = row % s_len, bh = row / s_len;
        const int h = (int)(bh % H);
        KvCoef<BITS, 8> cf;
        cf.load(t.cl[tensor], t.sc[tensor], t.zp[tensor], h * D + c8 * 8, g, err);
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const T *>(t.src[tensor]) + row * D + c8 * 8);
        uint4 xb[8 / VEC];
#pragma unroll
        for (int k = 0; k < 8 / VEC; ++k) xb[k] = ldg_stream(src + k);
        uint32_t grp[1];
        kv_quant_row<T, BITS, 8>(xb, cf, grp);
        uint8_t *o = t.dst[tensor] + (bh * S_max + s_begin + s) * (int64_t)(D * BITS / 8) + c8 * BITS;
        kv_store_row<BITS, 8>(o, grp);
    }
}

template <typename T>
static cudaError_t launch_kv_append_t(const KvAppendArgs &a)
{
    KvTensors t{{a.k, a.v}, {a.kq, a.vq}, {a.ck, a.cv}, {a.sk, a.sv}, {a.zk, a.zv}};
    const int64_t total = (int64_t)a.B * a.H * a.s_len * (a.D / 8);
    const unsigned grid = (unsigned)std::min<int64_t>((total + 255) / 256, (int64_t)a.num_sms * 8);
    const dim3 gd(grid, 2);
    if (a.bits == 4)
        kv_append_kernel<T, 4><<<gd, 256, 0, a.stream>>>(t, a.B, a.H, a.s_len, a.D, a.S_max, a.s_begin, a.g, a.err);
    else
        kv_append_kernel<T, 3><<<gd, 256, 0, a.stream>>>(t, a.B, a.H, a.s_len, a.D, a.S_max, a.s_begin, a.g, a.err);
    return cudaGetLastError();
}

cudaError_t launch_kv_append(const KvAppendArgs &a)
{
    if (a.s_len == 0 || a.B == 0) return cudaSuccess;
    switch (a.dtype) {
    case RPTQ_F32: return launch_kv_append_t<float>(a);
    case RPTQ_F16: return launch_kv_append_t<__half>(a);
    default: return launch_kv_append_t<__nv_bfloat16>(a);
    }
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

// ==========================================================================================
// Testing hook (include/rptq_testing.h): the K/V quantizer's quotient x / s for n values, in the
// packed form the kernels use (even n) and the scalar form of the integer path (last value of
// an odd n).
namespace rptq {
__global__ void kv_quotient_kernel(const float *x, int64_t n, float s, float *q)
{
    const bool fast = kv_fast_scale(s);
    const float r = __frcp_rn(s) * KV_QSCALE_INV, sp = s * KV_QSCALE;
    const f32x2 ns2 = mk2(-sp, -sp), r2 = mk2(r, r), up2 = mk2(KV_QSCALE, KV_QSCALE);
    for (int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x); i < n; i += 2 * (int64_t)gridDim.x * blockDim.x) {
        const float x1 = i + 1 < n ? x[i + 1] : 0.f;
        f32x2 v;
        if (fast)
            v = mul2(div_rn2(mk2(x[i], x1), ns2, r2), up2);
        else
            v = mk2(__fdiv_rn(x[i], s), __fdiv_rn(x1, s));
        q[i] = lo2(v);
        if (i + 1 < n) q[i + 1] = hi2(v);
    }
}
}  // namespace rptq

extern "C" int rptq_testing_kv_quotient(const float *x, int64_t n, float s, float *q, rptq_stream_t stream)
{
    if (n < 0 || !(s > 0.0f) || !(s < INFINITY)) return RPTQ_ERR_INVALID_ARG;
    if (n == 0) return RPTQ_OK;
    if (!x || !q) return RPTQ_ERR_INVALID_ARG;
    const int64_t pairs = (n + 1) / 2;
    const unsigned grid = (unsigned)std::min<int64_t>((pairs + 255) / 256, 4096);
    rptq::kv_quotient_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(x, n, s, q);
    if (cudaGetLastError() != cudaSuccess) return RPTQ_ERR_CUDA;
    return RPTQ_OK;
}

// ==========================================================================================
// The K/V cache in cluster order (rptq_kv_quant_cluster_ordered): the layout variant of the cache
// that stores every token's C = H*D channels (c = h*D + d) in cluster order, as the activation
// codes are stored -- RPTQ article, text after Fig. 2 (the channels of one cluster placed side
// by side, one (s, z) per cluster) and results paragraph (the K/V cache quantized per cluster).
// Output rows [B, S, C*bits/8]; stored column j holds channel R[j] with cluster col_cluster[j].
// The codes are those of the kept layout (the same quotient, rounding and clamp as kv_quant_row
// above), channel for channel.
//
// Persistent CTAs.  Each CTA first builds, in shared memory, the word offset of every channel's
// stored column and the channel's cluster (entries of R outside [0, C) are reported and leave
// the offset at 0, so every store stays inside the code buffer), and the per-cluster quotient
// coefficients.  Per quad of 4 tokens of one b: a thread takes groups of 8 channels of one head
// (16-byte loads, 4 rows apart by D), forms the 4 tokens' codes of each channel into one word and
// stores it at the channel's stored column; after a barrier, threads pack 32 stored columns x 4
// tokens each (the same 8 x 4 packers as the fused activation kernel) and write whole words.
namespace rptq {
namespace {
constexpr int KVO_THREADS = 256;
// per cluster, 16 bytes (one shared-memory load per channel): -s 2^24, RN(1/s) 2^-24 and the
// clamp of the rounded bit pattern, MAGIC_BITS - z .. + qmax; s and z for the IEEE path
struct KvoFast {
    float ns, r;
    int32_t lo, hi;
};
struct KvoSlow {
    float s;
    int32_t z;
};
__host__ __device__ inline size_t kvo_smem_bytes(int C, int g)
{
    return (size_t)C * 4 + ((size_t)g * (sizeof(KvoFast) + sizeof(KvoSlow)) + 15) / 16 * 16 + (size_t)C * 8;
}
}  // namespace

// The code of x in a cluster whose scale and zero point take the fast quotient (kv_fast_scale,
// |z| < 2^21): the same operations as kv_quant_row's fast path
__device__ __forceinline__ uint32_t kvo_code(float x, const KvoFast &k)
{
    const float q0 = x * k.r;
    const float qq = __fmaf_rn(__fmaf_rn(q0, k.ns, x), k.r, q0);  // RN(x / (s 2^24))
    const float b = __fmaf_rn(qq, KV_QSCALE, MAGIC_RINT);           // 1.5*2^23 + rint(x / s)
    const int32_t l = min(max((int32_t)__float_as_uint(b), k.lo), k.hi);
    return (uint32_t)(l - k.lo);
}

template <typename T, int BITS, int GPT, int NT>
__global__ void __launch_bounds__(NT)
    kv_quant_reordered_kernel(const T *__restrict__ kv, int H, int64_t S, int D, int64_t units,
                              const int32_t *__restrict__ R, const int32_t *__restrict__ col_cluster,
                              const float *__restrict__ scale, const int32_t *__restrict__ zero, int g,
                              uint8_t *__restrict__ codes, int *err)
{
    constexpr int VEC = Elem<T>::VEC;  // elements per 16 bytes
    constexpr uint32_t MAGIC_BITS = 0x4B400000u;
    constexpr int QMAX = (1 << BITS) - 1;
    extern __shared__ __align__(16) uint8_t kvo_smem[];
    const int C = H * D, tid = threadIdx.x;
    // [C] per channel c: its stored column j (bits 0-15) and cluster (bits 16-24)
    uint32_t *tab = reinterpret_cast<uint32_t *>(kvo_smem);
    KvoFast *clf = reinterpret_cast<KvoFast *>(tab + C);  // [g]
    KvoSlow *cls = reinterpret_cast<KvoSlow *>(clf + g);                                    // [g]
    // two code buffers used by turns, [C] words each: 4 tokens' codes per stored column (16-byte
    // aligned: read 4 words at a time); with two, one barrier per quad suffices
    uint32_t *cbuf2 = reinterpret_cast<uint32_t *>((reinterpret_cast<uintptr_t>(cls + g) + 15) & ~(uintptr_t)15);

    for (int c = tid; c < C; c += NT) tab[c] = 0;
    bool fast = true;
    for (int k = tid; k < g; k += NT) {
        const float sv = scale[k];
        const int z = zero[k];
        KvoFast e;
        e.ns = -(sv * KV_QSCALE);
        e.r = __frcp_rn(sv) * KV_QSCALE_INV;
        e.lo = (int32_t)(MAGIC_BITS - (uint32_t)z);
        e.hi = (int32_t)(MAGIC_BITS + (uint32_t)QMAX - (uint32_t)z);
        clf[k] = e;
        cls[k] = KvoSlow{sv, z};
        fast &= (z > -(1 << 21)) && (z < (1 << 21)) && kv_fast_scale(sv);
    }
    // every cluster takes the fast quotient, or every element the IEEE division (the same codes)
    const bool all_fast = __syncthreads_and(fast) != 0;
    for (int j = tid; j < C; j += NT) {
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
        tab[c] = (uint32_t)j | ((uint32_t)k << 16);
    }
    __syncthreads();

    const int64_t NQ = (S + 3) / 4, pitch = (int64_t)C * BITS / 8;
    const int NG8 = C / 8, NU = C / 32;
    // the rows of unit u: one bulk L2 prefetch per head (4 consecutive rows of a (b, h) block)
    auto prefetch_unit = [&](int64_t u) {
        if (u >= units) return;
        const int64_t b = u / NQ, s0 = (u - b * NQ) * 4;
        const int nt = (int)min((int64_t)4, S - s0);
        for (int h = tid; h < H; h += NT)
            prefetch_l2(kv + ((b * H + h) * S + s0) * D, (uint32_t)(nt * D * (int)sizeof(T)));
    };
    prefetch_unit(blockIdx.x);
    int par = 0;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x, par ^= 1) {
        const int64_t b = u / NQ, s0 = (u - b * NQ) * 4;
        const int nt = (int)min((int64_t)4, S - s0);
        uint32_t *cbuf = cbuf2 + (size_t)par * C;
        prefetch_unit(u + gridDim.x);
        // every row load of the thread's groups first (GPT groups of 8 channels, 4 tokens each)
        uint4 xv[GPT][4][8 / VEC];
#pragma unroll
        for (int gi = 0; gi < GPT; ++gi) {
            const int i = tid + gi * NT;
            const int c0 = 8 * i, h = c0 / D, d0 = c0 - h * D;
            const T *row = kv + ((b * H + h) * S + s0) * D + d0;
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int v = 0; v < 8 / VEC; ++v)
                    xv[gi][t][v] = (i < NG8 && t < nt) ? __ldg(reinterpret_cast<const uint4 *>(row + (int64_t)t * D) + v)
                                                      : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int gi = 0; gi < GPT; ++gi) {
            const int i = tid + gi * NT;
            if (i >= NG8) continue;
            const int c0 = 8 * i;
            const uint4 (&xg)[4][8 / VEC] = xv[gi];
            const uint4 ta = *reinterpret_cast<const uint4 *>(tab + c0), tb = *reinterpret_cast<const uint4 *>(tab + c0 + 4);
            const uint32_t te[8] = {ta.x, ta.y, ta.z, ta.w, tb.x, tb.y, tb.z, tb.w};
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                const int ka = (int)(te[e] >> 16), kb = (int)(te[e + 1] >> 16);
                uint32_t w0 = 0, w1 = 0;
                if (all_fast) {
                    const KvoFast k0 = clf[ka], k1 = clf[kb];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const f32x2 x2 = pair_of<T>(xg[t][e / VEC], (e % VEC) / 2);
                        w0 |= kvo_code(lo2(x2), k0) << (8 * t);
                        w1 |= kvo_code(hi2(x2), k1) << (8 * t);
                    }
                } else {
                    const KvoSlow k0 = cls[ka], k1 = cls[kb];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const f32x2 x2 = pair_of<T>(xg[t][e / VEC], (e % VEC) / 2);
                        w0 |= kv_code_ieee<QMAX>(lo2(x2), k0.s, k0.z) << (8 * t);
                        w1 |= kv_code_ieee<QMAX>(hi2(x2), k1.s, k1.z) << (8 * t);
                    }
                }
                cbuf[te[e] & 0xFFFFu] = w0;
                cbuf[te[e + 1] & 0xFFFFu] = w1;
            }
        }
        __syncthreads();
        for (int pu = tid; pu < NU; pu += NT) {
            uint32_t o[4][4];  // [group m of 8 stored columns][token]
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                uint32_t w[8];
                const uint4 a = *reinterpret_cast<const uint4 *>(cbuf + 32 * pu + 8 * m);
                const uint4 c4 = *reinterpret_cast<const uint4 *>(cbuf + 32 * pu + 8 * m + 4);
                w[0] = a.x, w[1] = a.y, w[2] = a.z, w[3] = a.w, w[4] = c4.x, w[5] = c4.y, w[6] = c4.z, w[7] = c4.w;
                if constexpr (BITS == 4)
                    pack8x4_a4(w, o[m]);
                else
                    pack8x4_a3(w, o[m]);
            }
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                if (t >= nt) continue;
                uint8_t *dst = codes + (b * S + s0 + t) * pitch + (int64_t)pu * (4 * BITS);
                if constexpr (BITS == 4) {
                    *reinterpret_cast<uint4 *>(dst) = make_uint4(o[0][t], o[1][t], o[2][t], o[3][t]);
                } else {  // four 24-bit groups -> three words
                    uint32_t *d32 = reinterpret_cast<uint32_t *>(dst);
                    d32[0] = o[0][t] | (o[1][t] << 24);
                    d32[1] = (o[1][t] >> 8) | (o[2][t] << 16);
                    d32[2] = (o[2][t] >> 16) | (o[3][t] << 8);
                }
            }
        }
        // no barrier: the next quad fills the other buffer, and the barrier after its scatter
        // comes before this buffer is filled again
    }
}

bool kv_quant_reordered_supported(int H, int D, int g, int max_smem)
{
    const int64_t C = (int64_t)H * D;
    return D >= 8 && D % 8 == 0 && C % 32 == 0 && C <= RPTQ_MAX_CHANNELS && g >= 1 &&
           g <= RPTQ_MAX_CLUSTERS && kvo_smem_bytes((int)C, g) <= (size_t)max_smem;
}

cudaError_t launch_kv_quant_reordered(const KvReorderedArgs &a)
{
    const int64_t units = (int64_t)a.B * ((a.S + 3) / 4);
    if (units == 0) return cudaSuccess;
    const int C = a.H * a.D;
    const size_t smem = kvo_smem_bytes(C, a.g);
    // wide rows (C > 8192) take 1024-thread CTAs (one per SM, by shared memory) so that every SM
    // keeps 32 warps; narrower ones 256-thread CTAs, several per SM; groups of 8 channels per
    // thread rounded up to a compiled count
    const bool wide = C > 8192;
    const int nt = wide ? 1024 : KVO_THREADS;
    const int gpt = (C / 8 + nt - 1) / nt;
    auto pick = [&](auto k1, auto k2, auto k4, auto k8, auto w2) {
        return wide ? (const void *)w2
                    : gpt <= 1 ? (const void *)k1 : gpt <= 2 ? (const void *)k2 : gpt <= 4 ? (const void *)k4 : (const void *)k8;
    };
#define KVO_PICK(T_, B_)                                                                                     \
    pick(kv_quant_reordered_kernel<T_, B_, 1, KVO_THREADS>, kv_quant_reordered_kernel<T_, B_, 2, KVO_THREADS>, \
         kv_quant_reordered_kernel<T_, B_, 4, KVO_THREADS>, kv_quant_reordered_kernel<T_, B_, 8, KVO_THREADS>, \
         kv_quant_reordered_kernel<T_, B_, 2, 1024>)
    const void *kern = nullptr;
    if (a.dtype == 0)
        kern = a.bits == 4 ? KVO_PICK(float, 4) : KVO_PICK(float, 3);
    else if (a.dtype == 1)
        kern = a.bits == 4 ? KVO_PICK(__half, 4) : KVO_PICK(__half, 3);
    else
        kern = a.bits == 4 ? KVO_PICK(__nv_bfloat16, 4) : KVO_PICK(__nv_bfloat16, 3);
#undef KVO_PICK
    cudaError_t e = kernel_smem(kern, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 1;
    e = kernel_occupancy(&per_sm, kern, nt, smem);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<int64_t>(units, (int64_t)a.num_sms * std::max(1, per_sm));
    int H = a.H, D = a.D, g = a.g;
    int64_t S = a.S, U = units;
    void *args[] = {(void *)&a.kv, (void *)&H, (void *)&S, (void *)&D, (void *)&U, (void *)&a.R,
                    (void *)&a.col_cluster, (void *)&a.scale, (void *)&a.zero, (void *)&g, (void *)&a.codes, (void *)&a.err};
    return cudaLaunchKernel(kern, dim3((unsigned)grid), dim3(nt), args, smem, a.stream);
}

}  // namespace rptq
