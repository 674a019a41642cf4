// common.cuh -- device helpers shared by the RPTQ kernels (sm_100a only).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/rptq.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "librptq is written for sm_100a (B200) only"
#endif

namespace rptq {

constexpr unsigned FULL = 0xffffffffu;
// Adding 1.5 * 2^23 to a float in [0, 2^22) rounds it to the nearest integer (ties to even)
// and leaves that integer in the low mantissa bits: bits = 0x4B400000 + n.
constexpr float MAGIC_RINT = 12582912.0f;

// Sticky device error word: kernels OR RPTQ_DEVERR_* bits into it and carry on.
__device__ __forceinline__ void raise_error(int *err, int bit)
{
    if (err) atomicOr(err, bit);
}

// ---- 16-byte chunks of the three element types ---------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
    static constexpr int VEC = 4;  // elements per 16-byte chunk
    static constexpr int dtype = RPTQ_F32;
    __device__ __forceinline__ static float get(const uint4 &v, int e)
    {
        const uint32_t w = (&v.x)[e];
        return __uint_as_float(w);
    }
};
template <> struct Elem<__nv_bfloat16> {
    static constexpr int VEC = 8;
    static constexpr int dtype = RPTQ_BF16;
    // bf16 -> fp32 is exact: the 16 bits become the high half of the fp32 word
    __device__ __forceinline__ static float get(const uint4 &v, int e)
    {
        const uint32_t w = (&v.x)[e >> 1];
        return (e & 1) ? __uint_as_float(w & 0xffff0000u) : __uint_as_float(w << 16);
    }
};
template <> struct Elem<__half> {
    static constexpr int VEC = 8;
    static constexpr int dtype = RPTQ_F16;
    __device__ __forceinline__ static float get(const uint4 &v, int e)
    {
        const uint32_t w = (&v.x)[e >> 1];
        const __half h = __ushort_as_half((unsigned short)((e & 1) ? (w >> 16) : (w & 0xffffu)));
        return __half2float(h);
    }
};

// Element e of a 16-byte chunk plus nsub, in fp32 with one rounding.  16-bit inputs use the
// sm_100 mixed-precision add, which widens and adds in one instruction; nsub = -0.0 gives the
// element exactly, and x - m for x near m is exact (Sterbenz), so the same code serves rows with
// and without a subtracted offset.
template <typename T> __device__ __forceinline__ float elem_plus(const uint4 &v, int e, float nsub);
template <> __device__ __forceinline__ float elem_plus<__nv_bfloat16>(const uint4 &v, int e, float nsub)
{
    const uint32_t w = (&v.x)[e >> 1];
    float r;
    if (e & 1)
        asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %1;\n add.rn.f32.bf16 %0, hi, %2;\n}" : "=f"(r) : "r"(w), "f"(nsub));
    else
        asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %1;\n add.rn.f32.bf16 %0, lo, %2;\n}" : "=f"(r) : "r"(w), "f"(nsub));
    return r;
}
template <> __device__ __forceinline__ float elem_plus<__half>(const uint4 &v, int e, float nsub)
{
    const uint32_t w = (&v.x)[e >> 1];
    float r;
    if (e & 1)
        asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %1;\n add.rn.f32.f16 %0, hi, %2;\n}" : "=f"(r) : "r"(w), "f"(nsub));
    else
        asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %1;\n add.rn.f32.f16 %0, lo, %2;\n}" : "=f"(r) : "r"(w), "f"(nsub));
    return r;
}
template <> __device__ __forceinline__ float elem_plus<float>(const uint4 &v, int e, float nsub)
{
    return __uint_as_float((&v.x)[e]) + nsub;
}

// Moments of a 16-byte chunk: s += sum(x), q += sum(x^2).  16-bit inputs use the sm_100
// mixed-precision add/fma (16-bit sources, fp32 accumulator, one rounding; identical to widening
// first), so no separate conversion instruction is spent on them.
template <typename T> __device__ __forceinline__ void chunk_moments(const uint4 &v, float &s, float &q);
template <> __device__ __forceinline__ void chunk_moments<float>(const uint4 &v, float &s, float &q)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float f = __uint_as_float(w[i]);
        s += f;
        q = fmaf(f, f, q);
    }
}
template <> __device__ __forceinline__ void chunk_moments<__nv_bfloat16>(const uint4 &v, float &s, float &q)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %2;\n add.rn.f32.bf16 %0, lo, %0;\n"
            " add.rn.f32.bf16 %0, hi, %0;\n fma.rn.f32.bf16 %1, lo, lo, %1;\n fma.rn.f32.bf16 %1, hi, hi, %1;\n}"
            : "+f"(s), "+f"(q)
            : "r"(w[i]));
}
template <> __device__ __forceinline__ void chunk_moments<__half>(const uint4 &v, float &s, float &q)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %2;\n add.rn.f32.f16 %0, lo, %0;\n"
            " add.rn.f32.f16 %0, hi, %0;\n fma.rn.f32.f16 %1, lo, lo, %1;\n fma.rn.f32.f16 %1, hi, hi, %1;\n}"
            : "+f"(s), "+f"(q)
            : "r"(w[i]));
}

// Streaming 16-byte global load that does not allocate in L1.
// Bulk prefetch of a contiguous range into L2 (one instruction; 16-byte aligned start, size a
// multiple of 16 bytes).  Brings a later work unit close without holding registers or shared
// memory for it.
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// three-input max / min (one instruction on sm_100; NaN operands are ignored like fmaxf/fminf)
__device__ __forceinline__ float max3f(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float min3f(float a, float b, float c)
{
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// 32-bit read-once load (no L1 allocation)
__device__ __forceinline__ uint32_t ldg_stream32(const void *p)
{
    uint32_t v;
    asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint4 ldg_stream(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float4 ldg_f4(const void *p)
{
    const uint4 v = ldg_stream(p);
    return make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z), __uint_as_float(v.w));
}

__device__ __forceinline__ float fma_sat(float a, float b, float c)
{
    float d;
    asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// ---- two fp32 lanes in one 64-bit register pair (sm_100 packed fp32 arithmetic) ---------
// __ffma2_rn / __fadd2_rn / __fmul2_rn round each lane exactly like the scalar operation.
using f32x2 = float2;
__device__ __forceinline__ f32x2 mk2(float lo, float hi) { return make_float2(lo, hi); }
__device__ __forceinline__ float lo2(f32x2 a) { return a.x; }
__device__ __forceinline__ float hi2(f32x2 a) { return a.y; }
__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) { return __fmul2_rn(a, b); }
// Elements 2p, 2p+1 of a 16-byte chunk as one fp32 pair (exact widening).
template <typename T> __device__ __forceinline__ f32x2 pair_of(const uint4 &v, int p);
template <> __device__ __forceinline__ f32x2 pair_of<__nv_bfloat16>(const uint4 &v, int p)
{
    const uint32_t w = (&v.x)[p];
    return mk2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
template <> __device__ __forceinline__ f32x2 pair_of<__half>(const uint4 &v, int p)
{
    const uint32_t w = (&v.x)[p];
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w));
    return mk2(f.x, f.y);
}
template <> __device__ __forceinline__ f32x2 pair_of<float>(const uint4 &v, int p)
{
    return mk2(__uint_as_float((&v.x)[2 * p]), __uint_as_float((&v.x)[2 * p + 1]));
}

// Order-independent float max/min through integer atomics (exact; finite inputs).
__device__ __forceinline__ void atomic_max_f32(float *addr, float v)
{
    if (__float_as_int(v) >= 0)
        atomicMax(reinterpret_cast<int *>(addr), __float_as_int(v));
    else
        atomicMin(reinterpret_cast<unsigned *>(addr), __float_as_uint(v));
}
__device__ __forceinline__ void atomic_min_f32(float *addr, float v)
{
    if (__float_as_int(v) >= 0)
        atomicMin(reinterpret_cast<int *>(addr), __float_as_int(v));
    else
        atomicMax(reinterpret_cast<unsigned *>(addr), __float_as_uint(v));
}

// ---- mbarrier + bulk asynchronous copy (TMA engine, non-tensor form, no multicast) ------
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
// Copy `bytes` (multiple of 16, both addresses 16-byte aligned) global -> shared; completion
// is signalled on `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
// Copy `bytes` (multiple of 16, both addresses 16-byte aligned) shared -> global as one bulk
// asynchronous copy of the calling thread's current bulk group (never multicast).
__device__ __forceinline__ void bulk_s2g(void *dst, uint32_t src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every bulk group of the thread but the newest N has finished READING its shared
// source (the buffer may be rewritten), or has fully completed (wait_all).
template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// One suspending try: the thread sleeps in hardware until the phase completes or a system
// time limit passes (no busy polling that would take issue slots from working warps).
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait for phase `parity` of `bar`: gives up after ~2 s of wall time, reports
// RPTQ_DEVERR_TIMEOUT and returns false (the caller then uses whatever is in the buffer).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, int *err)
{
    if (mbar_try(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        if (mbar_try(bar, parity)) return true;
        if (global_ns() - t0 > 2000000000ull) {
            raise_error(err, RPTQ_DEVERR_TIMEOUT);
            return false;
        }
    }
}

// ---- CTA-wide sum of 8 floats per thread, every thread receives the 8 totals -----------
// `red` is shared scratch of 8 * (blockDim.x / 32) floats.  Deterministic (fixed order).
// Contains one __syncthreads().  nwarps_: the CTA's warp count when the caller knows it at
// compile time (0: read it from blockDim).
__device__ __forceinline__ void cta_sum8(float (&v)[8], float *red, int nwarps_ = 0)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = nwarps_ ? nwarps_ : (int)(blockDim.x >> 5);
    const bool b16 = lane & 16, b8 = lane & 8, b4 = lane & 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = b16 ? v[i] : v[i + 4];
        const float keep = b16 ? v[i + 4] : v[i];
        v[i] = keep + __shfl_xor_sync(FULL, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = b8 ? v[i] : v[i + 2];
        const float keep = b8 ? v[i + 2] : v[i];
        v[i] = keep + __shfl_xor_sync(FULL, send, 8);
    }
    {
        const float send = b4 ? v[0] : v[1];
        const float keep = b4 ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(FULL, send, 4);
    }
    v[0] += __shfl_xor_sync(FULL, v[0], 2);
    v[0] += __shfl_xor_sync(FULL, v[0], 1);
    const int idx = (b16 ? 4 : 0) + (b8 ? 2 : 0) + (b4 ? 1 : 0);
    if ((lane & 3) == 0) red[warp * 8 + idx] = v[0];
    __syncthreads();
    // lane l sums value (l & 7) over warps (l >> 3), (l >> 3) + 4, ...
    float p = 0.f;
    for (int w = lane >> 3; w < nwarps; w += 4) p += red[w * 8 + (lane & 7)];
    p += __shfl_xor_sync(FULL, p, 8);
    p += __shfl_xor_sync(FULL, p, 16);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __shfl_sync(FULL, p, i);
}

// ---- code-buffer swizzle for the fused quantizer ---------------------------------------
// The code buffer holds one 32-bit word per stored column (the codes of 4 tokens).  Word j
// lives in 16-byte slot s = j / 4; slot s is placed at s ^ ((s >> 3) & 7) so that eight
// lanes reading eight consecutive 8-slot units hit eight different bank groups.
__host__ __device__ __forceinline__ uint32_t codebuf_offset(uint32_t j)
{
    const uint32_t s = j >> 2;
    return ((s ^ ((s >> 3) & 7u)) << 4) | ((j & 3u) << 2);
}
__host__ __device__ __forceinline__ uint32_t codebuf_index(uint32_t off)
{
    const uint32_t sp = off >> 4;
    return ((sp ^ ((sp >> 3) & 7u)) << 2) | ((off >> 2) & 3u);
}

// ---- packing of 8 consecutive positions x 4 tokens (byte lane r of a word = token r) ----
// 4x4 byte transpose: out[r] = {v0.byte r, v1.byte r, v2.byte r, v3.byte r}
__device__ __forceinline__ void transpose4x4(uint32_t v0, uint32_t v1, uint32_t v2, uint32_t v3,
                                             uint32_t (&o)[4])
{
    const uint32_t t0 = prmt(v0, v1, 0x5140), t1 = prmt(v0, v1, 0x7362);
    const uint32_t t2 = prmt(v2, v3, 0x5140), t3 = prmt(v2, v3, 0x7362);
    o[0] = prmt(t0, t2, 0x5410);
    o[1] = prmt(t0, t2, 0x7632);
    o[2] = prmt(t1, t3, 0x5410);
    o[3] = prmt(t1, t3, 0x7632);
}

// 4-bit: words w[0..7] (positions) -> per token r a 32-bit word (byte i = pos 2i | pos 2i+1 << 4)
__device__ __forceinline__ void pack8x4_a4(const uint32_t *w, uint32_t (&o)[4])
{
    const uint32_t v0 = w[0] + (w[1] << 4), v1 = w[2] + (w[3] << 4);
    const uint32_t v2 = w[4] + (w[5] << 4), v3 = w[6] + (w[7] << 4);
    transpose4x4(v0, v1, v2, v3, o);
}

// 3-bit: words w[0..7] -> per token r the 24-bit group (code k at bits [3k, 3k+3))
__device__ __forceinline__ void pack8x4_a3(const uint32_t *w, uint32_t (&o)[4])
{
    const uint32_t a0 = w[0] + (w[1] << 3), a1 = w[2] + (w[3] << 3);
    const uint32_t a2 = w[4] + (w[5] << 3), a3 = w[6] + (w[7] << 3);
    uint32_t t[4];
    transpose4x4(a0, a1, a2, a3, t);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        // byte lanes hold 6-bit fields f0..f3; gather them to f0 | f1<<6 | f2<<12 | f3<<18
        // u = f0 + f1 2^6 + (f2 + f3 2^6) 2^16; move the upper 12-bit field down by 4 bits
        const uint32_t u = prmt(t[r], 0u, 0x4240) + (prmt(t[r], 0u, 0x4341) << 6);
        o[r] = u - (u >> 16) * 61440u;
    }
}

}  // namespace rptq
