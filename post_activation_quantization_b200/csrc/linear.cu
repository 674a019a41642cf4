// linear.cu -- the reordered low-bit linear layer: a tcgen05 GEMM over packed cluster-ordered codes.
//
// RPTQ article (基于重排序的新量化方法RPTQ…), Fig. 3 caption and the text after it: the layer that
// follows the reorder-fused LayerNorm has its weight matrix permuted offline by the same reorder
// index, so it consumes the activations in cluster order and its output is unchanged; the text
// after Fig. 2: one (s, z) per cluster of activation channels; the results paragraph: W4A4 /
// W4A3.  With 4-bit weights quantized per output row (quantization-basics article, sections 1.3,
// 1.4) the layer computes, for token t and output n (k = col_cluster[j]):
//     Y[t][n] = sum_j s_k (q[t][j] - z_k) * s_w[n] (qw[n][R[j]] - z_w[n]).
// Offline preparation (rptq_linear_prepare) folds everything but the activation code into the
// weight operand, in fp16 with a power-of-two row scale lam[n] that keeps it in fp16's range:
//     B[n][j] = RN_fp16( RN(s_k (qw[n][R[j]] - z_w[n])) / lam[n] ),   bz[n] = sum_j z_k B[n][j]
// (the columns interleaved inside groups of 8, see lin_column),
// so that Y[t][n] = s_w[n] lam[n] (sum_j q[t][j] B[n][j] - bz[n]).  The code q itself (0..15) is
// the A operand, exact in fp16, decoded from the packed activation codes inside the kernel.
//
// GEMM (rptq_reordered_linear): one CTA per 128 x 256 output tile, fp32 accumulator in tensor
// memory (256 of the SM's 512 columns).  Eight producer warps decode a 64-column slab of codes
// into fp16 and copy the matching B slab, both into shared memory in the 128-byte-swizzled
// K-major layout the tensor core reads; one thread of a ninth warp issues four
// tcgen05.mma.kind::f16 (K = 16 each) per slab and commits them to the slab's "empty" barrier;
// four slabs are in flight.  After the last slab the producers read the accumulator back with
// tcgen05.ld and write Y.  Every wait is bounded; a wait that runs out sets the device error
// word, and the CTA still waits (bounded) for its issued MMAs and frees its tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace rptq {

// ---- tcgen05 / mbarrier wrappers (sm_100a) ---------------------------------------------------
__device__ __forceinline__ void lin_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// whole warp: allocate `cols` tensor-memory columns, the base address goes to shared `dst`
__device__ __forceinline__ void tc_alloc(uint32_t dst, uint32_t cols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst), "r"(cols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_dealloc(uint32_t taddr, uint32_t cols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, fp16 inputs, fp32 accumulator
__device__ __forceinline__ void tc_mma_f16(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}
// arrive once on `bar` when every tcgen05.mma this thread issued so far has completed
__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
// 32 consecutive fp32 columns of the calling thread's tensor-memory lane
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile whose rows are 128 bytes (64 fp16)
// in the 128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r mod 8); groups of 8 rows
// are 1024 bytes apart (stride byte offset); the tile starts on a 1024-byte boundary.  Fields:
// start address >> 4 (bits 0-13), leading byte offset 16 >> 4 (unused by this layout), stride
// byte offset 1024 >> 4 (bits 32-45), descriptor version 1 (bits 46-47), swizzle mode
// "128-byte" = 2 (bits 61-63).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1), fp16 A and B (bits 7-12
// = 0), both K-major (bits 15, 16 = 0), N >> 3 at bits 17-22, M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t f16_idesc(int M, int N)
{
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// The GEMM's A decoder turns one 8-code group (one 32-bit word of A4 codes, or 24 bits of A3
// codes) into four fp16 pairs (q0,q4) (q1,q5) (q2,q6) (q3,q7), one mask-and-or each.  The
// prepared weights store their columns in that same order inside every group of 8, so the dot
// products pair each code with its own weight: stored column js holds cluster-order column
//     j = 8*(js/8) + (js even ? (js%8)/2 : 4 + (js%8)/2).
__host__ __device__ __forceinline__ int lin_column(int js) { return (js & ~7) | ((js & 1) << 2) | ((js >> 1) & 3); }

// ---- offline preparation: one CTA per output row n -----------------------------------------
__global__ void __launch_bounds__(256)
    linear_prepare_kernel(const uint8_t *__restrict__ qw, const float *__restrict__ sw, const int32_t *__restrict__ zw,
                          const int32_t *__restrict__ R, const int32_t *__restrict__ col_cluster,
                          const float *__restrict__ scale, const int32_t *__restrict__ zero, int g, int C, int N,
                          __half *__restrict__ B, float *__restrict__ bz, float *__restrict__ lam, int *err)
{
    __shared__ float smax[8];
    __shared__ double ssum[8];
    const int n = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint8_t *row = qw + (int64_t)n * (C / 2);
    const int zwn = zw[n];
    auto value = [&](int j, int &k) -> float {  // RN(s_k (qw[n][R[j]] - z_w[n]))
        int c = R[j];
        if (c < 0 || c >= C) {
            raise_error(err, RPTQ_DEVERR_REORDER);
            c = 0;
        }
        k = col_cluster[j];
        if (k < 0 || k >= g) {
            raise_error(err, RPTQ_DEVERR_CLUSTER_ID);
            k = 0;
        }
        const int q = (row[c >> 1] >> ((c & 1) * 4)) & 15;
        return scale[k] * (float)(q - zwn);
    };
    float m = 0.f;
    for (int j = tid; j < C; j += 256) {
        int k;
        m = fmaxf(m, fabsf(value(j, k)));
    }
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
    if (lane == 0) smax[warp] = m;
    __syncthreads();
    m = smax[0];
    for (int w = 1; w < 8; ++w) m = fmaxf(m, smax[w]);
    // lam = 2^(e - 14) with m in [2^e, 2^(e+1)): the largest |B| lies in [2^14, 2^15)
    int e = 0;
    if (m > 0.f) frexpf(m, &e);
    const float l = m > 0.f ? ldexpf(1.f, e - 1 - 14) : 1.f;
    double acc = 0.0;
    for (int js = tid; js < C; js += 256) {
        int k;
        const float v = value(lin_column(js), k) / l;  // a power of two: exact
        const __half h = __float2half_rn(v);
        B[(int64_t)n * C + js] = h;
        acc += (double)zero[k] * (double)__half2float(h);
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(FULL, acc, o);
    if (lane == 0) ssum[warp] = acc;
    __syncthreads();
    if (tid == 0) {
        double t = 0.0;
        for (int w = 0; w < 8; ++w) t += ssum[w];
        bz[n] = (float)t;
        lam[n] = l;
    }
}

cudaError_t launch_linear_prepare(const LinPrepArgs &a)
{
    if (a.N == 0) return cudaSuccess;
    linear_prepare_kernel<<<a.N, 256, 0, a.stream>>>(a.qw, a.sw, a.zw, a.R, a.col_cluster, a.scale, a.zero, a.g, a.C,
                                                     a.N, a.B, a.bz, a.lam, a.err);
    return cudaGetLastError();
}

// ---- the GEMM ---------------------------------------------------------------------------------
constexpr int LIN_BM = 128, LIN_BN = 256, LIN_BK = 64, LIN_STAGES = 4;
constexpr int LIN_PROD = 256;               // warps 0-7: A producers, then the epilogue
constexpr int LIN_THREADS = LIN_PROD + 64;  // warp 8: weight copies, warp 9: MMA issue + TMEM
constexpr uint32_t LIN_A_BYTES = LIN_BM * LIN_BK * 2;
constexpr uint32_t LIN_B_BYTES = LIN_BN * LIN_BK * 2;
constexpr uint32_t LIN_TMEM_COLS = LIN_BN;  // one fp32 column per output of the tile
constexpr size_t LIN_SMEM = 1024 + (size_t)LIN_STAGES * (LIN_A_BYTES + LIN_B_BYTES);
static_assert(LIN_BK * 2 == 128, "one 128-byte swizzle row per K slab");

// fp16 pairs 1024 + q  ->  q (exact)
__device__ __forceinline__ uint32_t lin_sub1024(uint32_t v)
{
    uint32_t o;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(o) : "r"(v), "r"(0x64006400u));
    return o;
}
// One 8-code group -> four fp16 pairs (q0,q4) (q1,q5) (q2,q6) (q3,q7).  A4: the group is one
// little-endian word, code i in bits 4i..4i+3.  A3: 24 bits, code i in bits 3i..3i+2; codes 4-7
// move up to bit 16 first.  A code OR-ed into the mantissa of 1024.0 (0x6400) gives 1024 + q.
template <int BITS>
__device__ __forceinline__ uint4 lin_decode8(uint32_t w)
{
    if constexpr (BITS == 3) w = (w & 0xFFFu) | ((w & 0xFFF000u) << 4);
    constexpr uint32_t M = BITS == 4 ? 0x000F000Fu : 0x00070007u;
    uint4 o;
    o.x = lin_sub1024(((w >> 0) & M) | 0x64006400u);
    o.y = lin_sub1024(((w >> BITS) & M) | 0x64006400u);
    o.z = lin_sub1024(((w >> (2 * BITS)) & M) | 0x64006400u);
    o.w = lin_sub1024(((w >> (3 * BITS)) & M) | 0x64006400u);
    return o;
}
// Four 8-code groups of one row: 16 bytes (A4) or 12 bytes (A3) at p (4-byte aligned).
template <int BITS>
__device__ __forceinline__ void lin_load_groups(const uint8_t *p, uint32_t (&w)[4])
{
    if constexpr (BITS == 4) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p));
        w[0] = v.x, w[1] = v.y, w[2] = v.z, w[3] = v.w;
    } else {
        const uint32_t a = __ldg(reinterpret_cast<const uint32_t *>(p));
        const uint32_t b = __ldg(reinterpret_cast<const uint32_t *>(p) + 1);
        const uint32_t c = __ldg(reinterpret_cast<const uint32_t *>(p) + 2);
        w[0] = a;                          // bytes 0-2 (the decoder drops bits 24-31)
        w[1] = __funnelshift_r(a, b, 24);  // bytes 3-5
        w[2] = __funnelshift_r(b, c, 16);  // bytes 6-8
        w[3] = c >> 8;                     // bytes 9-11
    }
}
__device__ __forceinline__ void lin_tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Y[t][n] = f[n] (sum_j q[t][j] B[n][j] - bz[n]),  f = s_w lam.  Grid: x = token tiles of 128
// (consecutive CTAs share one weight tile, which then comes from DRAM once), y = output tiles
// of 256.  K = C is a multiple of 64: K / 64 slabs.
template <int BITS>
__global__ void __launch_bounds__(LIN_THREADS, 1)
    reordered_linear_kernel(const __grid_constant__ CUtensorMap wmap, const uint8_t *__restrict__ codes, int64_t T,
                            int K, int N, const float *__restrict__ bz, const float *__restrict__ lam,
                            const float *__restrict__ sw, float *__restrict__ Y, int vec_store, int *err)
{
    extern __shared__ uint8_t lin_smem_raw[];
    __shared__ __align__(8) uint64_t bars[3 * LIN_STAGES + 1];
    __shared__ uint32_t tmem_slot;
    __shared__ int s_abort;  // set by any role whose bounded wait ran out
    __shared__ float s_bz[LIN_BN], s_f[LIN_BN];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t m0 = (int64_t)blockIdx.x * LIN_BM;
    const int n0 = blockIdx.y * LIN_BN;
    const int KT = K / LIN_BK;
    const uint32_t sbase = (smem_u32(lin_smem_raw) + 1023u) & ~1023u;  // swizzled tiles: 1024-aligned
    const uint32_t sA = sbase, sB = sbase + LIN_STAGES * LIN_A_BYTES;
    const uint32_t full_a = smem_u32(&bars[0]), full_b = smem_u32(&bars[LIN_STAGES]);
    const uint32_t empty = smem_u32(&bars[2 * LIN_STAGES]), done = smem_u32(&bars[3 * LIN_STAGES]);

    if (tid == 0) {
        for (int s = 0; s < LIN_STAGES; ++s) {
            mbar_init(full_a + 8 * s, LIN_PROD);
            mbar_init(full_b + 8 * s, 1);
            mbar_init(empty + 8 * s, 1);
        }
        mbar_init(done, 1);
        fence_mbar_init();
        s_abort = 0;
    }
    if (tid < LIN_BN) {
        const int n = n0 + tid;
        s_bz[tid] = n < N ? bz[n] : 0.f;
        s_f[tid] = n < N ? sw[n] * lam[n] : 0.f;  // lam is a power of two
    }
    if (warp == 9) tc_alloc(smem_u32(&tmem_slot), LIN_TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    if (warp < 8) {
        // ---- A producers: thread = (row r, half h of the slab's 64 codes = 4 groups of 8) ----
        const int r = tid >> 1, h = tid & 1;
        const bool row_ok = m0 + r < T;
        const int64_t pitch = (int64_t)K * BITS / 8;
        const uint8_t *src = codes + (row_ok ? m0 + r : 0) * pitch + h * (4 * BITS);
        uint32_t wa[4] = {0, 0, 0, 0}, wb[4] = {0, 0, 0, 0};
        if (row_ok) lin_load_groups<BITS>(src, wa);
        if (row_ok && KT > 1) lin_load_groups<BITS>(src + 8 * BITS, wb);
        bool ok = true;
        for (int kt = 0; kt < KT; ++kt) {
            uint32_t wc[4] = {0, 0, 0, 0};
            if (row_ok && kt + 2 < KT) lin_load_groups<BITS>(src + (int64_t)(kt + 2) * (8 * BITS), wc);
            const int s = kt % LIN_STAGES, u = kt / LIN_STAGES;
            if (!mbar_wait_bounded(empty + 8 * s, (u & 1) ^ 1, err)) {
                ok = false;
                *(volatile int *)&s_abort = 1;
                break;
            }
            const uint32_t dst = sA + s * LIN_A_BYTES + r * 128;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 v = lin_decode8<BITS>(wa[i]);
                const uint32_t c = (uint32_t)(4 * h + i) ^ (uint32_t)(r & 7);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst + (c << 4)), "r"(v.x), "r"(v.y),
                             "r"(v.z), "r"(v.w)
                             : "memory");
            }
            fence_proxy_async_smem();  // generic-proxy stores -> visible to the tensor core
            lin_arrive(full_a + 8 * s);
#pragma unroll
            for (int i = 0; i < 4; ++i) wa[i] = wb[i], wb[i] = wc[i];
        }
        // ---- epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31, columns 128 (w / 4) .. +127 ----
        if (ok) ok = mbar_wait_bounded(done, 0, err);
        ok = __all_sync(FULL, ok);  // tcgen05.ld is warp-collective: the whole warp or none
        tc_fence_after();
        if (ok) {
            const int q = warp & 3;
            const int64_t row = m0 + 32 * q + lane;
            for (int i = 0; i < 4; ++i) {
                const int col0 = (warp >> 2) * 128 + 32 * i;
                uint32_t v[32];
                tc_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)col0, v);
                if (row >= T || n0 + col0 >= N) continue;
                float *yrow = Y + row * (int64_t)N + n0 + col0;
                if (vec_store && n0 + col0 + 32 <= N) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        float4 o;
                        o.x = (__uint_as_float(v[j + 0]) - s_bz[col0 + j + 0]) * s_f[col0 + j + 0];
                        o.y = (__uint_as_float(v[j + 1]) - s_bz[col0 + j + 1]) * s_f[col0 + j + 1];
                        o.z = (__uint_as_float(v[j + 2]) - s_bz[col0 + j + 2]) * s_f[col0 + j + 2];
                        o.w = (__uint_as_float(v[j + 3]) - s_bz[col0 + j + 3]) * s_f[col0 + j + 3];
                        *reinterpret_cast<float4 *>(yrow + j) = o;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (n0 + col0 + j < N) yrow[j] = (__uint_as_float(v[j]) - s_bz[col0 + j]) * s_f[col0 + j];
                }
            }
        }
    } else if (warp == 8) {
        // ---- weight slabs: one 256 x 64 fp16 box per slab, 128-byte swizzle, through TMA ----
        if (lane == 0) {
            int issued = 0;
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % LIN_STAGES, u = kt / LIN_STAGES;
                if (!mbar_wait_bounded(empty + 8 * s, (u & 1) ^ 1, err)) {
                    *(volatile int *)&s_abort = 1;
                    break;
                }
                mbar_expect_tx(full_b + 8 * s, LIN_B_BYTES);
                lin_tma_load_2d(sB + s * LIN_B_BYTES, &wmap, kt * LIN_BK, n0, full_b + 8 * s);
                issued = kt + 1;
            }
            // Nothing asynchronous may still write this CTA's shared memory when it exits: the
            // copies (their barrier phases), then the MMA commits to the last slabs' barriers.
            const int first = issued > LIN_STAGES ? issued - LIN_STAGES : 0;
            for (int kt = first; kt < issued; ++kt)
                mbar_wait_bounded(full_b + 8 * (kt % LIN_STAGES), (kt / LIN_STAGES) & 1, err);
            for (int kt = first; kt < issued && !*(volatile int *)&s_abort; ++kt)
                mbar_wait_bounded(empty + 8 * (kt % LIN_STAGES), (kt / LIN_STAGES) & 1, err);
        }
    } else {
        // ---- MMA issue: four K = 16 steps per slab; the descriptor start advances 32 bytes ----
        if (lane == 0) {
            constexpr uint32_t idesc = f16_idesc(LIN_BM, LIN_BN);
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % LIN_STAGES, u = kt / LIN_STAGES;
                if (!mbar_wait_bounded(full_b + 8 * s, u & 1, err) || !mbar_wait_bounded(full_a + 8 * s, u & 1, err)) {
                    *(volatile int *)&s_abort = 1;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = sw128_desc(sA + s * LIN_A_BYTES), bd = sw128_desc(sB + s * LIN_B_BYTES);
#pragma unroll
                for (int kk = 0; kk < LIN_BK / 16; ++kk)
                    tc_mma_f16(tmem, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc, (kt | kk) != 0);
                tc_commit(empty + 8 * s);  // the slab may be refilled once these MMAs are done
            }
            tc_commit(done);
            // the accumulator is released below: wait for every issued MMA first
            mbar_wait_bounded(done, 0, err);
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tc_dealloc(tmem, LIN_TMEM_COLS);
    }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link against libcuda).
static PFN_cuTensorMapEncodeTiled_v12000 encode_tiled_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool looked = false;
    if (!looked) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        looked = true;
    }
    return fn;
}

cudaError_t launch_reordered_linear(const LinArgs &a)
{
    if (a.T == 0) return cudaSuccess;
    PFN_cuTensorMapEncodeTiled_v12000 encode = encode_tiled_fn();
    if (!encode) return cudaErrorNotSupported;
    // the prepared weights [N, K] fp16, K contiguous: boxes of 64 columns x 256 rows, rows past N
    // read as zeros
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)a.C, (cuuint64_t)a.N};
    const cuuint64_t strides[1] = {(cuuint64_t)a.C * 2};
    const cuuint32_t box[2] = {(cuuint32_t)LIN_BK, (cuuint32_t)LIN_BN};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half *>(a.B), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const void *kern = a.bits == 4 ? (const void *)reordered_linear_kernel<4> : (const void *)reordered_linear_kernel<3>;
    cudaError_t e = kernel_smem(kern, LIN_SMEM);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((a.T + LIN_BM - 1) / LIN_BM), (unsigned)((a.N + LIN_BN - 1) / LIN_BN));
    const int vec = (a.N % 4 == 0 && (reinterpret_cast<uintptr_t>(a.Y) & 15) == 0) ? 1 : 0;
    void *args[] = {(void *)&map, (void *)&a.codes, (void *)&a.T,   (void *)&a.C, (void *)&a.N, (void *)&a.bz,
                    (void *)&a.lam, (void *)&a.sw,  (void *)&a.Y, (void *)&vec, (void *)&a.err};
    return cudaLaunchKernel(kern, grid, dim3(LIN_THREADS), args, LIN_SMEM, a.stream);
}

}  // namespace rptq
