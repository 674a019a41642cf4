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
// GEMM (rptq_reordered_linear): one CTA per 128 x 256 output tile, all 512 tensor-memory columns:
// the fp32 accumulator (256) and a ring of six A slabs (32 columns of fp16 pairs each).  Eight
// producer warps (0-3 the even K slabs, 4-7 the odd ones) decode a 64-column slab of their rows'
// codes into fp16 in registers and write it to its ring slot with tcgen05.st; warp 8 copies the
// matching 256 x 64 B slab with TMA into a six-slot shared-memory ring (128-byte swizzle, the
// K-major layout the tensor core reads); one thread of warp 9 issues four tcgen05.mma.kind::f16
// (K = 16 each, A from tensor memory) per slab and commits them to the slot's "empty" barrier.
// The codes reach the producers through a three-unit shared-memory ring that warp 8 fills by TMA
// (two K slabs x 128 rows per box) where the row pitch allows it, else by the producers' own
// loads.  After the last slab the producer warps read the accumulator back with tcgen05.ld and
// write Y.
// Every wait is bounded; a wait that runs out sets the device error word, and the CTA still
// waits (bounded) for its issued copies and MMAs and frees its tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>

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
// D[tmem] (+)= A[tmem] * B[smem desc]^T, fp16 inputs, fp32 accumulator
__device__ __forceinline__ void tc_mma_f16_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(d),
        "r"(a), "l"(bdesc), "r"(idesc), "r"(acc)
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

// 32 consecutive 32-bit columns of the calling thread's tensor-memory lane <- v (asynchronous:
// tc_wait_st before anything that must see them)
__device__ __forceinline__ void tc_st32(uint32_t taddr, const uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
        "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
        "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

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

// ---- offline preparation ----------------------------------------------------------------------
// Persistent CTAs, LP_ROWS output rows per iteration, one group of LP_GROUP threads per row.  Each
// CTA first builds, in shared memory, the table of stored column js -> (R[j] | k(j) << 16),
// j = lin_column(js), k = col_cluster[j] (range-checked once), and the per-cluster s_k and z_k (the
// latter as double).  Per iteration: the rows' packed codes are staged in shared memory (the next
// iteration's are loaded into registers meanwhile); a first pass finds max_j |b[n][j]| of each row
// and its lam[n]; a second recomputes b, scales it by the exact power of two 1 / lam[n], rounds
// pairs to fp16, writes B in 16-byte stores (one group of 8 stored columns per thread and step)
// and sums z_k B in fp64.  Three CTA barriers serve LP_ROWS rows.
constexpr int LP_THREADS = 512, LP_ROWS = 4, LP_GROUP = LP_THREADS / LP_ROWS;
constexpr int LP_PIECES = (RPTQ_MAX_CHANNELS / 32 + LP_GROUP - 1) / LP_GROUP;  // 16-byte pieces per thread and row

__host__ __device__ inline size_t lp_smem_bytes(int C, int g)
{
    return (size_t)g * 8 + (size_t)C * 4 + (size_t)g * 4 + (size_t)LP_ROWS * (((size_t)C / 2 + 15) & ~(size_t)15) + 16;
}

__global__ void __launch_bounds__(LP_THREADS)
    linear_prepare_kernel(const uint8_t *__restrict__ qw, const int32_t *__restrict__ zw, const int32_t *__restrict__ R,
                          const int32_t *__restrict__ col_cluster, const float *__restrict__ scale,
                          const int32_t *__restrict__ zero, int g, int C, int N, __half *__restrict__ B,
                          float *__restrict__ bz, float *__restrict__ lam, int *err)
{
    extern __shared__ __align__(16) uint8_t lp_smem[];
    double *zd = reinterpret_cast<double *>(lp_smem);      // g
    uint32_t *tab = reinterpret_cast<uint32_t *>(zd + g);  // C entries, stored order
    float *sc = reinterpret_cast<float *>(tab + C);        // g
    const size_t rowb = ((size_t)C / 2 + 15) & ~(size_t)15;
    uint8_t *qrows = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sc + g) + 15) & ~(uintptr_t)15);
    __shared__ float smax[LP_ROWS][LP_GROUP / 32];
    __shared__ double ssum[LP_ROWS][LP_GROUP / 32];
    const int tid = threadIdx.x, lane = tid & 31;
    const int rg = tid / LP_GROUP, t = tid % LP_GROUP, gw = t >> 5;  // row group, thread and warp in it
    constexpr int NW = LP_GROUP / 32;

    for (int js = tid; js < C; js += LP_THREADS) {
        const int j = lin_column(js);
        int c = R[j], k = col_cluster[j];
        if (c < 0 || c >= C) {
            raise_error(err, RPTQ_DEVERR_REORDER);
            c = 0;
        }
        if (k < 0 || k >= g) {
            raise_error(err, RPTQ_DEVERR_CLUSTER_ID);
            k = 0;
        }
        tab[js] = (uint32_t)c | ((uint32_t)k << 16);
    }
    for (int k = tid; k < g; k += LP_THREADS) {
        sc[k] = scale[k];
        zd[k] = (double)zero[k];
    }
    const int groups = C / 8, nv = C / 32;
    uint8_t *qrow = qrows + (size_t)rg * rowb;
    const int64_t stride = (int64_t)gridDim.x * LP_ROWS;
    // the codes of row n0 + rg: LP_PIECES 16-byte pieces per thread (zero past the row)
    uint4 pre[LP_PIECES];
    auto fetch = [&](int64_t n0) {
        const int64_t n = n0 + rg;
#pragma unroll
        for (int i = 0; i < LP_PIECES; ++i) {
            const int v = t + i * LP_GROUP;
            pre[i] = (n < N && v < nv) ? __ldg(reinterpret_cast<const uint4 *>(qw + n * (C / 2)) + v)
                                       : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    fetch((int64_t)blockIdx.x * LP_ROWS);
    for (int64_t n0 = (int64_t)blockIdx.x * LP_ROWS; n0 < N; n0 += stride) {
#pragma unroll
        for (int i = 0; i < LP_PIECES; ++i) {
            const int v = t + i * LP_GROUP;
            if (v < nv) reinterpret_cast<uint4 *>(qrow)[v] = pre[i];
        }
        fetch(n0 + stride);  // the next iteration's rows, while this one is processed
        __syncthreads();     // the rows (and, the first time, the tables) are in place
        const int64_t n = n0 + rg;
        const bool live = n < N;
        const int zwi = live ? zw[n] : 0;
        // q - z_w as a float: exactly (2^23 + q) - (2^23 + z_w) while |z_w| < 2^22, else a conversion
        const bool magic = zwi > -(1 << 22) && zwi < (1 << 22);
        const float base = 8388608.0f + (float)zwi;
        // b = RN(s_k (q - z_w)) of the stored column whose table entry is e
        auto bval = [&](uint32_t e) -> float {
            const uint32_t c = e & 0xFFFFu;
            const int q = (qrow[c >> 1] >> ((c & 1) * 4)) & 15;
            const float d = magic ? __int_as_float(0x4B000000 | q) - base : (float)(q - zwi);
            return sc[e >> 16] * d;
        };
        float m = 0.f;
        for (int gi = t; gi < groups; gi += LP_GROUP) {
            const uint4 t0 = reinterpret_cast<const uint4 *>(tab)[2 * gi];
            const uint4 t1 = reinterpret_cast<const uint4 *>(tab)[2 * gi + 1];
            m = fmaxf(m, fmaxf(fmaxf(fabsf(bval(t0.x)), fabsf(bval(t0.y))), fmaxf(fabsf(bval(t0.z)), fabsf(bval(t0.w)))));
            m = fmaxf(m, fmaxf(fmaxf(fabsf(bval(t1.x)), fabsf(bval(t1.y))), fmaxf(fabsf(bval(t1.z)), fabsf(bval(t1.w)))));
        }
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
        if (lane == 0) smax[rg][gw] = m;
        __syncthreads();
        m = smax[rg][0];
#pragma unroll
        for (int w = 1; w < NW; ++w) m = fmaxf(m, smax[rg][w]);
        // lam = 2^(e - 14) with m in [2^e, 2^(e+1)): the largest |B| lies in [2^14, 2^15)
        int ex = 0;
        if (m > 0.f) frexpf(m, &ex);
        const float l = m > 0.f ? ldexpf(1.f, ex - 1 - 14) : 1.f;
        const float rl = m > 0.f ? ldexpf(1.f, 15 - ex) : 1.f;  // 1 / l, exact
        double acc = 0.0;
        uint4 *dst = reinterpret_cast<uint4 *>(B + (live ? n : 0) * (int64_t)C);
        for (int gi = t; gi < groups && live; gi += LP_GROUP) {
            const uint4 t0 = reinterpret_cast<const uint4 *>(tab)[2 * gi];
            const uint4 t1 = reinterpret_cast<const uint4 *>(tab)[2 * gi + 1];
            const uint32_t te[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
            uint32_t h[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                // b / l = b * (1 / l) exactly (powers of two), then one rounding to fp16
                const __half2 hh = __floats2half2_rn(bval(te[2 * p]) * rl, bval(te[2 * p + 1]) * rl);
                const float2 f = __half22float2(hh);
                acc = fma(zd[te[2 * p] >> 16], (double)f.x, acc);
                acc = fma(zd[te[2 * p + 1] >> 16], (double)f.y, acc);
                h[p] = *reinterpret_cast<const uint32_t *>(&hh);
            }
            dst[gi] = make_uint4(h[0], h[1], h[2], h[3]);
        }
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(FULL, acc, o);
        if (lane == 0) ssum[rg][gw] = acc;
        __syncthreads();
        if (t == 0 && live) {
            double tsum = 0.0;
#pragma unroll
            for (int w = 0; w < NW; ++w) tsum += ssum[rg][w];
            bz[n] = (float)tsum;
            lam[n] = l;
        }
        __syncthreads();  // qrows, smax and ssum are reused by the next rows
    }
}

cudaError_t launch_linear_prepare(const LinPrepArgs &a)
{
    if (a.N == 0) return cudaSuccess;
    const size_t smem = lp_smem_bytes(a.C, a.g);
    cudaError_t e = kernel_smem((const void *)linear_prepare_kernel, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 1;
    e = kernel_occupancy(&per_sm, (const void *)linear_prepare_kernel, LP_THREADS, smem);
    if (e != cudaSuccess) return e;
    const int64_t units = (a.N + LP_ROWS - 1) / LP_ROWS;
    const int grid = (int)std::min<int64_t>(units, (int64_t)a.num_sms * std::max(1, per_sm));
    linear_prepare_kernel<<<grid, LP_THREADS, smem, a.stream>>>(a.qw, a.zw, a.R, a.col_cluster, a.scale, a.zero, a.g,
                                                                a.C, a.N, a.B, a.bz, a.lam, a.err);
    return cudaGetLastError();
}

// ---- the GEMM ---------------------------------------------------------------------------------
constexpr int LIN_BM = 128, LIN_BN = 256, LIN_BK = 64, LIN_STAGES = 6;
// A producers: LIN_GROUPS groups of 4 warps, group i taking the K slabs kt = i (mod LIN_GROUPS);
// warps 0-7 then run the epilogue
constexpr int LIN_GROUPS = 2;
constexpr int LIN_PROD = 128 * LIN_GROUPS;
constexpr int LIN_TMA_WARP = LIN_PROD / 32, LIN_MMA_WARP = LIN_TMA_WARP + 1;  // weight / code copies; MMA + TMEM
constexpr int LIN_THREADS = LIN_PROD + 64;
constexpr uint32_t LIN_B_BYTES = LIN_BN * LIN_BK * 2;
constexpr uint32_t LIN_TMEM_COLS = 512;     // the accumulator (256 columns) + the A ring (6 x 32)
constexpr uint32_t LIN_A_COL = LIN_BN;      // A slab s at columns LIN_A_COL + 32 s
constexpr size_t LIN_SMEM = 1024 + (size_t)LIN_STAGES * LIN_B_BYTES;
// codes staged by TMA: a ring of units of two K slabs (128 rows x 16 BITS bytes, at most 64)
constexpr int LIN_C_UNITS = 3;
constexpr uint32_t LIN_C_BYTES = LIN_BM * 64;
constexpr size_t LIN_SMEM_CTMA = LIN_SMEM + (size_t)LIN_C_UNITS * LIN_C_BYTES;
static_assert(LIN_BK * 2 == 128, "one 128-byte swizzle row per K slab");
static_assert(LIN_STAGES % LIN_GROUPS == 0, "a ring slot always holds slabs of one producer group");
static_assert(LIN_A_COL + LIN_STAGES * (LIN_BK / 2) <= LIN_TMEM_COLS, "tensor memory budget");

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
__device__ __forceinline__ void lin_decode8(uint32_t w, uint32_t *o)
{
    if constexpr (BITS == 3) w = (w & 0xFFFu) | ((w & 0xFFF000u) << 4);
    constexpr uint32_t M = BITS == 4 ? 0x000F000Fu : 0x00070007u;
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = lin_sub1024(((w >> (BITS * i)) & M) | 0x64006400u);
}
// The 64 codes of one row and one K slab (8 groups): 32 bytes (A4) or 24 bytes (A3) at p
// (16- resp. 8-byte aligned).  A3 group m sits in bytes 3m..3m+2; w[m] holds it in bits 0-23.
// A3: the 24 bytes x[0..5] of one slab -> w[m] = group m in bits 0-23
__device__ __forceinline__ void lin_unpack_a3(const uint32_t (&x)[6], uint32_t (&w)[8])
{
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // 12 bytes = 4 groups
        w[4 * h + 0] = x[3 * h];
        w[4 * h + 1] = __funnelshift_r(x[3 * h], x[3 * h + 1], 24);
        w[4 * h + 2] = __funnelshift_r(x[3 * h + 1], x[3 * h + 2], 16);
        w[4 * h + 3] = x[3 * h + 2] >> 8;
    }
}
// the same 32 (A4) or 24 (A3) bytes from shared memory (16- resp. 8-byte aligned)
template <int BITS>
__device__ __forceinline__ void lin_load_slab_smem(uint32_t saddr, uint32_t (&w)[8])
{
    if constexpr (BITS == 4) {
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(saddr) : "memory");
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7]) : "r"(saddr + 16) : "memory");
    } else {
        uint32_t x[6];
#pragma unroll
        for (int i = 0; i < 3; ++i)
            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(x[2 * i]), "=r"(x[2 * i + 1]) : "r"(saddr + 8 * i)
                         : "memory");
        lin_unpack_a3(x, w);
    }
}
template <int BITS>
__device__ __forceinline__ void lin_load_slab(const uint8_t *p, uint32_t (&w)[8])
{
    if constexpr (BITS == 4) {
        const uint4 a = __ldg(reinterpret_cast<const uint4 *>(p));
        const uint4 b = __ldg(reinterpret_cast<const uint4 *>(p) + 1);
        w[0] = a.x, w[1] = a.y, w[2] = a.z, w[3] = a.w, w[4] = b.x, w[5] = b.y, w[6] = b.z, w[7] = b.w;
    } else {
        const uint2 a = __ldg(reinterpret_cast<const uint2 *>(p));
        const uint2 b = __ldg(reinterpret_cast<const uint2 *>(p) + 1);
        const uint2 c = __ldg(reinterpret_cast<const uint2 *>(p) + 2);
        const uint32_t x[6] = {a.x, a.y, b.x, b.y, c.x, c.y};
        lin_unpack_a3(x, w);
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
// of 256.  K = C is a multiple of 64: K / 64 slabs.  The decoded codes go straight from the
// producers' registers into tensor memory (tcgen05.st) and the MMA reads A from there, so shared
// memory carries only the weight slabs.  With CTMA the producers read their codes from a ring of
// units (two K slabs x 128 rows) that warp 8 fills by TMA ahead of the weight slabs (cmap: the
// codes [T, K BITS / 8] as bytes), instead of loading them from global memory themselves.
template <int BITS, bool CTMA>
__global__ void __launch_bounds__(LIN_THREADS, 1)
    reordered_linear_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap cmap,
                            const uint8_t *__restrict__ codes, int64_t T, int K, int N,
                            const float *__restrict__ bz, const float *__restrict__ lam,
                            const float *__restrict__ sw, float *__restrict__ Y, int vec_store, int *err)
{
    extern __shared__ uint8_t lin_smem_raw[];
    __shared__ __align__(8) uint64_t bars[3 * LIN_STAGES + 1 + 2 * LIN_C_UNITS];
    __shared__ uint32_t tmem_slot;
    __shared__ int s_abort;  // set by any role whose bounded wait ran out
    __shared__ float s_bz[LIN_BN], s_f[LIN_BN];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t m0 = (int64_t)blockIdx.x * LIN_BM;
    const int n0 = blockIdx.y * LIN_BN;
    const int KT = K / LIN_BK;
    const uint32_t sB = (smem_u32(lin_smem_raw) + 1023u) & ~1023u;  // swizzled tiles: 1024-aligned
    const uint32_t full_a = smem_u32(&bars[0]), full_b = smem_u32(&bars[LIN_STAGES]);
    const uint32_t empty = smem_u32(&bars[2 * LIN_STAGES]), done = smem_u32(&bars[3 * LIN_STAGES]);
    const uint32_t full_c = done + 8, empty_c = full_c + 8 * LIN_C_UNITS;  // the code ring (CTMA)
    const uint32_t sC = sB + LIN_STAGES * LIN_B_BYTES;
    constexpr uint32_t UB = 16 * BITS;  // bytes of one row in a code unit

    if (tid == 0) {
        for (int s = 0; s < LIN_STAGES; ++s) {
            mbar_init(full_a + 8 * s, LIN_PROD / LIN_GROUPS);  // the 4 warps of one producer group
            mbar_init(full_b + 8 * s, 1);
            mbar_init(empty + 8 * s, 1);
        }
        mbar_init(done, 1);
        for (int c = 0; c < LIN_C_UNITS; ++c) {
            mbar_init(full_c + 8 * c, 1);
            mbar_init(empty_c + 8 * c, 8);  // one lane of each warp of the two groups reading the unit
        }
        fence_mbar_init();
        s_abort = 0;
    }
    if (tid < LIN_BN) {
        const int n = n0 + tid;
        s_bz[tid] = n < N ? bz[n] : 0.f;
        s_f[tid] = n < N ? sw[n] * lam[n] : 0.f;  // lam is a power of two
    }
    if (warp == LIN_MMA_WARP) tc_alloc(smem_u32(&tmem_slot), LIN_TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    if (warp < LIN_PROD / 32) {
        // ---- A producers: warp w owns TMEM lanes 32 (w % 4) .. +31 (the tile's rows) and the
        //      slabs of parity w / 4; a thread decodes its row's 64 codes into 32 columns ----
        const int qd = warp & 3, par = warp >> 2;
        const int r = 32 * qd + lane;
        const bool row_ok = m0 + r < T;
        const int64_t pitch = (int64_t)K * BITS / 8;
        const uint8_t *src = codes + (row_ok ? m0 + r : 0) * pitch;
        const uint32_t ta = tmem + ((uint32_t)(32 * qd) << 16) + LIN_A_COL;
        // slab kt: wait for its A slot (the whole warp agrees: tcgen05.st is warp-collective),
        // decode, store into tensor memory, signal the MMA
        auto put = [&](int kt, const uint32_t (&w)[8]) -> bool {
            const int s = kt % LIN_STAGES, u = kt / LIN_STAGES;
            if (!__all_sync(FULL, mbar_wait_bounded(empty + 8 * s, (u & 1) ^ 1, err))) return false;
            tc_fence_after();  // the slot's previous MMAs are complete
            uint32_t d[32];
#pragma unroll
            for (int gi = 0; gi < 8; ++gi) lin_decode8<BITS>(w[gi], d + 4 * gi);
            tc_st32(ta + 32 * s, d);
            tc_wait_st();
            tc_fence_before();
            lin_arrive(full_a + 8 * s);
            return true;
        };
        bool ok = true;
        if constexpr (CTMA) {
            // codes from the ring: unit kt / 2, this slab's half of the row
            for (int kt = par; kt < KT && ok; kt += LIN_GROUPS) {
                const int u = kt >> 1, cu = u % LIN_C_UNITS;
                if (!(ok = __all_sync(FULL, mbar_wait_bounded(full_c + 8 * cu, (uint32_t)(u / LIN_C_UNITS) & 1, err))))
                    break;
                uint32_t w[8];
                lin_load_slab_smem<BITS>(sC + cu * LIN_C_BYTES + r * UB + (kt & 1) * (UB / 2), w);
                ok = put(kt, w);
                // the unit is released only after the decode in put() has consumed the loaded
                // words: a shared-memory load still in flight at the release could read bytes
                // of the next unit, which the TMA may already be writing (measured: an earlier
                // release made the A4 results differ from run to run)
                __syncwarp();
                if (lane == 0) lin_arrive(empty_c + 8 * cu);
            }
        } else {
            uint32_t wa[8], wb[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) wa[i] = wb[i] = 0;
            if (row_ok && par < KT) lin_load_slab<BITS>(src + (int64_t)par * (8 * BITS), wa);
            if (row_ok && par + LIN_GROUPS < KT)
                lin_load_slab<BITS>(src + (int64_t)(par + LIN_GROUPS) * (8 * BITS), wb);
            for (int kt = par; kt < KT && ok; kt += LIN_GROUPS) {
                uint32_t wc[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) wc[i] = 0;
                if (row_ok && kt + 2 * LIN_GROUPS < KT)
                    lin_load_slab<BITS>(src + (int64_t)(kt + 2 * LIN_GROUPS) * (8 * BITS), wc);
                ok = put(kt, wa);
#pragma unroll
                for (int i = 0; i < 8; ++i) wa[i] = wb[i], wb[i] = wc[i];
            }
        }
        if (!ok) *(volatile int *)&s_abort = 1;
        // ---- epilogue (warps 0-7): warp w reads TMEM lanes 32 (w % 4) .. +31, the (w / 4)-th half of
        //      the columns ----
        if (warp >= 8) ok = false;
        if (ok) ok = mbar_wait_bounded(done, 0, err);
        ok = __all_sync(FULL, ok);  // tcgen05.ld is warp-collective: the whole warp or none
        tc_fence_after();
        if (ok) {
            const int64_t row = m0 + r;
            for (int i = 0; i < LIN_BN / 64; ++i) {
                const int col0 = par * (LIN_BN / 2) + 32 * i;
                uint32_t v[32];
                tc_ld32(tmem + ((uint32_t)(32 * qd) << 16) + (uint32_t)col0, v);
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
    } else if (warp == LIN_TMA_WARP) {
        // ---- weight slabs: one 256 x 64 fp16 box per slab, 128-byte swizzle, through TMA ----
        if (lane == 0) {
            // code units (CTMA) go two units ahead of the weight slabs
            const int units = (KT + 1) >> 1;
            int cissued = 0;
            auto issue_unit = [&](int u) -> bool {
                const int cu = u % LIN_C_UNITS;
                if (!mbar_wait_bounded(empty_c + 8 * cu, ((uint32_t)(u / LIN_C_UNITS) & 1) ^ 1, err)) return false;
                mbar_expect_tx(full_c + 8 * cu, LIN_BM * UB);
                lin_tma_load_2d(sC + cu * LIN_C_BYTES, &cmap, u * (int)UB, (int)m0, full_c + 8 * cu);
                cissued = u + 1;
                return true;
            };
            bool ok = true;
            if constexpr (CTMA)
                for (int u = 0; u < 2 && u < units && ok; ++u) ok = issue_unit(u);
            int issued = 0;
            for (int kt = 0; kt < KT && ok; ++kt) {
                if (CTMA && (kt & 1) == 0 && kt / 2 + 2 < units && !(ok = issue_unit(kt / 2 + 2))) break;
                const int s = kt % LIN_STAGES, u = kt / LIN_STAGES;
                if (!(ok = mbar_wait_bounded(empty + 8 * s, (u & 1) ^ 1, err))) break;
                mbar_expect_tx(full_b + 8 * s, LIN_B_BYTES);
                lin_tma_load_2d(sB + s * LIN_B_BYTES, &wmap, kt * LIN_BK, n0, full_b + 8 * s);
                issued = kt + 1;
            }
            if (!ok) *(volatile int *)&s_abort = 1;
            // Nothing asynchronous may still write this CTA's shared memory when it exits: the
            // copies (their barrier phases), then the MMA commits to the last slabs' barriers.
            for (int u = cissued > LIN_C_UNITS ? cissued - LIN_C_UNITS : 0; u < cissued; ++u)
                mbar_wait_bounded(full_c + 8 * (u % LIN_C_UNITS), (uint32_t)(u / LIN_C_UNITS) & 1, err);
            const int first = issued > LIN_STAGES ? issued - LIN_STAGES : 0;
            for (int kt = first; kt < issued; ++kt)
                mbar_wait_bounded(full_b + 8 * (kt % LIN_STAGES), (kt / LIN_STAGES) & 1, err);
            for (int kt = first; kt < issued && !*(volatile int *)&s_abort; ++kt)
                mbar_wait_bounded(empty + 8 * (kt % LIN_STAGES), (kt / LIN_STAGES) & 1, err);
        }
    } else {
        // ---- MMA issue: four K = 16 steps per slab (8 TMEM columns of A, 32 bytes of B each) ----
        if (lane == 0) {
            constexpr uint32_t idesc = f16_idesc(LIN_BM, LIN_BN);
            for (int kt = 0; kt < KT; ++kt) {
                const int s = kt % LIN_STAGES, u = kt / LIN_STAGES;
                if (!mbar_wait_bounded(full_b + 8 * s, u & 1, err) || !mbar_wait_bounded(full_a + 8 * s, u & 1, err)) {
                    *(volatile int *)&s_abort = 1;
                    break;
                }
                tc_fence_after();
                const uint64_t bd = sw128_desc(sB + s * LIN_B_BYTES);
                const uint32_t at = tmem + LIN_A_COL + 32 * s;
#pragma unroll
                for (int kk = 0; kk < LIN_BK / 16; ++kk)
                    tc_mma_f16_ts(tmem, at + 8 * kk, bd + (uint64_t)(2 * kk), idesc, (kt | kk) != 0);
                tc_commit(empty + 8 * s);  // the slot may be refilled once these MMAs are done
            }
            tc_commit(done);
            // the accumulator is released below: wait for every issued MMA first
            mbar_wait_bounded(done, 0, err);
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == LIN_MMA_WARP) {
        tc_fence_after();
        tc_dealloc(tmem, LIN_TMEM_COLS);
    }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link against libcuda).
static PFN_cuTensorMapEncodeTiled_v12000 encode_tiled_fn()
{
    // looked up once per process (a function-local static is initialised exactly once, also when
    // several host threads call at the same time)
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    }();
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
    // the codes [T, K bits / 8] as bytes, boxes of 128 rows x one unit (two K slabs), rows past T
    // read as zeros: where TMA can address them (row pitch a multiple of 16 bytes, row index
    // within int32), otherwise the producers load their codes themselves
    const int64_t pitch = (int64_t)a.C * a.bits / 8;
    CUtensorMap cmap;
    memset(&cmap, 0, sizeof(cmap));
    bool ctma = pitch % 16 == 0 && a.T <= 0x7fffffffLL;
    if (ctma) {
        const cuuint64_t cdims[2] = {(cuuint64_t)pitch, (cuuint64_t)a.T};
        const cuuint64_t cstrides[1] = {(cuuint64_t)pitch};
        const cuuint32_t cbox[2] = {(cuuint32_t)(16 * a.bits), (cuuint32_t)LIN_BM};
        ctma = encode(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(a.codes), cdims, cstrides, cbox,
                      estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    const void *kern = a.bits == 4 ? (ctma ? (const void *)reordered_linear_kernel<4, true>
                                           : (const void *)reordered_linear_kernel<4, false>)
                                   : (ctma ? (const void *)reordered_linear_kernel<3, true>
                                           : (const void *)reordered_linear_kernel<3, false>);
    const size_t smem = ctma ? LIN_SMEM_CTMA : LIN_SMEM;
    cudaError_t e = kernel_smem(kern, smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((a.T + LIN_BM - 1) / LIN_BM), (unsigned)((a.N + LIN_BN - 1) / LIN_BN));
    const int vec = (a.N % 4 == 0 && (reinterpret_cast<uintptr_t>(a.Y) & 15) == 0) ? 1 : 0;
    void *args[] = {(void *)&map,  (void *)&cmap, (void *)&a.codes, (void *)&a.T, (void *)&a.C, (void *)&a.N,
                    (void *)&a.bz, (void *)&a.lam, (void *)&a.sw,   (void *)&a.Y, (void *)&vec, (void *)&a.err};
    return cudaLaunchKernel(kern, grid, dim3(LIN_THREADS), args, smem, a.stream);
}

}  // namespace rptq
