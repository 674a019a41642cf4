// kmeans.cu -- channel clustering, reorder index and per-cluster quantization parameters.
//
// RPTQ article (基于重排序的新量化方法RPTQ…), text after Fig. 2: KMeans splits the channels into
// g clusters using the 2-D points (channel max, channel min); channels of one cluster are then
// placed next to each other, and each cluster gets its own scale s and zero point z.
// Quantization-basics article, section 一 (s = float range / integer range) and 1.3 (zero point).
//
// The pages leave the KMeans details open; this library fixes them (the same readings as the
// CPU oracle): fp64 points, quantile initialisation from the (max, min, index) order, squared
// Euclidean distance dx*dx + dy*dy without fused multiply-add, ties to the lowest index, mean
// update with empty clusters kept, `iters` rounds then a final assignment.
//
// Launch sequence on the caller's stream (no host synchronisation), two kernels:
//   km_prep   clears the exchange cells and the grid-barrier words of the workspace
//   km_fused  one cooperative launch of ceil(C/512) CTAs, 512 points per CTA (2 per thread):
//     ranks   each CTA sorts its points' (max, min, index) keys (bitonic, shared memory) and
//             publishes the sorted segment; after one grid barrier every CTA copies all
//             segments into shared memory and ranks its points by binary search in each one
//             (segments are contiguous index ranges, so equal keys are ordered by segment);
//             lanes of a warp take neighbouring sorted keys, so their searches read the same
//             entries; the point of rank floor((2k+1) C / (2g)) seeds centroid k
//     Lloyd   per iteration: assignment (below), per-warp cluster sums in lane order, per-CTA
//             sums in warp order, then an all-to-all exchange of the per-CTA sums in which
//             every 8-byte word carries the iteration number next to 32 bits of data, so a
//             reader knows from the word itself that it is current (no separate barrier);
//             every CTA folds the records in CTA order into identical centroids.  Records
//             alternate between two buffers by iteration parity: a CTA overwrites a buffer only
//             after it has read every CTA's next record, which each CTA writes only after
//             reading this one.  An assignment that repeats the previous one ends the loop.
//     final   the final assignment; per-CTA cluster sizes, minima and maxima are exchanged the
//             same way; every CTA derives the cluster offsets, its own base in each cluster
//             (the sizes of the CTAs before it) and the (s, z) of each cluster, and scatters
//             its channels to their stable positions (cluster, then channel index).
//   Assignment: one fp32 pass over the centroids (packed f32x2, two points at a time) finds the
//   smallest and second smallest fp32 distance; an error bound (see `certified`) proves for
//   almost every point that the fp32 winner is the fp64 argmin, and the rest (about 1e-5 of
//   the points) take the exhaustive fp64 scan.  Labels are those of the exhaustive scan.
//   Every wait is bounded (2 s, then the device error word and no further waiting).
#include <algorithm>

#include "../../include/rptq_testing.h"
#include "common.cuh"
#include "launch.h"

namespace rptq {

constexpr int KM_THREADS = 256;
constexpr int KM_WARPS = KM_THREADS / 32;
constexpr int KM_PPT = 2;                   // points per thread
constexpr int KM_PTS = KM_THREADS * KM_PPT;  // points per CTA
constexpr int KM_MAX_NB = (RPTQ_MAX_CHANNELS + KM_PTS - 1) / KM_PTS;
static_assert(KM_PTS == 512, "the binary search below assumes 512-point segments");

__host__ __device__ inline size_t km_align(size_t v) { return (v + 255) & ~(size_t)255; }
__host__ __device__ inline int km_blocks(int C) { return (C + KM_PTS - 1) / KM_PTS; }
// 16-byte cells of one CTA's iteration record: g sums of max, g sums of min (one double per
// cell), then the g cluster sizes and the CTA's changed-label count, two per cell
__host__ __device__ inline int km_rec_cells(int g) { return 2 * g + (g + 2) / 2; }

struct KmWs {
    uint4 *seeds;     // [2g] cells: seed k's x in cell 2k, y in cell 2k+1
    uint4 *sums;      // [2][nb][rec] cells: per-CTA iteration records by iteration parity
    uint64_t *fin;    // [3][nb][g] words: per-CTA size, min, max of every final cluster
    unsigned *bar;    // grid-barrier words
    uint64_t *keys;   // [nb * 512] sorted point keys, one segment per CTA
    size_t clear;     // bytes from `seeds` up to `keys` that must be zero at launch
};

static KmWs km_carve(void *ws, int C, int g)
{
    const size_t nb = (size_t)km_blocks(C);
    uint8_t *p = static_cast<uint8_t *>(ws);
    KmWs w;
    w.seeds = reinterpret_cast<uint4 *>(p);
    p += km_align((size_t)2 * g * 16);
    w.sums = reinterpret_cast<uint4 *>(p);
    p += km_align(2 * nb * (size_t)km_rec_cells(g) * 16);
    w.fin = reinterpret_cast<uint64_t *>(p);
    p += km_align(3 * nb * (size_t)g * 8);
    w.bar = reinterpret_cast<unsigned *>(p);
    p += 256;
    w.keys = reinterpret_cast<uint64_t *>(p);
    w.clear = (size_t)(p - static_cast<uint8_t *>(ws));
    return w;
}

size_t kmeans_ws_bytes(int C, int g)
{
    const size_t nb = (size_t)km_blocks(C);
    return km_align((size_t)2 * g * 16) + km_align(2 * nb * (size_t)km_rec_cells(g) * 16) +
           km_align(3 * nb * (size_t)g * 8) + 256 + km_align(nb * KM_PTS * 8);
}

// Dynamic shared memory of km_fused: the centroids and their sorted copy, then one region
// reused by the phases.
__host__ __device__ inline size_t km_persist_bytes(int g) { return ((size_t)24 * g + 15) & ~(size_t)15; }
size_t kmeans_smem_bytes(int C, int g)
{
    const size_t nb = (size_t)km_blocks(C);
    const size_t ranks = nb * KM_PTS * 8 + KM_PTS * (8 + 2);
    const size_t lloyd = (size_t)KM_PTS * 16 + (size_t)KM_WARPS * 3 * g * 8 + (size_t)2 * g * 8 + (size_t)(g + 2) * 4;
    const size_t fin = (size_t)2 * KM_WARPS * g * 4 + (size_t)g * 4 * 4 + (size_t)(g + 1) * 4;
    return km_persist_bytes(g) + std::max(ranks, std::max(lloyd, fin));
}

__device__ __forceinline__ double sq_dist(double px, double py, double cx, double cy)
{
    const double dx = __dsub_rn(px, cx), dy = __dsub_rn(py, cy);
    return __dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy));
}

// Oracle's assignment of one point, exhaustive: argmin over k of the fp64 squared distance
// dx*dx + dy*dy (no fused multiply-add), strict < so that ties keep the lowest k.
__device__ __noinline__ int nearest_exact(double px, double py, const double *cx, const double *cy, int g)
{
    double best = sq_dist(px, py, cx[0], cy[0]);
    int lab = 0;
    for (int k = 1; k < g; ++k) {
        const double d = sq_dist(px, py, cx[k], cy[k]);
        if (d < best) {
            best = d;
            lab = k;
        }
    }
    return lab;
}

// True when the fp32 scan's winner is certainly the fp64 argmin: b1 <= b2 are the smallest and
// second smallest fp32 distances, P = |px| + |py|.
//
// Error bound.  With the point exact in fp32 (it is a float statistic), the centroid rounded to
// fp32 and dx = px - cx, dy = py - cy in fp32, d32 = fma(dy, dy, dx*dx) differs from the fp64
// distance D of the same centroid by at most E(D) = 2^-20 (D + P sqrt(D)) + 2^-45 P^2 (the
// centroid's rounding gives |dx32 - dx| <= 2^-24 (|px| + 2|dx|), and similarly for y, three fp32
// roundings add 2^-23 D, D's own fp64 roundings add 2^-50 D).  From |d32 - D| <= E(D) it follows
// that D <= U(d32) = d32 + 2^-18 (d32 + P sqrt(d32)) + 2^-38 P^2, and for d32 >= 2^-36 P^2 that
// D >= L(d32) = d32 - 2^-18 (d32 + P sqrt(d32)) - 2^-38 P^2, L increasing there.  Every other
// centroid has d32 >= b2, so its D >= L(b2); if L(b2) > U(b1) the winner's D is strictly the
// smallest and the exhaustive fp64 scan returns the same index.  Points with P < 2^-40 (no
// relative error bound near the fp32 subnormal range) and non-finite values fail the test and
// take the exhaustive scan.
__device__ __forceinline__ bool certified(float b1f, float b2f, double P)
{
    if (!(P >= 0x1p-40)) return false;
    const double b1 = b1f, b2 = b2f, P2 = P * P;
    if (!(b2 >= 0x1p-36 * P2)) return false;
    const double up = b1 + 0x1p-18 * (b1 + P * sqrt(b1)) + 0x1p-38 * P2;
    const double lw = b2 - 0x1p-18 * (b2 + P * sqrt(b2)) - 0x1p-38 * P2;
    return lw > up * (1.0 + 0x1p-40);
}

// Nearest centroids of a thread's two points.  One fp32 pass over the centroids (both points at
// once in packed f32x2 arithmetic; ncf holds the negated fp32 centroids) finds each point's
// smallest and second smallest fp32 distance; a certified winner is the answer, any other point
// (about 1e-5 of them on activation statistics) takes the exhaustive fp64 scan.
__device__ __forceinline__ void nearest2(const double (&px)[2], const double (&py)[2], const bool (&own)[2],
                                         const float2 *ncf, const double *cx, const double *cy, int g,
                                         int (&lab)[2])
{
    const f32x2 X = mk2((float)px[0], (float)px[1]), Y = mk2((float)py[0], (float)py[1]);
    float b1a = INFINITY, b2a = INFINITY, b1b = INFINITY, b2b = INFINITY;
    int ka = 0, kb = 0;
#pragma unroll 4
    for (int k = 0; k < g; ++k) {
        const float2 c = ncf[k];
        const f32x2 dx = add2(X, mk2(c.x, c.x)), dy = add2(Y, mk2(c.y, c.y));
        const f32x2 d = fma2(dy, dy, mul2(dx, dx));
        const float da = lo2(d), db = hi2(d);
        bool lt = da < b1a;
        b2a = lt ? b1a : fminf(b2a, da);
        b1a = lt ? da : b1a;
        ka = lt ? k : ka;
        lt = db < b1b;
        b2b = lt ? b1b : fminf(b2b, db);
        b1b = lt ? db : b1b;
        kb = lt ? k : kb;
    }
    lab[0] = ka;
    lab[1] = kb;
    if (own[0] && !certified(b1a, b2a, fabs(px[0]) + fabs(py[0]))) lab[0] = nearest_exact(px[0], py[0], cx, cy, g);
    if (own[1] && !certified(b1b, b2b, fabs(px[1]) + fabs(py[1]))) lab[1] = nearest_exact(px[1], py[1], cx, cy, g);
    if (!own[0]) lab[0] = -1;
    if (!own[1]) lab[1] = -1;
}

__global__ void km_prep(uint4 *clear, size_t n16)
{
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (size_t)gridDim.x * blockDim.x)
        clear[i] = make_uint4(0, 0, 0, 0);
}

// Order-preserving 32-bit image of a float (finite values): unsigned comparison of the images
// orders the floats.
__device__ __forceinline__ uint32_t ordered_bits(float f)
{
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ uint64_t point_key(float mx, float mn)
{
    return ((uint64_t)ordered_bits(mx) << 32) | ordered_bits(mn);
}

// Number of keys of the sorted segment s[0, len) (len <= 512) below `key` (or not above it).
template <bool UPPER>
__device__ __forceinline__ int seg_count(const uint64_t *s, int len, uint64_t key)
{
    int pos = 0;
#pragma unroll
    for (int step = 512; step > 0; step >>= 1) {
        if (pos + step <= len) {
            const uint64_t v = s[pos + step - 1];
            if (UPPER ? v <= key : v < key) pos += step;
        }
    }
    return pos;
}

// ---- exchange words: 32 bits of data + a 32-bit flag in one naturally aligned 8-byte word
__device__ __forceinline__ uint64_t ll_word(uint32_t data, uint32_t flag) { return data | ((uint64_t)flag << 32); }
__device__ __forceinline__ void ll_put2(uint4 *p, uint32_t a, uint32_t b, uint32_t flag)
{
    asm volatile("st.relaxed.gpu.global.v2.u64 [%0], {%1, %2};" ::"l"(p), "l"(ll_word(a, flag)),
                 "l"(ll_word(b, flag))
                 : "memory");
}
__device__ __forceinline__ void ll_put1(uint64_t *p, uint32_t a, uint32_t flag)
{
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(ll_word(a, flag)) : "memory");
}
__device__ __forceinline__ void ll_get2(const uint4 *p, uint64_t &w0, uint64_t &w1)
{
    asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(w0), "=l"(w1) : "l"(p) : "memory");
}
__device__ __forceinline__ void ll_get1(const uint64_t *p, uint64_t &w)
{
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
}
__device__ __forceinline__ bool ll_ok(uint64_t w, uint32_t flag) { return (uint32_t)(w >> 32) == flag; }

// Limit of every exchange wait and grid barrier of the KMeans kernel (2 s), and the CTA that
// leaves out its first Lloyd record (-1: none).  Both change only through the testing hook
// rptq_testing_kmeans_wait (include/rptq_testing.h), so that a test can make a wait run out.
static __device__ unsigned long long g_km_wait_ns = 2000000000ull;
static __device__ int g_km_withhold = -1;

// Read cells p[b * stride], b < n (n <= N), until both words of each carry `flag`: all reads
// are issued together and only the cells still stale are read again, all together.  Bounded by
// the wait limit, after which the device error word is set and `abort` makes every later wait
// of the CTA give up at once.
template <int N>
__device__ __forceinline__ void ll_gather2(const uint4 *p, size_t stride, int n, uint32_t flag, uint64_t (&v0)[N],
                                           uint64_t (&v1)[N], int *err, volatile int *abort)
{
#pragma unroll
    for (int b = 0; b < N; ++b)
        if (b < n) ll_get2(p + b * stride, v0[b], v1[b]);
    unsigned pend = 0;
#pragma unroll
    for (int b = 0; b < N; ++b)
        if (b < n && !(ll_ok(v0[b], flag) && ll_ok(v1[b], flag))) pend |= 1u << b;
    if (!pend) return;
    const uint64_t t0 = global_ns();
    while (pend && !*abort) {
        __nanosleep(32);
#pragma unroll
        for (int b = 0; b < N; ++b)
            if ((pend >> b) & 1u) ll_get2(p + b * stride, v0[b], v1[b]);
#pragma unroll
        for (int b = 0; b < N; ++b)
            if (((pend >> b) & 1u) && ll_ok(v0[b], flag) && ll_ok(v1[b], flag)) pend &= ~(1u << b);
        if (pend && global_ns() - t0 > g_km_wait_ns) {
            raise_error(err, RPTQ_DEVERR_TIMEOUT);
            *abort = 1;
        }
    }
}
template <int N>
__device__ __forceinline__ void ll_gather1(const uint64_t *p, size_t stride, int n, uint32_t flag, uint64_t (&v)[N],
                                           int *err, volatile int *abort)
{
#pragma unroll
    for (int b = 0; b < N; ++b)
        if (b < n) ll_get1(p + b * stride, v[b]);
    unsigned pend = 0;
#pragma unroll
    for (int b = 0; b < N; ++b)
        if (b < n && !ll_ok(v[b], flag)) pend |= 1u << b;
    if (!pend) return;
    const uint64_t t0 = global_ns();
    while (pend && !*abort) {
        __nanosleep(32);
#pragma unroll
        for (int b = 0; b < N; ++b)
            if ((pend >> b) & 1u) ll_get1(p + b * stride, v[b]);
#pragma unroll
        for (int b = 0; b < N; ++b)
            if (((pend >> b) & 1u) && ll_ok(v[b], flag)) pend &= ~(1u << b);
        if (pend && global_ns() - t0 > g_km_wait_ns) {
            raise_error(err, RPTQ_DEVERR_TIMEOUT);
            *abort = 1;
        }
    }
}

// Grid-wide barrier for a cooperative launch: arrival counter + generation word.  The wait is
// bounded by the wait limit; on expiry the device error word and `abort` are set, and a CTA
// that has aborted no longer waits at all (its later exchange waits give up at once too), so
// one straggler costs at most one limit per CTA.
__device__ __forceinline__ void km_grid_barrier(unsigned *bar, int *err, volatile int *abort)
{
    __syncthreads();
    if (threadIdx.x == 0 && !*abort) {
        unsigned g0;
        asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(g0) : "l"(bar + 1) : "memory");
        unsigned prior;
        asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(prior) : "l"(bar) : "memory");
        if (prior == gridDim.x - 1) {
            asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" ::"l"(bar) : "memory");
            asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(bar + 1) : "memory");
        } else {
            const uint64_t t0 = global_ns();
            uint32_t spin = 0;
            for (;;) {
                unsigned gv;
                asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(gv) : "l"(bar + 1) : "memory");
                if (gv != g0) break;
                if ((++spin & 255u) == 0 && global_ns() - t0 > g_km_wait_ns) {
                    raise_error(err, RPTQ_DEVERR_TIMEOUT);
                    *abort = 1;
                    break;
                }
            }
        }
    }
    __syncthreads();
}

__device__ __forceinline__ double dbl_of(uint64_t w0, uint64_t w1)
{
    return __hiloint2double((int)(uint32_t)w1, (int)(uint32_t)w0);
}

__global__ void __launch_bounds__(KM_THREADS, 1)
    km_fused(const float *__restrict__ mx, const float *__restrict__ mn, int C, int g, int iters, int bits,
             KmWs w, double *cent, int32_t *labels, int32_t *R, int32_t *col_cluster, int32_t *offsets,
             float *scale, int32_t *zero, int *err)
{
    extern __shared__ __align__(16) uint8_t ksm[];
    __shared__ int s_abort;
    volatile int *abort = &s_abort;
    // centroids (fp64) and their negated fp32 copy for the certified scan
    double *cx = reinterpret_cast<double *>(ksm), *cy = cx + g;
    float2 *ncf = reinterpret_cast<float2 *>(cy + g);
    uint8_t *U = ksm + km_persist_bytes(g);  // region shared by the phases
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nb = gridDim.x, me = blockIdx.x, base = me * KM_PTS;
    const unsigned lanes_below = (1u << lane) - 1u;

    // own points: before the local sort slot j holds point base + j*256 + tid (local index li)
    double px[KM_PPT], py[KM_PPT];
    bool own[KM_PPT];
    uint64_t key[KM_PPT];
    int li[KM_PPT];
#pragma unroll
    for (int j = 0; j < KM_PPT; ++j) {
        const int c = base + j * KM_THREADS + tid;
        own[j] = c < C;
        const float fx = own[j] ? mx[c] : 0.f, fy = own[j] ? mn[c] : 0.f;
        px[j] = fx;
        py[j] = fy;
        key[j] = own[j] ? point_key(fx, fy) : ~0ull;  // padding sorts after every real key
        li[j] = j * KM_THREADS + tid;
    }
    if (tid == 0) s_abort = 0;

    // ================= ranks in the (max, min, index) order and the quantile seeds
    {
        uint64_t *allk = reinterpret_cast<uint64_t *>(U);
        uint64_t *sk = allk + (size_t)nb * KM_PTS;
        uint16_t *si = reinterpret_cast<uint16_t *>(sk + KM_PTS);
#pragma unroll
        for (int j = 0; j < KM_PPT; ++j) {
            sk[j * KM_THREADS + tid] = key[j];
            si[j * KM_THREADS + tid] = (uint16_t)(j * KM_THREADS + tid);
        }
        __syncthreads();
        // bitonic sort of the 512 (key, local index) pairs, ascending
        for (int size = 2; size <= KM_PTS; size <<= 1)
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                const int i = ((tid & ~(stride - 1)) << 1) | (tid & (stride - 1)), k2 = i + stride;
                const uint64_t a = sk[i], b = sk[k2];
                const uint16_t ia = si[i], ib = si[k2];
                const bool gt = a > b || (a == b && ia > ib);
                if (gt == ((i & size) == 0)) {
                    sk[i] = b;
                    sk[k2] = a;
                    si[i] = ib;
                    si[k2] = ia;
                }
                __syncthreads();
            }
        // From here on slot j of a thread is the point at sorted position j*256 + tid: the lanes
        // of a warp hold neighbours in the (max, min) order, so their searches below and their
        // nearest-centroid walks read the same or adjacent shared-memory entries (broadcasts,
        // not bank conflicts) and take similar numbers of steps.
        const int nvalid = min(KM_PTS, C - base);
        int rank[KM_PPT];
#pragma unroll
        for (int j = 0; j < KM_PPT; ++j) {
            const int p = j * KM_THREADS + tid;
            li[j] = si[p];
            key[j] = sk[p];
            own[j] = p < nvalid;
            const int c = base + li[j];
            px[j] = own[j] ? (double)mx[c] : 0.0;
            py[j] = own[j] ? (double)mn[c] : 0.0;
            if (own[j]) w.keys[base + p] = key[j];
            rank[j] = p;  // keys of the own segment below this one
        }
        __threadfence();
        km_grid_barrier(w.bar, err, abort);
        for (int i = tid; i < C; i += KM_THREADS) allk[i] = __ldcg(w.keys + i);
        __syncthreads();
        // rank = own-segment position + keys below (other segments); equal keys: a lower
        // segment holds lower channel indices.  Both points and four segments at a time:
        // eight independent branch-free searches in flight.
        for (int b0 = 0; b0 < nb; b0 += 4) {
            int pos[KM_PPT][4], len[4];
            bool upper[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int b = b0 + u;
                len[u] = (b < nb && b != me) ? min(KM_PTS, C - b * KM_PTS) : 0;
                upper[u] = b < me;
#pragma unroll
                for (int j = 0; j < KM_PPT; ++j) pos[j][u] = 0;
            }
#pragma unroll
            for (int step = KM_PTS; step > 0; step >>= 1)
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int j = 0; j < KM_PPT; ++j) {
                        const int i = max(min(pos[j][u] + step, len[u]) - 1, 0);
                        const uint64_t v = allk[(size_t)min(b0 + u, nb - 1) * KM_PTS + i];
                        const bool take = pos[j][u] + step <= len[u] && (v < key[j] || (upper[u] && v == key[j]));
                        pos[j][u] += take ? step : 0;
                    }
#pragma unroll
            for (int j = 0; j < KM_PPT; ++j) rank[j] += pos[j][0] + pos[j][1] + pos[j][2] + pos[j][3];
        }
#pragma unroll
        for (int j = 0; j < KM_PPT; ++j) {
            if (!own[j]) continue;
            const int r = rank[j];
            // the point of rank floor((2k+1) C / (2g)) seeds centroid k
            const int64_t num = 2 * (int64_t)g * r - C;
            const int64_t k = num <= 0 ? 0 : (num + 2 * (int64_t)C - 1) / (2 * (int64_t)C);
            if (k < g && ((2 * k + 1) * (int64_t)C) / (2 * (int64_t)g) == r) {
                const double x = px[j], y = py[j];
                ll_put2(w.seeds + 2 * k, (uint32_t)__double2loint(x), (uint32_t)__double2hiint(x), 1u);
                ll_put2(w.seeds + 2 * k + 1, (uint32_t)__double2loint(y), (uint32_t)__double2hiint(y), 1u);
            }
        }
        for (int k = tid; k < g; k += KM_THREADS) {
            uint64_t a[2], b[2];
            ll_gather2<2>(w.seeds + 2 * k, 1, 2, 1u, a, b, err, abort);
            cx[k] = dbl_of(a[0], b[0]);
            cy[k] = dbl_of(a[1], b[1]);
            ncf[k] = make_float2(-(float)cx[k], -(float)cy[k]);
        }
        __syncthreads();
    }

    // ================= Lloyd iterations
    {
        const int G3 = 3 * g, rec = km_rec_cells(g);
        double *spx = reinterpret_cast<double *>(U), *spy = spx + KM_PTS;  // [slot * 256 + tid]
        double *wsum = spy + KM_PTS;                                         // [warp][x | y | n][g]
        double *totd = wsum + (size_t)KM_WARPS * G3;                         // [x | y][g]
        int *totn = reinterpret_cast<int *>(totd + 2 * g);                   // [g] sizes, [g] changed
        // back to index order: slot j of a thread is point base + j*256 + tid (small same-label
        // groups per warp for the sums below)
#pragma unroll
        for (int j = 0; j < KM_PPT; ++j) {
            const int c = base + j * KM_THREADS + tid;
            own[j] = c < C;
            px[j] = own[j] ? (double)mx[c] : 0.0;
            py[j] = own[j] ? (double)mn[c] : 0.0;
            spx[j * KM_THREADS + tid] = px[j];
            spy[j * KM_THREADS + tid] = py[j];
        }
        int prev[KM_PPT] = {-1, -1};
        double *mw = wsum + (size_t)warp * G3;
        for (int it = 0; it < iters; ++it) {
            for (int i = lane; i < G3; i += 32) mw[i] = 0.0;
            int lab[KM_PPT];
            bool changed = false;
            nearest2(px, py, own, ncf, cx, cy, g, lab);
#pragma unroll
            for (int j = 0; j < KM_PPT; ++j) {
                changed |= lab[j] != prev[j];
                prev[j] = lab[j];
            }
            __syncwarp();
            // per-warp sums, slot 0 then slot 1; the lowest lane of each same-label group adds
            // the group in lane order
#pragma unroll
            for (int j = 0; j < KM_PPT; ++j) {
                const unsigned same = __match_any_sync(FULL, lab[j]);
                if (lab[j] >= 0 && (same & lanes_below) == 0) {
                    double sx = 0.0, sy = 0.0;
                    for (unsigned m = same; m; m &= m - 1) {
                        const int q = j * KM_THREADS + warp * 32 + __ffs(m) - 1;
                        sx = __dadd_rn(sx, spx[q]);
                        sy = __dadd_rn(sy, spy[q]);
                    }
                    mw[lab[j]] = __dadd_rn(mw[lab[j]], sx);
                    mw[g + lab[j]] = __dadd_rn(mw[g + lab[j]], sy);
                    mw[2 * g + lab[j]] += (double)__popc(same);
                }
                __syncwarp();
            }
            const int nchg = __syncthreads_count(changed);
            // publish this CTA's record: warps folded in warp order (a CTA named by the testing
            // hook leaves out its first record, so the other CTAs' gathers run out)
            const uint32_t flag = (uint32_t)it + 1u;
            uint4 *out = w.sums + ((size_t)(it & 1) * nb + me) * rec;
            const bool publish = !(it == 0 && me == g_km_withhold);
            for (int q = tid; q < rec && publish; q += KM_THREADS) {
                if (q < 2 * g) {
                    double a = 0.0;
#pragma unroll
                    for (int v = 0; v < KM_WARPS; ++v) a = __dadd_rn(a, wsum[(size_t)v * G3 + q]);
                    ll_put2(out + q, (uint32_t)__double2loint(a), (uint32_t)__double2hiint(a), flag);
                } else {
                    uint32_t n[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int i = 2 * (q - 2 * g) + h;
                        double a = 0.0;
                        if (i < g)
#pragma unroll
                            for (int v = 0; v < KM_WARPS; ++v) a += wsum[(size_t)v * G3 + 2 * g + i];
                        n[h] = i < g ? (uint32_t)a : (i == g ? (uint32_t)nchg : 0u);
                    }
                    ll_put2(out + q, n[0], n[1], flag);
                }
            }
            // gather every CTA's record and fold in CTA order
            const uint4 *in = w.sums + (size_t)(it & 1) * nb * rec;
            for (int q = tid; q < rec; q += KM_THREADS) {
                uint64_t v0[KM_MAX_NB], v1[KM_MAX_NB];
                ll_gather2<KM_MAX_NB>(in + q, rec, nb, flag, v0, v1, err, abort);
                if (q < 2 * g) {
                    double a = 0.0;
#pragma unroll
                    for (int b = 0; b < KM_MAX_NB; ++b)
                        if (b < nb) a = __dadd_rn(a, dbl_of(v0[b], v1[b]));
                    totd[q] = a;
                } else {
                    uint32_t n0 = 0, n1 = 0;
#pragma unroll
                    for (int b = 0; b < KM_MAX_NB; ++b)
                        if (b < nb) {
                            n0 += (uint32_t)v0[b];
                            n1 += (uint32_t)v1[b];
                        }
                    const int i = 2 * (q - 2 * g);
                    totn[i] = (int)n0;
                    totn[i + 1] = (int)n1;
                }
            }
            __syncthreads();
            for (int q = tid; q < 2 * g; q += KM_THREADS) {
                const int k = q < g ? q : q - g, n = totn[k];
                if (n > 0) {  // an empty cluster keeps its centroid
                    const double v = __ddiv_rn(totd[q], (double)n);
                    (q < g ? cx : cy)[k] = v;
                    reinterpret_cast<float *>(ncf + k)[q < g ? 0 : 1] = -(float)v;
                }
            }
            const bool stop = (totn[g] == 0 && it > 0) || *abort;
            __syncthreads();
            if (stop) break;
        }
    }

    // ================= final assignment, stable counting sort, (s, z)
    {
        int *hist = reinterpret_cast<int *>(U);  // [slot * 8 + warp][g], then exclusive prefixes
        float *cmn = reinterpret_cast<float *>(hist + 2 * KM_WARPS * g), *cmx = cmn + g;
        int *csize = reinterpret_cast<int *>(cmx + g), *cbase = csize + g, *offs = cbase + g;
        int L[KM_PPT];
        nearest2(px, py, own, ncf, cx, cy, g, L);
        for (int i = tid; i < 2 * KM_WARPS * g; i += KM_THREADS) hist[i] = 0;
        for (int k = tid; k < g; k += KM_THREADS) {
            cmn[k] = INFINITY;
            cmx[k] = -INFINITY;
        }
        __syncthreads();
        unsigned same[KM_PPT];
#pragma unroll
        for (int j = 0; j < KM_PPT; ++j) {
            same[j] = __match_any_sync(FULL, L[j]);
            if (L[j] >= 0) {
                if ((same[j] & lanes_below) == 0) hist[(j * KM_WARPS + warp) * g + L[j]] = __popc(same[j]);
                atomic_min_f32(cmn + L[j], (float)py[j]);
                atomic_max_f32(cmx + L[j], (float)px[j]);
                labels[base + j * KM_THREADS + tid] = L[j];
            }
        }
        __syncthreads();
        for (int k = tid; k < g; k += KM_THREADS) {
            int run = 0;
            for (int i = 0; i < 2 * KM_WARPS; ++i) {
                const int t = hist[i * g + k];
                hist[i * g + k] = run;
                run += t;
            }
            ll_put1(w.fin + ((size_t)0 * nb + me) * g + k, (uint32_t)run, 1u);
            ll_put1(w.fin + ((size_t)1 * nb + me) * g + k, __float_as_uint(cmn[k]), 1u);
            ll_put1(w.fin + ((size_t)2 * nb + me) * g + k, __float_as_uint(cmx[k]), 1u);
        }
        __syncthreads();  // the CTA's own min / max are read above before being replaced below
        for (int item = tid; item < 3 * g; item += KM_THREADS) {
            const int f = item >= 2 * g ? 2 : (item >= g ? 1 : 0), k = item - f * g;
            const uint64_t *src = w.fin + (size_t)f * nb * g + k;
            uint64_t v[KM_MAX_NB];
            ll_gather1<KM_MAX_NB>(src, g, nb, 1u, v, err, abort);
            if (f == 0) {
                int tot = 0, before = 0;
#pragma unroll
                for (int b = 0; b < KM_MAX_NB; ++b)
                    if (b < nb) {
                        if (b == me) before = tot;
                        tot += (int)(uint32_t)v[b];
                    }
                csize[k] = tot;
                cbase[k] = before;
            } else {
                float r = f == 1 ? INFINITY : -INFINITY;
#pragma unroll
                for (int b = 0; b < KM_MAX_NB; ++b)
                    if (b < nb) {
                        const float e = __uint_as_float((uint32_t)v[b]);
                        r = f == 1 ? fminf(r, e) : fmaxf(r, e);
                    }
                (f == 1 ? cmn : cmx)[k] = r;
            }
        }
        __syncthreads();
        if (warp == 0) {  // cluster offsets: exclusive scan of the sizes
            int carry = 0;
            for (int k0 = 0; k0 < g; k0 += 32) {
                const int v = k0 + lane < g ? csize[k0 + lane] : 0;
                int incl = v;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(FULL, incl, o);
                    if (lane >= o) incl += t;
                }
                if (k0 + lane < g) offs[k0 + lane] = carry + incl - v;
                carry += __shfl_sync(FULL, incl, 31);
            }
            if (lane == 0) offs[g] = carry;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < KM_PPT; ++j)
            if (L[j] >= 0) {
                const int c = base + j * KM_THREADS + tid;
                const int pos = offs[L[j]] + cbase[L[j]] + hist[(j * KM_WARPS + warp) * g + L[j]] +
                                __popc(same[j] & lanes_below);
                if (pos >= 0 && pos < C) {  // always, unless an exchange wait gave up
                    R[pos] = c;
                    col_cluster[pos] = L[j];
                } else {
                    raise_error(err, RPTQ_DEVERR_TIMEOUT);
                }
            }
        if (me == 0) {
            // per-cluster scale and zero point (fp32 IEEE operations, round half to even)
            const float qmax = (float)((1 << bits) - 1);
            for (int k = tid; k < g; k += KM_THREADS) {
                offsets[k] = offs[k];
                cent[2 * k] = cx[k];
                cent[2 * k + 1] = cy[k];
                if (csize[k] == 0) {
                    scale[k] = 1.0f;
                    zero[k] = 0;
                    continue;
                }
                const float M = cmx[k], m = cmn[k];
                float s;
                if (M == m) {
                    float r = fmaxf(fabsf(m), fabsf(M));
                    if (r == 0.0f) r = 1.0f;
                    s = __fdiv_rn(r, qmax);
                } else {
                    s = __fdiv_rn(__fsub_rn(M, m), qmax);
                }
                scale[k] = s;
                zero[k] = (int32_t)rintf(__fdiv_rn(-m, s));
            }
            if (tid == 0) offsets[g] = offs[g];
        }
    }
}

// ------------------------------------------------------------------------------------------
// Per-cluster (s, z) for fixed clusters from per-channel statistics: the parameter step of the
// calibration on its own, for dynamic (per-batch) ranges.  One CTA of CP_THREADS: the members'
// max / min are folded per cluster with order-independent shared-memory atomics (exact), then s
// and z follow with the same fp32 IEEE operations as in the calibration above.  A thread loads
// the (label, max, min) of CP_UNROLL channels before folding any, so the loads of a whole pass
// over the channels are in flight together instead of one round trip per CP_THREADS channels.
constexpr int CP_THREADS = 1024, CP_UNROLL = 4;
__global__ void __launch_bounds__(CP_THREADS)
    cluster_params_kernel(const float *__restrict__ mx, const float *__restrict__ mn, int C,
                          const int32_t *__restrict__ labels, int g, int bits, float *__restrict__ scale,
                          int32_t *__restrict__ zero, int *err)
{
    __shared__ float cmx[RPTQ_MAX_CLUSTERS], cmn[RPTQ_MAX_CLUSTERS];
    __shared__ int cnt[RPTQ_MAX_CLUSTERS];
    for (int k = threadIdx.x; k < g; k += blockDim.x) {
        cmx[k] = -INFINITY;
        cmn[k] = INFINITY;
        cnt[k] = 0;
    }
    __syncthreads();
    for (int c0 = threadIdx.x; c0 < C; c0 += CP_THREADS * CP_UNROLL) {
        int kk[CP_UNROLL];
        float vx[CP_UNROLL], vn[CP_UNROLL];
#pragma unroll
        for (int u = 0; u < CP_UNROLL; ++u) {
            const int c = c0 + u * CP_THREADS;
            kk[u] = c < C ? __ldg(labels + c) : -1;
            vx[u] = c < C ? __ldg(mx + c) : 0.f;
            vn[u] = c < C ? __ldg(mn + c) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < CP_UNROLL; ++u) {
            if (c0 + u * CP_THREADS >= C) continue;
            const int k = kk[u];
            if (k < 0 || k >= g) {
                raise_error(err, RPTQ_DEVERR_CLUSTER_ID);
                continue;
            }
            atomic_max_f32(cmx + k, vx[u]);
            atomic_min_f32(cmn + k, vn[u]);
            atomicAdd(cnt + k, 1);
        }
    }
    __syncthreads();
    const float qmax = (float)((1 << bits) - 1);
    for (int k = threadIdx.x; k < g; k += blockDim.x) {
        if (cnt[k] == 0) {
            scale[k] = 1.0f;
            zero[k] = 0;
            continue;
        }
        const float M = cmx[k], m = cmn[k];
        float s;
        if (M == m) {
            float r = fmaxf(fabsf(m), fabsf(M));
            if (r == 0.0f) r = 1.0f;
            s = __fdiv_rn(r, qmax);
        } else {
            s = __fdiv_rn(__fsub_rn(M, m), qmax);
        }
        scale[k] = s;
        zero[k] = (int32_t)rintf(__fdiv_rn(-m, s));
    }
}

cudaError_t launch_cluster_params(const float *mx, const float *mn, int C, const int32_t *labels, int g, int bits,
                                  float *scale, int32_t *zero, int *err, cudaStream_t stream)
{
    cluster_params_kernel<<<1, CP_THREADS, 0, stream>>>(mx, mn, C, labels, g, bits, scale, zero, err);
    return cudaGetLastError();
}

bool kmeans_supported(int C, int g, int max_smem)
{
    return C >= 1 && C <= RPTQ_MAX_CHANNELS && g >= 1 && g <= C && kmeans_smem_bytes(C, g) <= (size_t)max_smem;
}

cudaError_t launch_kmeans(const KmArgs &a)
{
    const KmWs w = km_carve(a.ws, a.C, a.g);
    const int nb = km_blocks(a.C);
    const size_t n16 = w.clear / 16;
    km_prep<<<(unsigned)std::min<size_t>((n16 + 255) / 256, (size_t)4 * a.num_sms), 256, 0, a.stream>>>(w.seeds, n16);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t sm = kmeans_smem_bytes(a.C, a.g);
    e = kernel_smem((const void *)km_fused, sm);
    if (e != cudaSuccess) return e;
    int C = a.C, g = a.g, iters = a.iters, bits = a.bits;
    KmWs wc = w;
    void *args[] = {(void *)&a.mx, (void *)&a.mn, &C, &g, &iters, &bits, &wc, (void *)&a.cent, (void *)&a.labels,
                    (void *)&a.R, (void *)&a.col_cluster, (void *)&a.offsets, (void *)&a.scale, (void *)&a.zero,
                    (void *)&a.err};
    return cudaLaunchCooperativeKernel((const void *)km_fused, dim3(nb), dim3(KM_THREADS), args, sm, a.stream);
}

}  // namespace rptq

// ==========================================================================================
// Allocation-free KMeans entry point.
//
// Some callers cannot allocate device memory once they are running: a plugin inside a host
// application that owns every byte of GPU memory through its own pool, or a serving loop that
// forbids cudaMalloc / cudaFree after start-up because they can synchronise the device and
// stall other work.  rptq_kmeans_noalloc gives them the KMeans + reorder + (s, z) call without
// a caller-provided workspace: its scratch is the fixed array below, which every GPU that
// loads this library holds until the process exits.
//
// Limits and sharing rules (also stated in include/rptq.h):
//   - the scratch holds RPTQ_KMEANS_NOALLOC_SCRATCH_BYTES (2 MiB, include/rptq.h); a (C, g) whose workspace
//     would be larger is refused with RPTQ_ERR_UNSUPPORTED (every C <= 16384 with g <= 512 fits:
//     at most 1.85 MB);
//   - all calls on one device share the array and it keeps the previous call's contents; the
//     launch sequence clears the parts that must start at zero (exchange cells, barrier words)
//     and overwrites the rest before reading it, so stale contents never leak into results;
//   - two calls whose kernels overlap on the GPU (different streams, no ordering) race on the
//     array and may give wrong results: order them on one stream or with events;
//   - the first call on a device looks up the array's device address and the device's
//     properties with that device current; make that first call before any stream capture.
// ==========================================================================================
#include <mutex>

static __device__ __align__(256) unsigned char g_kmeans_scratch[RPTQ_KMEANS_NOALLOC_SCRATCH_BYTES];

namespace {
struct NoAllocDev {
    bool ready = false;
    void *scratch = nullptr;  // device address of g_kmeans_scratch on this device
    int num_sms = 0;
    int max_smem = 0;
};
NoAllocDev g_noalloc_dev[64];
std::mutex g_noalloc_mu;

// One-time set-up per device, run with that device current.
int noalloc_setup(NoAllocDev *out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RPTQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoAllocDev &d = g_noalloc_dev[dev];
    if (!d.ready) {
        void *p = nullptr;
        // In host code g_kmeans_scratch names a host-side stand-in; this returns the address
        // of the array in the current device's memory, the only address a kernel may be given.
        if (cudaGetSymbolAddress(&p, g_kmeans_scratch) != cudaSuccess) {
            cudaGetLastError();
            return RPTQ_ERR_CUDA;
        }
        if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
                cudaSuccess) {
            cudaGetLastError();
            return RPTQ_ERR_CUDA;
        }
        d.scratch = p;
        d.ready = true;
    }
    *out = d;
    return RPTQ_OK;
}
}  // namespace

extern "C" int rptq_kmeans_noalloc(const float *ch_max, const float *ch_min, int C, int g,
                                   int iters, int bits, int32_t *labels, double *centroids,
                                   int32_t *R, int32_t *col_cluster, int32_t *offsets,
                                   float *scale, int32_t *zero, rptq_stream_t stream)
{
    if (bits != 3 && bits != 4) return RPTQ_ERR_UNSUPPORTED;
    if (C <= 0 || C > RPTQ_MAX_CHANNELS) return RPTQ_ERR_UNSUPPORTED;
    if (g <= 0 || g > C || g > RPTQ_MAX_CLUSTERS || iters < 0) return RPTQ_ERR_INVALID_ARG;
    if (!ch_max || !ch_min || !labels || !centroids || !R || !col_cluster || !offsets || !scale ||
        !zero)
        return RPTQ_ERR_INVALID_ARG;
    if (rptq::kmeans_ws_bytes(C, g) > RPTQ_KMEANS_NOALLOC_SCRATCH_BYTES) return RPTQ_ERR_UNSUPPORTED;
    NoAllocDev d;
    const int st = noalloc_setup(&d);
    if (st != RPTQ_OK) return st;
    if (!rptq::kmeans_supported(C, g, d.max_smem)) return RPTQ_ERR_UNSUPPORTED;
    int *err = rptq::device_error_word();
    if (!err) return RPTQ_ERR_CUDA;
    rptq::KmArgs a{ch_max, ch_min, C, g, iters, bits, labels, centroids, R, col_cluster, offsets,
                   scale, zero, d.scratch, (cudaStream_t)stream, d.num_sms, d.max_smem, err};
    const cudaError_t e = rptq::launch_kmeans(a);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return RPTQ_ERR_CUDA;
    }
    return RPTQ_OK;
}

// ==========================================================================================
// Testing hook (include/rptq_testing.h): the exchange wait limit and the CTA that leaves out its
// first Lloyd record, on the current device.
extern "C" int rptq_testing_kmeans_wait(unsigned long long limit_ns, int withhold_cta)
{
    const unsigned long long lim = limit_ns ? limit_ns : 2000000000ull;
    if (withhold_cta < -1) return RPTQ_ERR_INVALID_ARG;
    if (cudaMemcpyToSymbol(rptq::g_km_wait_ns, &lim, sizeof(lim)) != cudaSuccess ||
        cudaMemcpyToSymbol(rptq::g_km_withhold, &withhold_cta, sizeof(withhold_cta)) != cudaSuccess) {
        cudaGetLastError();
        return RPTQ_ERR_CUDA;
    }
    return RPTQ_OK;
}
