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
// Launch sequence on the caller's stream (no host synchronisation), four kernels:
//   km_prep   zero the rank counters and the grid-barrier words
//   km_rank   rank of every point in the (max, min, index) order by counting (exact, O(C^2)
//             comparisons spread over the GPU, integer atomics)
//   km_lloyd  one cooperative launch of ceil(C/256) CTAs, one point per thread: quantile seeds
//             (every CTA finds the points of rank floor((2k+1) C / (2g))), then per iteration
//             assignment, per-CTA cluster sums in a fixed order, one grid barrier, and every CTA
//             folds all CTA sums in the same fixed order into identical new centroids.  The
//             per-CTA sums are double-buffered by iteration parity, so one barrier per
//             iteration suffices.  An assignment that repeats the previous one ends the loop
//             (a fixed point: the remaining rounds would change nothing).  Then the final
//             assignment writes the labels.  The barrier waits are bounded (2 s, then the
//             device error word) so a stalled CTA cannot hang the GPU.
//   km_final  one CTA: stable counting sort (R, col_cluster, offsets), cluster ranges, (s, z).
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace rptq {

constexpr int KM_THREADS = 256;

struct KmWs {
    double *partials;  // [2][NB][g][3]: sum of max, sum of min, count (by iteration parity)
    int *chg;          // [2][NB]: labels changed per CTA
    unsigned *bar;     // [0] arrivals, [1] generation of the grid barrier
    int *rankcnt;      // [C]
};

__host__ __device__ inline size_t km_align(size_t v) { return (v + 255) & ~(size_t)255; }
__host__ __device__ inline int km_blocks(int C) { return (C + KM_THREADS - 1) / KM_THREADS; }

size_t kmeans_ws_bytes(int C, int g)
{
    const size_t nb = (size_t)km_blocks(C);
    return km_align(2 * nb * (size_t)g * 3 * sizeof(double)) + km_align(2 * nb * sizeof(int)) + 256 +
           km_align((size_t)C * sizeof(int));
}

static KmWs km_carve(void *ws, int C, int g)
{
    const size_t nb = (size_t)km_blocks(C);
    uint8_t *p = static_cast<uint8_t *>(ws);
    KmWs w;
    w.partials = reinterpret_cast<double *>(p);
    p += km_align(2 * nb * (size_t)g * 3 * sizeof(double));
    w.chg = reinterpret_cast<int *>(p);
    p += km_align(2 * nb * sizeof(int));
    w.bar = reinterpret_cast<unsigned *>(p);
    p += 256;
    w.rankcnt = reinterpret_cast<int *>(p);
    return w;
}

__device__ __forceinline__ bool key_less(float ax, float ay, int ai, float bx, float by, int bi)
{
    if (ax != bx) return ax < bx;
    if (ay != by) return ay < by;
    return ai < bi;
}

__device__ __forceinline__ double sq_dist(double px, double py, double cx, double cy)
{
    const double dx = __dsub_rn(px, cx), dy = __dsub_rn(py, cy);
    return __dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy));
}

__device__ __forceinline__ int nearest(double px, double py, const double *cx, const double *cy, int g)
{
    double best = sq_dist(px, py, cx[0], cy[0]);
    int lab = 0;
    for (int k = 1; k < g; ++k) {
        const double d = sq_dist(px, py, cx[k], cy[k]);
        if (d < best) {  // strict: ties keep the lowest index
            best = d;
            lab = k;
        }
    }
    return lab;
}

__global__ void km_prep(int C, int *rankcnt, unsigned *bar)
{
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c < C) rankcnt[c] = 0;
    if (c < 64) bar[c] = 0;
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

// Rank of every point in the (max, min, index) order, by counting.  blockIdx.x: 4*KM_THREADS
// points (4 per thread) whose rank is counted; blockIdx.y: the slice of points compared with.
constexpr int KM_RANK_PPT = 4;
__global__ void __launch_bounds__(KM_THREADS)
    km_rank(const float *__restrict__ mx, const float *__restrict__ mn, int C, int slice, int *rankcnt)
{
    __shared__ uint64_t skey[KM_THREADS];
    uint64_t key[KM_RANK_PPT];
    int idx[KM_RANK_PPT], cnt[KM_RANK_PPT];
#pragma unroll
    for (int j = 0; j < KM_RANK_PPT; ++j) {
        idx[j] = blockIdx.x * KM_THREADS * KM_RANK_PPT + j * KM_THREADS + threadIdx.x;
        key[j] = idx[j] < C ? point_key(mx[idx[j]], mn[idx[j]]) : 0;
        cnt[j] = 0;
    }
    const int b0 = blockIdx.y * slice, b1 = min(C, b0 + slice);
    for (int t0 = b0; t0 < b1; t0 += KM_THREADS) {
        const int o = t0 + threadIdx.x;
        __syncthreads();
        skey[threadIdx.x] = o < b1 ? point_key(mx[o], mn[o]) : ~0ull;
        __syncthreads();
        const int n = min(KM_THREADS, b1 - t0);
        for (int i = 0; i < n; ++i) {
            const uint64_t kb = skey[i];
            const int ib = t0 + i;
#pragma unroll
            for (int j = 0; j < KM_RANK_PPT; ++j) cnt[j] += (kb < key[j]) | ((kb == key[j]) & (ib < idx[j]));
        }
    }
#pragma unroll
    for (int j = 0; j < KM_RANK_PPT; ++j)
        if (idx[j] < C && cnt[j]) atomicAdd(rankcnt + idx[j], cnt[j]);
}

// Grid-wide barrier for a cooperative launch: arrival counter + generation word.  The wait is
// bounded by wall time; on expiry the device error word is set and the CTA goes on.
__device__ __forceinline__ void km_grid_barrier(unsigned *bar, int *err)
{
    __syncthreads();
    if (threadIdx.x == 0) {
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
                if ((++spin & 255u) == 0 && global_ns() - t0 > 2000000000ull) {
                    raise_error(err, RPTQ_DEVERR_TIMEOUT);
                    break;
                }
            }
        }
    }
    __syncthreads();
}

__global__ void __launch_bounds__(KM_THREADS)
    km_lloyd(const float *__restrict__ mx, const float *__restrict__ mn, int C, int g, int iters,
             const int *__restrict__ rankcnt, double *cent, int32_t *labels, double *partials, int *chg,
             unsigned *bar, int *err)
{
    extern __shared__ double ksm[];
    double *cx = ksm, *cy = ksm + g;
    double *wsum = ksm + 2 * g;  // [8 warps][g][3]: per-warp cluster sums
    double *tot = wsum + 8 * 3 * g;  // [g][3]: all-CTA totals
    __shared__ double spx[KM_THREADS], spy[KM_THREADS];
    __shared__ int s_stop;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nb = gridDim.x;
    const int G3 = 3 * g;

    // quantile seeds: the point of rank floor((2k+1) C / (2g)) becomes centroid k
    for (int c = tid; c < C; c += KM_THREADS) {
        const int64_t r = rankcnt[c];
        const int64_t num = 2 * (int64_t)g * r - C;
        const int64_t k = num <= 0 ? 0 : (num + 2 * (int64_t)C - 1) / (2 * (int64_t)C);
        if (k < g && ((2 * k + 1) * (int64_t)C) / (2 * (int64_t)g) == r) {
            cx[k] = (double)mx[c];
            cy[k] = (double)mn[c];
        }
    }
    const int c = blockIdx.x * KM_THREADS + tid;
    const bool own = c < C;
    const double px = own ? (double)mx[c] : 0.0, py = own ? (double)mn[c] : 0.0;
    spx[tid] = px;
    spy[tid] = py;
    int prev = -1;
    __syncthreads();

    for (int it = 0; it < iters; ++it) {
        const int par = it & 1;
        for (int i = tid; i < 8 * G3; i += KM_THREADS) wsum[i] = 0.0;
        const int lab = own ? nearest(px, py, cx, cy, g) : -1;
        const int changed = __syncthreads_count(own && lab != prev);  // also orders the zeroing
        prev = lab;
        // per-warp sums: the lowest lane of each same-label group adds the group in lane order
        const unsigned same = __match_any_sync(FULL, lab);
        if (lab >= 0 && (same & ((1u << lane) - 1u)) == 0) {
            double sx = 0.0, sy = 0.0;
            for (unsigned m = same; m; m &= m - 1) {
                const int j = warp * 32 + __ffs(m) - 1;
                sx = __dadd_rn(sx, spx[j]);
                sy = __dadd_rn(sy, spy[j]);
            }
            double *w = wsum + (warp * g + lab) * 3;
            w[0] = sx;
            w[1] = sy;
            w[2] = (double)__popc(same);
        }
        __syncthreads();
        // this CTA's sums: warps folded in warp order
        double *mine = partials + ((size_t)par * nb + blockIdx.x) * (size_t)G3;
        for (int t = tid; t < G3; t += KM_THREADS) {
            double a = 0.0;
#pragma unroll
            for (int w = 0; w < KM_THREADS / 32; ++w) a = __dadd_rn(a, wsum[w * G3 + t]);
            mine[t] = a;
        }
        if (tid == 0) chg[par * nb + blockIdx.x] = changed;
        __threadfence();
        km_grid_barrier(bar, err);

        // every CTA folds all CTA sums in CTA order (16 loads in flight per thread)
        const double *all = partials + (size_t)par * nb * (size_t)G3;
        for (int t = tid; t < G3; t += KM_THREADS) {
            double a = 0.0;
            for (int b0 = 0; b0 < nb; b0 += 16) {
                double v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = b0 + i < nb ? __ldcg(all + (size_t)(b0 + i) * G3 + t) : 0.0;
#pragma unroll
                for (int i = 0; i < 16; ++i) a = __dadd_rn(a, v[i]);
            }
            tot[t] = a;
        }
        if (warp == (KM_THREADS / 32) - 1) {
            int tc = 0;
            for (int b = lane; b < nb; b += 32) tc += __ldcg(chg + par * nb + b);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) tc += __shfl_xor_sync(FULL, tc, o);
            if (lane == 0) s_stop = (tc == 0 && it > 0);
        }
        __syncthreads();
        for (int k = tid; k < g; k += KM_THREADS) {
            const double n = tot[3 * k + 2];
            if (n > 0.0) {  // an empty cluster keeps its centroid
                cx[k] = __ddiv_rn(tot[3 * k], n);
                cy[k] = __ddiv_rn(tot[3 * k + 1], n);
            }
        }
        __syncthreads();
        if (s_stop) break;
    }
    if (own) labels[c] = nearest(px, py, cx, cy, g);  // the final assignment
    if (blockIdx.x == 0)
        for (int k = tid; k < g; k += KM_THREADS) {
            cent[2 * k] = cx[k];
            cent[2 * k + 1] = cy[k];
        }
}
size_t km_lloyd_smem(int g, int nb) { return (size_t)g * 16 + (size_t)g * 3 * 8 * (8 + 1); }

// One CTA of 1024 threads: stable counting sort by label, cluster ranges, (s, z).
// Channels are taken in groups of 32 (one warp); a batch of NGB groups is counted per cluster
// into `hist`, scanned per cluster in group order (carrying the running count `base` from the
// previous batch), and each channel's stored position is its cluster's running count at its
// group plus its rank among the same-cluster lanes of its group.
// Dynamic shared memory: labs C ints | counts, base g ints | cmax, cmin g floats | hist NGB*g.
size_t km_final_smem(int C, int g, int ngb) { return (size_t)C * 4 + (size_t)g * 16 + (size_t)ngb * g * 4; }
int km_final_batch(int C, int g, int max_smem)
{
    const int NG = (C + 31) / 32;
    const long long room = (long long)max_smem - 64 - (long long)C * 4 - (long long)g * 16;
    if (room < 4LL * g) return 0;
    return (int)std::min<long long>(NG, room / (4LL * g));
}

__global__ void __launch_bounds__(1024)
    km_final(const float *__restrict__ mx, const float *__restrict__ mn, int C, int g, int bits, int NGB,
             const int32_t *__restrict__ labels, int32_t *R, int32_t *col_cluster, int32_t *offsets,
             float *scale, int32_t *zero)
{
    extern __shared__ __align__(16) uint8_t fsm[];
    const int NG = (C + 31) / 32;
    int *labs = reinterpret_cast<int *>(fsm);
    int *counts = labs + C;
    int *base = counts + g;
    float *cmax = reinterpret_cast<float *>(base + g);
    float *cmin = cmax + g;
    int *hist = reinterpret_cast<int *>(cmin + g);  // [NGB][g]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, NW = blockDim.x >> 5;
    for (int k = tid; k < g; k += blockDim.x) {
        counts[k] = 0;
        cmax[k] = -INFINITY;
        cmin[k] = INFINITY;
    }
    __syncthreads();
    for (int c = tid; c < C; c += blockDim.x) {
        int L = labels[c];
        L = L < 0 ? 0 : (L >= g ? g - 1 : L);  // labels come from km_lloyd, always in range
        labs[c] = L;
        atomicAdd(counts + L, 1);
        atomic_max_f32(cmax + L, mx[c]);
        atomic_min_f32(cmin + L, mn[c]);
    }
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int k = 0; k < g; ++k) {
            offsets[k] = run;
            base[k] = run;
            run += counts[k];
        }
        offsets[g] = run;
    }
    // TPC threads scan one cluster: a power of two <= 32 (segments of one warp), TPC * g <= 1024
    int TPC = 1;
    while (TPC < 32 && 2 * TPC * g <= (int)blockDim.x) TPC *= 2;
    for (int gb0 = 0; gb0 < NG; gb0 += NGB) {
        const int nbg = min(NGB, NG - gb0);
        for (int i = tid; i < nbg * g; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        for (int gi = warp; gi < nbg; gi += NW) {
            const int c = (gb0 + gi) * 32 + lane;
            const int L = c < C ? labs[c] : -1;
            const unsigned same = __match_any_sync(FULL, L);
            if (L >= 0 && (same & ((1u << lane) - 1u)) == 0) hist[gi * g + L] = __popc(same);
        }
        __syncthreads();
        // exclusive scan of hist[.][k] over this batch's groups, TPC threads per cluster
        for (int k0 = 0; k0 < g; k0 += blockDim.x / TPC) {
            const int k = k0 + tid / TPC, part = tid % TPC;
            const int seg = (nbg + TPC - 1) / TPC;
            const int i0 = min(nbg, part * seg), i1 = min(nbg, i0 + seg);
            int local = 0;
            if (k < g)
                for (int i = i0; i < i1; ++i) local += hist[i * g + k];
            int incl = local;
            for (int o = 1; o < TPC; o <<= 1) {  // TPC divides 32: segments of one warp
                const int v = __shfl_up_sync(FULL, incl, o, TPC);
                if (part >= o) incl += v;
            }
            const int total = __shfl_sync(FULL, incl, TPC - 1, TPC);
            if (k < g) {
                int run = base[k] + incl - local;
                for (int i = i0; i < i1; ++i) {
                    const int t = hist[i * g + k];
                    hist[i * g + k] = run;
                    run += t;
                }
            }
            __syncwarp();
            if (k < g && part == 0) base[k] += total;
        }
        __syncthreads();
        for (int gi = warp; gi < nbg; gi += NW) {
            const int c = (gb0 + gi) * 32 + lane;
            const int L = c < C ? labs[c] : -1;
            const unsigned same = __match_any_sync(FULL, L);
            if (L >= 0) {
                const int pos = hist[gi * g + L] + __popc(same & ((1u << lane) - 1u));
                R[pos] = c;
                col_cluster[pos] = L;
            }
        }
        __syncthreads();
    }
    // per-cluster scale and zero point (fp32 IEEE operations, round half to even)
    const float qmax = (float)((1 << bits) - 1);
    for (int k = tid; k < g; k += blockDim.x) {
        if (counts[k] == 0) {
            scale[k] = 1.0f;
            zero[k] = 0;
            continue;
        }
        const float M = cmax[k], m = cmin[k];
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

cudaError_t launch_kmeans(const KmArgs &a)
{
    const KmWs w = km_carve(a.ws, a.C, a.g);
    const int nb = km_blocks(a.C);
    cudaError_t e;
    km_prep<<<std::max(nb, 1), KM_THREADS, 0, a.stream>>>(a.C, w.rankcnt, w.bar);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // rank counting: about 4 CTAs per SM, slices of at least one tile
    const int nbr = (a.C + KM_THREADS * KM_RANK_PPT - 1) / (KM_THREADS * KM_RANK_PPT);
    int splits = std::max(1, std::min((a.num_sms * 4 + nbr - 1) / nbr, (a.C + KM_THREADS - 1) / KM_THREADS));
    const int slice = ((a.C + splits - 1) / splits + KM_THREADS - 1) / KM_THREADS * KM_THREADS;
    splits = (a.C + slice - 1) / slice;
    km_rank<<<dim3(nbr, splits), KM_THREADS, 0, a.stream>>>(a.mx, a.mn, a.C, slice, w.rankcnt);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t lsm = km_lloyd_smem(a.g, nb);
    e = cudaFuncSetAttribute(km_lloyd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lsm);
    if (e != cudaSuccess) return e;
    int g = a.g, C = a.C, iters = a.iters;
    void *args[] = {(void *)&a.mx, (void *)&a.mn, &C, &g, &iters, (void *)&w.rankcnt, (void *)&a.cent,
                    (void *)&a.labels, (void *)&w.partials, (void *)&w.chg, (void *)&w.bar, (void *)&a.err};
    e = cudaLaunchCooperativeKernel((const void *)km_lloyd, dim3(nb), dim3(KM_THREADS), args, lsm, a.stream);
    if (e != cudaSuccess) return e;
    const int ngb = km_final_batch(a.C, a.g, a.max_smem);
    if (ngb < 1) return cudaErrorInvalidValue;
    const size_t fsm = km_final_smem(a.C, a.g, ngb) + 16;
    e = cudaFuncSetAttribute(km_final, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fsm);
    if (e != cudaSuccess) return e;
    km_final<<<1, 1024, fsm, a.stream>>>(a.mx, a.mn, a.C, a.g, a.bits, ngb, a.labels, a.R, a.col_cluster,
                                         a.offsets, a.scale, a.zero);
    return cudaGetLastError();
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
//   - the scratch holds RPTQ_KMEANS_NOALLOC_SCRATCH_BYTES (1 MiB, include/rptq.h); a (C, g) whose workspace
//     would be larger is refused with RPTQ_ERR_UNSUPPORTED (every C <= 16384 fits for g <= 256);
//   - all calls on one device share the array and it keeps the previous call's contents; the
//     launch sequence clears the parts that must start at zero (rank counters, control words)
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
    if (rptq::km_final_batch(C, g, d.max_smem) < 1) return RPTQ_ERR_UNSUPPORTED;
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
