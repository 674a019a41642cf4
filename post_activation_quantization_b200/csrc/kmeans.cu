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
// Launch sequence on the caller's stream (no host synchronisation):
//   km_prep   zero the rank counters and control words, labels := -1
//   km_rank   rank of every point in the (max, min, index) order by counting (exact, O(C^2)
//             comparisons spread over the GPU, integer atomics)
//   km_seed   centroid k := point of rank floor((2k+1) C / (2g))
//   km_iter   x iters: assignment of one point per thread, per-CTA cluster sums in a fixed
//             order, and the last CTA to finish (atomic ticket, no waiting) folds the CTA sums
//             in CTA order into the new centroids.  Once an assignment repeats the previous one
//             the centroids are a fixed point and later launches return at once.
//   km_final  one CTA: final assignment, stable counting sort (R, col_cluster, offsets),
//             cluster ranges and (s, z).
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace rptq {

constexpr int KM_THREADS = 256;

struct KmWs {
    double *partials;  // [NB][g][3]: sum of max, sum of min, count
    int *ctrl;         // [0] ticket, [1] changed count, [2] converged flag
    int *rankcnt;      // [C]
};

__host__ __device__ inline size_t km_align(size_t v) { return (v + 255) & ~(size_t)255; }
__host__ __device__ inline int km_blocks(int C) { return (C + KM_THREADS - 1) / KM_THREADS; }

size_t kmeans_ws_bytes(int C, int g)
{
    const size_t nb = (size_t)km_blocks(C);
    return km_align(nb * (size_t)g * 3 * sizeof(double)) + 256 + km_align((size_t)C * sizeof(int));
}

static KmWs km_carve(void *ws, int C, int g)
{
    uint8_t *p = static_cast<uint8_t *>(ws);
    KmWs w;
    w.partials = reinterpret_cast<double *>(p);
    p += km_align((size_t)km_blocks(C) * (size_t)g * 3 * sizeof(double));
    w.ctrl = reinterpret_cast<int *>(p);
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

__global__ void km_prep(int C, int *rankcnt, int *ctrl, int32_t *labels)
{
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c < C) {
        rankcnt[c] = 0;
        labels[c] = -1;
    }
    if (c < 64) ctrl[c] = 0;
}

// blockIdx.x: a tile of KM_THREADS points whose rank is counted; blockIdx.y: a slice of the
// points they are compared with.
__global__ void __launch_bounds__(KM_THREADS)
    km_rank(const float *__restrict__ mx, const float *__restrict__ mn, int C, int slice, int *rankcnt)
{
    __shared__ float sx[KM_THREADS], sy[KM_THREADS];
    const int c = blockIdx.x * KM_THREADS + threadIdx.x;
    const float px = c < C ? mx[c] : 0.f, py = c < C ? mn[c] : 0.f;
    const int b0 = blockIdx.y * slice, b1 = min(C, b0 + slice);
    int cnt = 0;
    for (int t0 = b0; t0 < b1; t0 += KM_THREADS) {
        const int o = t0 + threadIdx.x;
        __syncthreads();
        sx[threadIdx.x] = o < b1 ? mx[o] : 0.f;
        sy[threadIdx.x] = o < b1 ? mn[o] : 0.f;
        __syncthreads();
        const int n = min(KM_THREADS, b1 - t0);
        for (int i = 0; i < n; ++i) cnt += key_less(sx[i], sy[i], t0 + i, px, py, c) ? 1 : 0;
    }
    if (c < C && cnt) atomicAdd(rankcnt + c, cnt);
}

__global__ void km_seed(const float *__restrict__ mx, const float *__restrict__ mn, int C, int g,
                        const int *__restrict__ rankcnt, double *cent)
{
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= C) return;
    const int64_t r = rankcnt[c];
    // the k with floor((2k+1) C / (2g)) == r, if any
    const int64_t num = 2 * (int64_t)g * r - C;
    int64_t k = num <= 0 ? 0 : (num + 2 * (int64_t)C - 1) / (2 * (int64_t)C);
    if (k < g && ((2 * k + 1) * (int64_t)C) / (2 * (int64_t)g) == r) {
        cent[2 * k] = (double)mx[c];
        cent[2 * k + 1] = (double)mn[c];
    }
}

__global__ void __launch_bounds__(KM_THREADS)
    km_iter(const float *__restrict__ mx, const float *__restrict__ mn, int C, int g, double *cent,
            int32_t *labels, double *partials, int *ctrl, int iter)
{
    if (*(volatile int *)(ctrl + 2)) return;  // converged earlier: nothing can change
    extern __shared__ double ksm[];
    double *cx = ksm, *cy = ksm + g;
    __shared__ int slab[KM_THREADS];
    __shared__ double spx[KM_THREADS], spy[KM_THREADS];
    __shared__ int s_changed, s_last;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int k = tid; k < g; k += KM_THREADS) {
        cx[k] = cent[2 * k];
        cy[k] = cent[2 * k + 1];
    }
    if (tid == 0) s_changed = 0;
    __syncthreads();

    const int c = blockIdx.x * KM_THREADS + tid;
    int lab = -1;
    double px = 0.0, py = 0.0;
    if (c < C) {
        px = (double)mx[c];
        py = (double)mn[c];
        double best = sq_dist(px, py, cx[0], cy[0]);
        lab = 0;
        for (int k = 1; k < g; ++k) {
            const double d = sq_dist(px, py, cx[k], cy[k]);
            if (d < best) {
                best = d;
                lab = k;
            }
        }
        if (labels[c] != lab) atomicAdd(&s_changed, 1);
        labels[c] = lab;
    }
    slab[tid] = lab;
    spx[tid] = px;
    spy[tid] = py;
    __syncthreads();

    // per-CTA sums of each cluster in a fixed order: lane strides, then a butterfly
    for (int k = warp; k < g; k += KM_THREADS / 32) {
        double sx = 0.0, sy = 0.0, n = 0.0;
#pragma unroll
        for (int i = 0; i < KM_THREADS / 32; ++i) {
            const int p = lane + 32 * i;
            if (slab[p] == k) {
                sx = __dadd_rn(sx, spx[p]);
                sy = __dadd_rn(sy, spy[p]);
                n += 1.0;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            sx = __dadd_rn(sx, __shfl_xor_sync(FULL, sx, o));
            sy = __dadd_rn(sy, __shfl_xor_sync(FULL, sy, o));
            n += __shfl_xor_sync(FULL, n, o);
        }
        if (lane == 0) {
            double *pp = partials + ((size_t)blockIdx.x * g + k) * 3;
            pp[0] = sx;
            pp[1] = sy;
            pp[2] = n;
        }
    }
    __threadfence();  // every writer publishes its sums before the ticket below
    __syncthreads();
    if (tid == 0) {
        if (s_changed) atomicAdd(ctrl + 1, s_changed);
        __threadfence();
        s_last = atomicAdd(ctrl + 0, 1) == (int)gridDim.x - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int nb = gridDim.x;
    for (int k = tid; k < g; k += KM_THREADS) {
        double sx = 0.0, sy = 0.0, n = 0.0;
        for (int b = 0; b < nb; ++b) {
            const double *pp = partials + ((size_t)b * g + k) * 3;
            sx = __dadd_rn(sx, __ldcg(pp));
            sy = __dadd_rn(sy, __ldcg(pp + 1));
            n += __ldcg(pp + 2);
        }
        if (n > 0.0) {
            cent[2 * k] = __ddiv_rn(sx, n);
            cent[2 * k + 1] = __ddiv_rn(sy, n);
        }
    }
    if (tid == 0) {
        const int changed = __ldcg(ctrl + 1);
        if (changed == 0 && iter > 0) ctrl[2] = 1;
        ctrl[1] = 0;
        ctrl[0] = 0;
        __threadfence();
    }
}

// One CTA of 1024 threads.  Dynamic shared memory (bytes):
//   labs C*4 | cent 2g*8 | counts g*4 | base g*4 | cmax g*4 | cmin g*4 | wcnt 32*g*4
size_t km_final_smem(int C, int g) { return (size_t)C * 4 + (size_t)g * 16 + (size_t)g * 16 + (size_t)g * 128; }

__global__ void __launch_bounds__(1024)
    km_final(const float *__restrict__ mx, const float *__restrict__ mn, int C, int g, int bits,
             const double *__restrict__ cent, int32_t *labels, int32_t *R, int32_t *col_cluster,
             int32_t *offsets, float *scale, int32_t *zero)
{
    extern __shared__ __align__(16) uint8_t fsm[];
    int *labs = reinterpret_cast<int *>(fsm);
    double *cc = reinterpret_cast<double *>(fsm + (size_t)C * 4 + ((size_t)C * 4 % 8));
    int *counts = reinterpret_cast<int *>(cc + 2 * g);
    int *base = counts + g;
    float *cmax = reinterpret_cast<float *>(base + g);
    float *cmin = cmax + g;
    int *wcnt = reinterpret_cast<int *>(cmin + g);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int k = tid; k < g; k += blockDim.x) {
        cc[2 * k] = cent[2 * k];
        cc[2 * k + 1] = cent[2 * k + 1];
        counts[k] = 0;
        cmax[k] = -INFINITY;
        cmin[k] = INFINITY;
    }
    __syncthreads();
    // final assignment, cluster sizes and ranges
    for (int c = tid; c < C; c += blockDim.x) {
        const float fx = mx[c], fy = mn[c];
        const double px = (double)fx, py = (double)fy;
        double best = sq_dist(px, py, cc[0], cc[1]);
        int lab = 0;
        for (int k = 1; k < g; ++k) {
            const double d = sq_dist(px, py, cc[2 * k], cc[2 * k + 1]);
            if (d < best) {
                best = d;
                lab = k;
            }
        }
        labs[c] = lab;
        labels[c] = lab;
        atomicAdd(counts + lab, 1);
        atomic_max_f32(cmax + lab, fx);
        atomic_min_f32(cmin + lab, fy);
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
    __syncthreads();
    // stable counting sort, 1024 channels at a time in channel order
    for (int c0 = 0; c0 < C; c0 += blockDim.x) {
        for (int i = tid; i < 32 * g; i += blockDim.x) wcnt[i] = 0;
        __syncthreads();
        const int c = c0 + tid;
        const int L = c < C ? labs[c] : -1;
        const unsigned same = __match_any_sync(FULL, L);
        const unsigned lower = same & ((1u << lane) - 1u);
        const int rank = __popc(lower);
        if (L >= 0 && lower == 0) wcnt[warp * g + L] = __popc(same);
        __syncthreads();
        for (int k = tid; k < g; k += blockDim.x) {
            int run = base[k];
            for (int w = 0; w < 32; ++w) {
                const int t = wcnt[w * g + k];
                wcnt[w * g + k] = run;
                run += t;
            }
            base[k] = run;
        }
        __syncthreads();
        if (L >= 0) {
            const int pos = wcnt[warp * g + L] + rank;
            R[pos] = c;
            col_cluster[pos] = L;
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
    km_prep<<<std::max(nb, 1), KM_THREADS, 0, a.stream>>>(a.C, w.rankcnt, w.ctrl, a.labels);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // rank counting: about 4 CTAs per SM, slices of at least one tile
    int splits = std::max(1, std::min((a.num_sms * 4 + nb - 1) / nb, (a.C + KM_THREADS - 1) / KM_THREADS));
    const int slice = ((a.C + splits - 1) / splits + KM_THREADS - 1) / KM_THREADS * KM_THREADS;
    splits = (a.C + slice - 1) / slice;
    km_rank<<<dim3(nb, splits), KM_THREADS, 0, a.stream>>>(a.mx, a.mn, a.C, slice, w.rankcnt);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    km_seed<<<nb, KM_THREADS, 0, a.stream>>>(a.mx, a.mn, a.C, a.g, w.rankcnt, a.cent);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t ism = (size_t)a.g * 2 * sizeof(double);
    if (ism > 48 * 1024) {
        e = cudaFuncSetAttribute(km_iter, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ism);
        if (e != cudaSuccess) return e;
    }
    for (int it = 0; it < a.iters; ++it) {
        km_iter<<<nb, KM_THREADS, ism, a.stream>>>(a.mx, a.mn, a.C, a.g, a.cent, a.labels, w.partials,
                                                    w.ctrl, it);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const size_t fsm = km_final_smem(a.C, a.g) + 16;
    e = cudaFuncSetAttribute(km_final, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fsm);
    if (e != cudaSuccess) return e;
    km_final<<<1, 1024, fsm, a.stream>>>(a.mx, a.mn, a.C, a.g, a.bits, a.cent, a.labels, a.R,
                                         a.col_cluster, a.offsets, a.scale, a.zero);
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
//     would be larger is refused with RPTQ_ERR_UNSUPPORTED (every C <= 16384 fits for g <= 512);
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
    if (rptq::km_final_smem(C, g) + 16 > (size_t)d.max_smem) return RPTQ_ERR_UNSUPPORTED;
    rptq::KmArgs a{ch_max, ch_min, C, g, iters, bits, labels, centroids, R, col_cluster, offsets,
                   scale, zero, d.scratch, (cudaStream_t)stream, d.num_sms};
    const cudaError_t e = rptq::launch_kmeans(a);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return RPTQ_ERR_CUDA;
    }
    return RPTQ_OK;
}
