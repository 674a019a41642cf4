// api.cu -- the extern "C" entry points of librptq.so (declared in include/rptq.h).
//
// Every entry point validates its arguments on the host, then enqueues kernels on the
// caller's stream and returns without synchronising.  Nothing here allocates device memory:
// the only library-owned device storage is the sticky error word below.
#include <algorithm>
#include <cstdio>
#include <mutex>
#include <unordered_map>

#include "../../include/rptq_baseline.h"
#include "common.cuh"
#include "launch.h"

namespace rptq {

// Sticky device error word (one per device that loads the library).
__device__ int g_device_error;

namespace {
constexpr int kMaxDevices = 64;
struct DevInfo {
    bool ready = false;
    int num_sms = 0;
    int max_smem = 0;
    int *err = nullptr;
};
DevInfo g_dev[kMaxDevices];
std::mutex g_mu;

// ---- launch settings, cached per kernel and device -------------------------------------
struct SmemKey {
    const void *f;
    int dev;
    bool operator==(const SmemKey &o) const { return f == o.f && dev == o.dev; }
};
struct OccKey {
    const void *f;
    int dev, threads;
    size_t smem;
    bool operator==(const OccKey &o) const
    {
        return f == o.f && dev == o.dev && threads == o.threads && smem == o.smem;
    }
};
struct KeyHash {
    size_t operator()(const SmemKey &k) const { return std::hash<const void *>()(k.f) * 31u + (size_t)k.dev; }
    size_t operator()(const OccKey &k) const
    {
        return ((std::hash<const void *>()(k.f) * 31u + (size_t)k.dev) * 31u + (size_t)k.threads) * 31u + k.smem;
    }
};
std::mutex g_launch_mu;
std::unordered_map<SmemKey, size_t, KeyHash> g_smem_set;
std::unordered_map<OccKey, int, KeyHash> g_occupancy;

// Per-device facts, looked up once per device with that device current.
int dev_info(DevInfo *out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RPTQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DevInfo &d = g_dev[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return RPTQ_ERR_CUDA;
        if (cudaDeviceGetAttribute(&d.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
            return RPTQ_ERR_CUDA;
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return RPTQ_ERR_CUDA;
        d.err = static_cast<int *>(p);
        d.ready = true;
    }
    *out = d;
    return RPTQ_OK;
}

}  // namespace

cudaError_t kernel_smem(const void *func, size_t bytes)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const SmemKey k{func, dev};
    {
        std::lock_guard<std::mutex> lock(g_launch_mu);
        auto it = g_smem_set.find(k);
        if (it != g_smem_set.end() && it->second >= bytes) return cudaSuccess;
    }
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) {
        std::lock_guard<std::mutex> lock(g_launch_mu);
        size_t &v = g_smem_set[k];
        v = std::max(v, bytes);
    }
    return e;
}

cudaError_t kernel_occupancy(int *per_sm, const void *func, int threads, size_t smem)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const OccKey k{func, dev, threads, smem};
    {
        std::lock_guard<std::mutex> lock(g_launch_mu);
        auto it = g_occupancy.find(k);
        if (it != g_occupancy.end()) {
            *per_sm = it->second;
            return cudaSuccess;
        }
    }
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, func, threads, smem);
    if (e == cudaSuccess) {
        std::lock_guard<std::mutex> lock(g_launch_mu);
        g_occupancy[k] = *per_sm;
    }
    return e;
}

int *device_error_word()
{
    DevInfo d;
    return dev_info(&d) == RPTQ_OK ? d.err : nullptr;
}

namespace {
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool dtype_ok(int d) { return d == RPTQ_F32 || d == RPTQ_F16 || d == RPTQ_BF16; }
int esize(int d) { return d == RPTQ_F32 ? 4 : 2; }

int cuda_status(cudaError_t e)
{
    if (e == cudaSuccess) return RPTQ_OK;
    cudaGetLastError();  // clear a sticky launch-configuration error of this thread
    return RPTQ_ERR_CUDA;
}
}  // namespace
}  // namespace rptq

using namespace rptq;

extern "C" {

const char *rptq_status_string(int status)
{
    switch (status) {
    case RPTQ_OK: return "ok";
    case RPTQ_ERR_INVALID_ARG: return "invalid argument";
    case RPTQ_ERR_UNSUPPORTED: return "unsupported shape, bit width or type";
    case RPTQ_ERR_WORKSPACE: return "workspace missing or too small";
    case RPTQ_ERR_CUDA: return "CUDA error";
    case RPTQ_ERR_DEVICE: return "device-side error flag set";
    default: return "unknown status";
    }
}

int rptq_version(void) { return 100; }

int rptq_device_error(rptq_stream_t stream, int *code)
{
    if (!code) return RPTQ_ERR_INVALID_ARG;
    DevInfo d;
    int st = dev_info(&d);
    if (st) return st;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return cuda_status(cudaErrorUnknown);
    int v = 0;
    if (cudaMemcpy(&v, d.err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return cuda_status(cudaErrorUnknown);
    const int zero = 0;
    if (cudaMemcpy(d.err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
        return cuda_status(cudaErrorUnknown);
    *code = v;
    return RPTQ_OK;
}

int rptq_calib_minmax(const void *x, int dtype, int64_t T, int C, const float *gamma,
                      const float *beta, float eps, float *ch_max, float *ch_min, int accumulate,
                      rptq_stream_t stream)
{
    if (!dtype_ok(dtype)) return RPTQ_ERR_UNSUPPORTED;
    if (C <= 0 || C % 8 != 0 || C > RPTQ_MAX_CHANNELS) return RPTQ_ERR_UNSUPPORTED;
    if (T < 0 || !ch_max || !ch_min || (accumulate != 0 && accumulate != 1)) return RPTQ_ERR_INVALID_ARG;
    if (T > 0 && (!x || !aligned16(x))) return RPTQ_ERR_INVALID_ARG;
    if ((gamma == nullptr) != (beta == nullptr)) return RPTQ_ERR_INVALID_ARG;
    if (gamma && !(eps >= 0.0f)) return RPTQ_ERR_INVALID_ARG;
    DevInfo d;
    int st = dev_info(&d);
    if (st) return st;
    CalibArgs a{x, dtype, T, C, gamma, beta, eps, ch_max, ch_min, accumulate, d.err,
                (cudaStream_t)stream, d.num_sms, d.max_smem};
    return cuda_status(launch_calib(a));
}

int rptq_kv_calib_minmax(const void *kv, int dtype, int B, int H, int64_t S, int D, float *ch_max,
                         float *ch_min, int accumulate, rptq_stream_t stream)
{
    if (!dtype_ok(dtype)) return RPTQ_ERR_UNSUPPORTED;
    if (D <= 0 || D % 8 != 0 || D > 2048 || H <= 0 || (int64_t)H * D > RPTQ_MAX_CHANNELS)
        return RPTQ_ERR_UNSUPPORTED;
    if (B < 0 || S < 0 || !ch_max || !ch_min || (accumulate != 0 && accumulate != 1))
        return RPTQ_ERR_INVALID_ARG;
    if (B > 0 && S > 0 && (!kv || !aligned16(kv))) return RPTQ_ERR_INVALID_ARG;
    if ((int64_t)B * H > 0x7fffffffLL) return RPTQ_ERR_UNSUPPORTED;
    DevInfo d;
    int st = dev_info(&d);
    if (st) return st;
    KvCalibArgs a{kv, dtype, B, H, S, D, ch_max, ch_min, accumulate, d.err, (cudaStream_t)stream, d.num_sms};
    return cuda_status(launch_kv_calib(a));
}

size_t rptq_kmeans_workspace_size(int C, int g)
{
    if (C <= 0 || g <= 0 || g > C || C > RPTQ_MAX_CHANNELS || g > RPTQ_MAX_CLUSTERS) return 0;
    return kmeans_ws_bytes(C, g);
}

int rptq_kmeans(const float *ch_max, const float *ch_min, int C, int g, int iters, int bits,
                int32_t *labels, double *centroids, int32_t *R, int32_t *col_cluster,
                int32_t *offsets, float *scale, int32_t *zero, void *workspace,
                size_t workspace_bytes, rptq_stream_t stream)
{
    if (bits != 3 && bits != 4) return RPTQ_ERR_UNSUPPORTED;
    if (C <= 0 || C > RPTQ_MAX_CHANNELS) return RPTQ_ERR_UNSUPPORTED;
    if (g <= 0 || g > C || g > RPTQ_MAX_CLUSTERS || iters < 0) return RPTQ_ERR_INVALID_ARG;
    if (!ch_max || !ch_min || !labels || !centroids || !R || !col_cluster || !offsets || !scale ||
        !zero)
        return RPTQ_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < kmeans_ws_bytes(C, g)) return RPTQ_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return RPTQ_ERR_WORKSPACE;
    DevInfo d;
    int st = dev_info(&d);
    if (st) return st;
    if (!kmeans_supported(C, g, d.max_smem)) return RPTQ_ERR_UNSUPPORTED;
    KmArgs a{ch_max, ch_min, C, g, iters, bits, labels, centroids, R, col_cluster, offsets,
             scale, zero, workspace, (cudaStream_t)stream, d.num_sms, d.max_smem, d.err};
    return cuda_status(launch_kmeans(a));
}

int rptq_cluster_params(const float *ch_max, const float *ch_min, int C, const int32_t *labels,
                        int g, int bits, float *scale, int32_t *zero, rptq_stream_t stream)
{
    if (bits != 3 && bits != 4) return RPTQ_ERR_UNSUPPORTED;
    if (C <= 0 || C > RPTQ_MAX_CHANNELS) return RPTQ_ERR_UNSUPPORTED;
    if (g <= 0 || g > C || g > RPTQ_MAX_CLUSTERS) return RPTQ_ERR_INVALID_ARG;
    if (!ch_max || !ch_min || !labels || !scale || !zero) return RPTQ_ERR_INVALID_ARG;
    DevInfo d;
    int st = dev_info(&d);
    if (st) return st;
    return cuda_status(launch_cluster_params(ch_max, ch_min, C, labels, g, bits, scale, zero, d.err,
                                             (cudaStream_t)stream));
}

int rptq_ln_reorder_quant(const void *x, int dtype, int64_t T, int C, const float *gamma,
                          const float *beta, float eps, const int32_t *R,
                          const int32_t *col_cluster, const float *scale, const int32_t *zero,
                          int g, int bits, uint8_t *codes, void *ln_out, rptq_stream_t stream)
{
    if (!dtype_ok(dtype)) return RPTQ_ERR_UNSUPPORTED;
    if (bits != 3 && bits != 4) return RPTQ_ERR_UNSUPPORTED;
    if (C <= 0 || C % 8 != 0 || C > RPTQ_MAX_CHANNELS) return RPTQ_ERR_UNSUPPORTED;
    if (T < 0 || g <= 0 || g > C || !(eps >= 0.0f)) return RPTQ_ERR_INVALID_ARG;
    if (!gamma || !beta || !R || !col_cluster || !scale || !zero) return RPTQ_ERR_INVALID_ARG;
    if (T == 0) return RPTQ_OK;  // no rows: nothing to launch, outputs may be empty (NULL)
    if (!codes && !ln_out) return RPTQ_ERR_INVALID_ARG;
    if (!x || !aligned16(x)) return RPTQ_ERR_INVALID_ARG;
    if (codes && !aligned16(codes)) return RPTQ_ERR_INVALID_ARG;
    if (ln_out && !aligned16(ln_out)) return RPTQ_ERR_INVALID_ARG;
    DevInfo d;
    int st = dev_info(&d);
    if (st) return st;
    if ((size_t)C * 5 > (size_t)d.max_smem) return RPTQ_ERR_UNSUPPORTED;
    LnQuantArgs a{x, dtype, T, C, gamma, beta, eps, R, col_cluster, scale, zero, g, bits, codes,
                  ln_out, d.err, (cudaStream_t)stream, d.num_sms, d.max_smem};
    return cuda_status(launch_ln_quant(a, 0));
}

size_t rptq_ln_quant_plan_bytes(int C) { return C > 0 ? (size_t)C * 12 : 0; }

int rptq_ln_quant_plan(const float *gamma, const float *beta, const int32_t *R, const int32_t *col_cluster,
                       const float *scale, const int32_t *zero, int C, int g, int bits, void *plan,
                       rptq_stream_t stream)
{
    if (bits != 3 && bits != 4) return RPTQ_ERR_UNSUPPORTED;
    if (C <= 0 || C % 8 != 0 || C > RPTQ_MAX_CHANNELS) return RPTQ_ERR_UNSUPPORTED;
    if (g <= 0 || g > C) return RPTQ_ERR_INVALID_ARG;
    if (!gamma || !beta || !R || !col_cluster || !scale || !zero || !plan || !aligned16(plan))
        return RPTQ_ERR_INVALID_ARG;
    DevInfo d;
    int st = dev_info(&d);
    if (st) return st;
    return cuda_status(launch_ln_quant_plan(gamma, beta, R, col_cluster, scale, zero, C, g, bits, plan, d.err,
                                            (cudaStream_t)stream));
}

int rptq_ln_reorder_quant_planned(const void *x, int dtype, int64_t T, int C, float eps, const void *plan,
                                  int bits, uint8_t *codes, rptq_stream_t stream)
{
    if (!dtype_ok(dtype)) return RPTQ_ERR_UNSUPPORTED;
    if (bits != 3 && bits != 4) return RPTQ_ERR_UNSUPPORTED;
    if (C <= 0 || C % 8 != 0 || C > RPTQ_MAX_CHANNELS) return RPTQ_ERR_UNSUPPORTED;
    if (T < 0 || !(eps >= 0.0f) || !plan || !aligned16(plan)) return RPTQ_ERR_INVALID_ARG;
    if (C % 32 != 0) return RPTQ_ERR_UNSUPPORTED;  // no direct kernel, so no planned launch
    if (T == 0) return RPTQ_OK;
    if (!x || !codes || !aligned16(x) || !aligned16(codes)) return RPTQ_ERR_INVALID_ARG;
    DevInfo d;
    int st = dev_info(&d);
    if (st) return st;
    if (!ln_quant_plan_supported(C, esize(dtype), d.max_smem)) return RPTQ_ERR_UNSUPPORTED;
    LnQuantArgs a{x, dtype, T, C, nullptr, nullptr, eps, nullptr, nullptr, nullptr, nullptr, 0, bits, codes,
                  nullptr, d.err, (cudaStream_t)stream, d.num_sms, d.max_smem, plan};
    return cuda_status(launch_ln_quant(a, 0));
}

int rptq_kv_quant(const void *k, const void *v, int dtype, int B, int H, int64_t S, int D,
                  const int32_t *cluster_k, const float *scale_k, const int32_t *zero_k,
                  const int32_t *cluster_v, const float *scale_v, const int32_t *zero_v, int g,
                  int bits, uint8_t *k_codes, uint8_t *v_codes, rptq_stream_t stream)
{
    if (!dtype_ok(dtype)) return RPTQ_ERR_UNSUPPORTED;
    if (bits != 3 && bits != 4) return RPTQ_ERR_UNSUPPORTED;
    if (D <= 0 || D % 8 != 0 || D > 2048 || H <= 0 || (int64_t)H * D > RPTQ_MAX_CHANNELS)
        return RPTQ_ERR_UNSUPPORTED;
    if (B < 0 || S < 0 || g <= 0) return RPTQ_ERR_INVALID_ARG;
    if (B == 0 || S == 0) return RPTQ_OK;  // an empty cache: nothing to launch, no pointer read
    if (!k && !v) return RPTQ_ERR_INVALID_ARG;
    if (k && (!cluster_k || !scale_k || !zero_k || !k_codes || !aligned16(k_codes) || !aligned16(k)))
        return RPTQ_ERR_INVALID_ARG;
    if (v && (!cluster_v || !scale_v || !zero_v || !v_codes || !aligned16(v_codes) || !aligned16(v)))
        return RPTQ_ERR_INVALID_ARG;
    if ((int64_t)B * H > 0x7fffffffLL) return RPTQ_ERR_UNSUPPORTED;
    DevInfo d;
    int st = dev_info(&d);
    if (st) return st;
    KvArgs a{k, v, dtype, B, H, S, D, cluster_k, scale_k, zero_k, cluster_v, scale_v, zero_v, g,
             bits, k_codes, v_codes, d.err, (cudaStream_t)stream, d.num_sms};
    return cuda_status(launch_kv_quant(a));
}

int rptq_kv_append(const void *k_new, const void *v_new, int dtype, int B, int H, int64_t s_len, int D,
                   int64_t S_max, int64_t s_begin, const int32_t *cluster_k, const float *scale_k,
                   const int32_t *zero_k, const int32_t *cluster_v, const float *scale_v,
                   const int32_t *zero_v, int g, int bits, uint8_t *k_cache, uint8_t *v_cache,
                   rptq_stream_t stream)
{
    if (!dtype_ok(dtype)) return RPTQ_ERR_UNSUPPORTED;
    if (bits != 3 && bits != 4) return RPTQ_ERR_UNSUPPORTED;
    if (D <= 0 || D % 8 != 0 || D > 2048 || H <= 0 || (int64_t)H * D > RPTQ_MAX_CHANNELS)
        return RPTQ_ERR_UNSUPPORTED;
    if (B < 0 || s_len < 0 || S_max < 0 || s_begin < 0 || g <= 0) return RPTQ_ERR_INVALID_ARG;
    if (s_begin + s_len > S_max) return RPTQ_ERR_INVALID_ARG;  // past the end of the cache
    if (B == 0 || s_len == 0) return RPTQ_OK;  // nothing to append: no pointer is read
    if (!k_new && !v_new) return RPTQ_ERR_INVALID_ARG;
    if (k_new && (!cluster_k || !scale_k || !zero_k || !k_cache || !aligned16(k_new) || !aligned16(k_cache)))
        return RPTQ_ERR_INVALID_ARG;
    if (v_new && (!cluster_v || !scale_v || !zero_v || !v_cache || !aligned16(v_new) || !aligned16(v_cache)))
        return RPTQ_ERR_INVALID_ARG;
    if ((int64_t)B * H > 0x7fffffffLL) return RPTQ_ERR_UNSUPPORTED;
    DevInfo d;
    int st = dev_info(&d);
    if (st) return st;
    KvAppendArgs a{k_new, v_new, dtype, B, H, s_len, D, S_max, s_begin, cluster_k, scale_k, zero_k,
                   cluster_v, scale_v, zero_v, g, bits, k_cache, v_cache, d.err, (cudaStream_t)stream,
                   d.num_sms};
    return cuda_status(launch_kv_append(a));
}

int rptq_kv_quant_cluster_ordered(const void *kv, int dtype, int B, int H, int64_t S, int D, const int32_t *R,
                                  const int32_t *col_cluster, const float *scale, const int32_t *zero, int g,
                                  int bits, uint8_t *codes, rptq_stream_t stream)
{
    if (bits != 3 && bits != 4) return RPTQ_ERR_UNSUPPORTED;
    if (dtype != RPTQ_F32 && dtype != RPTQ_F16 && dtype != RPTQ_BF16) return RPTQ_ERR_UNSUPPORTED;
    if (B < 0 || H <= 0 || S < 0 || D <= 0 || g <= 0 || g > RPTQ_MAX_CLUSTERS) return RPTQ_ERR_INVALID_ARG;
    const int64_t C = (int64_t)H * D;
    if (D % 8 != 0 || C % 32 != 0 || C > RPTQ_MAX_CHANNELS) return RPTQ_ERR_UNSUPPORTED;
    if (B == 0 || S == 0) return RPTQ_OK;
    if (!kv || !R || !col_cluster || !scale || !zero || !codes) return RPTQ_ERR_INVALID_ARG;
    if (!aligned16(kv) || !aligned16(codes)) return RPTQ_ERR_INVALID_ARG;
    if ((int64_t)B * ((S + 3) / 4) > ((int64_t)1 << 40)) return RPTQ_ERR_UNSUPPORTED;
    DevInfo d;
    int st = dev_info(&d);
    if (st) return st;
    if (!kv_quant_reordered_supported(H, D, g, d.max_smem)) return RPTQ_ERR_UNSUPPORTED;
    KvReorderedArgs a{kv, dtype, B, H, S, D, R, col_cluster, scale, zero, g, bits, codes, d.err,
                      (cudaStream_t)stream, d.num_sms};
    return cuda_status(launch_kv_quant_reordered(a));
}

int rptq_kv_decode_attention(const float *q, int B, int H, int D, const uint8_t *k_cache,
                             const uint8_t *v_cache, int64_t S_max, int64_t L,
                             const int32_t *cluster_k, const float *scale_k, const int32_t *zero_k,
                             const int32_t *cluster_v, const float *scale_v, const int32_t *zero_v,
                             int g, int bits, float scale, float *out, rptq_stream_t stream)
{
    if (bits != 3 && bits != 4) return RPTQ_ERR_UNSUPPORTED;
    if (D < 8 || D > 256 || (D & (D - 1)) != 0 || H <= 0 || (int64_t)H * D > RPTQ_MAX_CHANNELS)
        return RPTQ_ERR_UNSUPPORTED;
    if (L > KV_ATTN_MAX_L) return RPTQ_ERR_UNSUPPORTED;
    if (B < 0 || L < 1 || L > S_max || g <= 0 || !(scale >= 0.0f) || !(scale < INFINITY))
        return RPTQ_ERR_INVALID_ARG;
    if (B == 0) return RPTQ_OK;
    if (!q || !k_cache || !v_cache || !out || !cluster_k || !scale_k || !zero_k || !cluster_v ||
        !scale_v || !zero_v)
        return RPTQ_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(q) || !aligned16(out))
        return RPTQ_ERR_INVALID_ARG;
    if ((int64_t)B * H > 0x7fffffffLL) return RPTQ_ERR_UNSUPPORTED;
    DevInfo d;
    int st = dev_info(&d);
    if (st) return st;
    KvAttnArgs a{q, B, H, D, k_cache, v_cache, S_max, L, cluster_k, scale_k, zero_k, cluster_v,
                 scale_v, zero_v, g, bits, scale, out, d.err, (cudaStream_t)stream, d.max_smem};
    return cuda_status(launch_kv_attention(a));
}

int rptq_baseline_explicit_reorder_quant(const void *x, int dtype, int64_t T, int C,
                                         const float *gamma, const float *beta, float eps,
                                         const int32_t *R, const int32_t *col_cluster,
                                         const float *scale, const int32_t *zero, int g, int bits,
                                         float *y, float *y_reordered, uint8_t *codes,
                                         rptq_stream_t stream)
{
    if (!dtype_ok(dtype)) return RPTQ_ERR_UNSUPPORTED;
    if (bits != 3 && bits != 4) return RPTQ_ERR_UNSUPPORTED;
    if (C <= 0 || C % 8 != 0 || C > RPTQ_MAX_CHANNELS) return RPTQ_ERR_UNSUPPORTED;
    if (T < 0 || g <= 0 || g > C || !(eps >= 0.0f)) return RPTQ_ERR_INVALID_ARG;
    if (!gamma || !beta || !R || !col_cluster || !scale || !zero) return RPTQ_ERR_INVALID_ARG;
    if (T == 0) return RPTQ_OK;
    if (!x || !y || !y_reordered || !codes) return RPTQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y) || !aligned16(y_reordered) || !aligned16(codes) || !aligned16(R) ||
        !aligned16(col_cluster) || !aligned16(gamma) || !aligned16(beta))
        return RPTQ_ERR_INVALID_ARG;
    DevInfo d;
    int st = dev_info(&d);
    if (st) return st;
    if ((size_t)C * 8 > (size_t)d.max_smem) return RPTQ_ERR_UNSUPPORTED;
    XrArgs a{x, dtype, T, C, gamma, beta, eps, R, col_cluster, scale, zero, g, bits, y, y_reordered,
             codes, d.err, (cudaStream_t)stream, d.num_sms};
    return cuda_status(launch_explicit_reorder(a));
}

int rptq_linear_prepare(const uint8_t *w_codes, const int32_t *w_zero, int N, int C,
                        const int32_t *R, const int32_t *col_cluster, const float *scale,
                        const int32_t *zero, int g, void *w_prep, float *w_bias, float *w_lambda,
                        rptq_stream_t stream)
{
    if (C < 64 || C % 64 != 0 || C > RPTQ_MAX_CHANNELS) return RPTQ_ERR_UNSUPPORTED;
    if (N < 1 || g < 1 || g > C) return RPTQ_ERR_INVALID_ARG;
    if (!w_codes || !w_zero || !R || !col_cluster || !scale || !zero || !w_prep || !w_bias ||
        !w_lambda)
        return RPTQ_ERR_INVALID_ARG;
    if (!aligned16(w_prep) || !aligned16(w_codes)) return RPTQ_ERR_INVALID_ARG;
    DevInfo d;
    int st = dev_info(&d);
    if (st) return st;
    if ((size_t)C * 4 + (size_t)g * 12 + (size_t)4 * (C / 2 + 16) + 16 > (size_t)d.max_smem) return RPTQ_ERR_UNSUPPORTED;
    LinPrepArgs a{w_codes, w_zero, R, col_cluster, scale, zero, g, C, N,
                  static_cast<__half *>(w_prep), w_bias, w_lambda, d.err, (cudaStream_t)stream, d.num_sms};
    return cuda_status(launch_linear_prepare(a));
}

int rptq_reordered_linear(const uint8_t *codes, int64_t T, int C, int bits, const void *w_prep,
                          const float *w_bias, const float *w_lambda, const float *w_scale, int N,
                          float *out, rptq_stream_t stream)
{
    if (bits != 3 && bits != 4) return RPTQ_ERR_UNSUPPORTED;
    if (C < 64 || C % 64 != 0 || C > RPTQ_MAX_CHANNELS) return RPTQ_ERR_UNSUPPORTED;
    if (T < 0 || N < 1 || N > 65535 * 256) return RPTQ_ERR_INVALID_ARG;  // output tiles of 256 columns
    if (!w_prep || !w_bias || !w_lambda || !w_scale || !aligned16(w_prep)) return RPTQ_ERR_INVALID_ARG;
    if (T == 0) return RPTQ_OK;
    if (!codes || !out || !aligned16(codes) || !aligned16(out)) return RPTQ_ERR_INVALID_ARG;
    if ((T + 127) / 128 > 0x7fffffffLL) return RPTQ_ERR_UNSUPPORTED;
    DevInfo d;
    int st = dev_info(&d);
    if (st) return st;
    LinArgs a{codes, T, C, bits, static_cast<const __half *>(w_prep), w_bias, w_lambda, w_scale, N, out,
              d.err, (cudaStream_t)stream};
    return cuda_status(launch_reordered_linear(a));
}

int rptq_dequant(const uint8_t *codes, int layout, int64_t n0, int n1, int64_t S, int D,
                 const int32_t *cluster, const float *scale, const int32_t *zero, int g,
                 int bits, void *out, int out_dtype, rptq_stream_t stream)
{
    if (!dtype_ok(out_dtype)) return RPTQ_ERR_UNSUPPORTED;
    if (bits != 3 && bits != 4) return RPTQ_ERR_UNSUPPORTED;
    if (layout != RPTQ_LAYOUT_ROWS && layout != RPTQ_LAYOUT_BHSD) return RPTQ_ERR_INVALID_ARG;
    if (n0 < 0 || n1 <= 0 || g <= 0) return RPTQ_ERR_INVALID_ARG;
    if (!cluster || !scale || !zero) return RPTQ_ERR_INVALID_ARG;
    // no rows (or no positions): nothing to launch, codes / out may be empty (NULL)
    const bool work = n0 > 0 && (layout == RPTQ_LAYOUT_ROWS || S > 0);
    if (work && (!codes || !out || !aligned16(codes) || !aligned16(out)))
        return RPTQ_ERR_INVALID_ARG;
    if (layout == RPTQ_LAYOUT_ROWS) {
        if (n1 % 8 != 0 || n1 > RPTQ_MAX_CHANNELS) return RPTQ_ERR_UNSUPPORTED;
    } else {
        if (D <= 0 || D % 8 != 0 || D > 2048 || (int64_t)n1 * D > RPTQ_MAX_CHANNELS)
            return RPTQ_ERR_UNSUPPORTED;
        if (S < 0 || S > 0x7fffffffLL || n0 * n1 > 0x7fffffffLL) return RPTQ_ERR_INVALID_ARG;
    }
    if (!work) return RPTQ_OK;
    DevInfo d;
    int st = dev_info(&d);
    if (st) return st;
    DequantArgs a{codes, layout, n0, n1, S, D, cluster, scale, zero, g, bits, out, out_dtype,
                  d.err, (cudaStream_t)stream, d.num_sms};
    return cuda_status(launch_dequant(a));
}

}  // extern "C"
