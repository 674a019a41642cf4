// launch.h -- argument bundles and host launchers shared by api.cu and the kernel files.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace rptq {

// Launch settings remembered per kernel and device (api.cu): the kernel's dynamic shared-memory
// limit is raised once to the largest size asked for, and each (threads, bytes) occupancy
// answer is looked up once, so a repeated launch makes no driver query.
cudaError_t kernel_smem(const void *func, size_t bytes);
cudaError_t kernel_occupancy(int *per_sm, const void *func, int threads, size_t smem);

struct LnQuantArgs {
    const void *x;
    int dtype;
    int64_t T;
    int C;
    const float *gamma, *beta;
    float eps;
    const int32_t *R, *col_cluster;
    const float *scale;
    const int32_t *zero;
    int g, bits;
    uint8_t *codes;
    void *ln_out;
    int *err;
    cudaStream_t stream;
    int num_sms;
    int max_smem;
    const void *plan;  // rptq_ln_quant_plan's output, or NULL (tables built from R, s, z, gamma, beta)
};

struct CalibArgs {
    const void *x;
    int dtype;
    int64_t T;
    int C;
    const float *gamma, *beta;
    float eps;
    float *ch_max, *ch_min;
    int accumulate;
    int *err;
    cudaStream_t stream;
    int num_sms;
    int max_smem;
};

struct KvCalibArgs {
    const void *x;
    int dtype, B, H;
    int64_t S;
    int D;
    float *ch_max, *ch_min;
    int accumulate;
    int *err;
    cudaStream_t stream;
    int num_sms;
};

struct KvArgs {
    const void *k, *v;
    int dtype, B, H;
    int64_t S;
    int D;
    const int32_t *ck;
    const float *sk;
    const int32_t *zk;
    const int32_t *cv;
    const float *sv;
    const int32_t *zv;
    int g, bits;
    uint8_t *kq, *vq;
    int *err;
    cudaStream_t stream;
    int num_sms;
};

struct KvAppendArgs {
    const void *k, *v;
    int dtype, B, H;
    int64_t s_len;
    int D;
    int64_t S_max, s_begin;
    const int32_t *ck;
    const float *sk;
    const int32_t *zk;
    const int32_t *cv;
    const float *sv;
    const int32_t *zv;
    int g, bits;
    uint8_t *kq, *vq;
    int *err;
    cudaStream_t stream;
    int num_sms;
};

// rptq_kv_quant_cluster_ordered: K or V [B, H, S, D] -> codes [B, S, C*bits/8] in cluster order
struct KvReorderedArgs {
    const void *kv;
    int dtype, B, H;
    int64_t S;
    int D;
    const int32_t *R, *col_cluster;
    const float *scale;
    const int32_t *zero;
    int g, bits;
    uint8_t *codes;
    int *err;
    cudaStream_t stream;
    int num_sms;
};

struct KvAttnArgs {
    const float *q;
    int B, H, D;
    const uint8_t *kq, *vq;
    int64_t S_max, L;
    const int32_t *ck;
    const float *sk;
    const int32_t *zk;
    const int32_t *cv;
    const float *sv;
    const int32_t *zv;
    int g, bits;
    float scale;
    float *out;
    int *err;
    cudaStream_t stream;
    int max_smem;
};

struct XrArgs {
    const void *x;
    int dtype;
    int64_t T;
    int C;
    const float *gamma, *beta;
    float eps;
    const int32_t *R, *col_cluster;
    const float *scale;
    const int32_t *zero;
    int g, bits;
    float *y, *yr;
    uint8_t *codes;
    int *err;
    cudaStream_t stream;
    int num_sms;
};

struct LinPrepArgs {
    const uint8_t *qw;  // [N, C/2] 4-bit weight codes, original channel order, low nibble first
    const int32_t *zw;
    const int32_t *R, *col_cluster;
    const float *scale;
    const int32_t *zero;
    int g, C, N;
    __half *B;  // [N, C] prepared fp16 weights
    float *bz, *lam;
    int *err;
    cudaStream_t stream;
    int num_sms;
};

struct LinArgs {
    const uint8_t *codes;  // [T, C*bits/8]
    int64_t T;
    int C, bits;
    const __half *B;
    const float *bz, *lam, *sw;
    int N;
    float *Y;  // [T, N] fp32
    int *err;
    cudaStream_t stream;
};

struct DequantArgs {
    const uint8_t *codes;
    int layout;
    int64_t n0;
    int n1;
    int64_t S;
    int D;
    const int32_t *cluster;
    const float *scale;
    const int32_t *zero;
    int g, bits;
    void *out;
    int out_dtype;
    int *err;
    cudaStream_t stream;
    int num_sms;
};

struct KmArgs {
    const float *mx, *mn;
    int C, g, iters, bits;
    int32_t *labels;
    double *cent;
    int32_t *R, *col_cluster, *offsets;
    float *scale;
    int32_t *zero;
    void *ws;
    cudaStream_t stream;
    int num_sms;
    int max_smem;
    int *err;
};

// force_simple = 1 routes codes-only calls to the general kernel (used by tests of that path)
cudaError_t launch_ln_quant(const LnQuantArgs &a, int force_simple);
cudaError_t launch_ln_quant_plan(const float *gamma, const float *beta, const int32_t *R, const int32_t *col_cluster,
                                 const float *scale, const int32_t *zero, int C, int g, int bits, void *plan,
                                 int *err, cudaStream_t stream);
bool ln_quant_plan_supported(int C, int esize, int max_smem);
bool ln_quant_fast_plan(int C, int esize, int max_smem, bool allow_direct, int *CPT, int *NT, int *NS, int *alias);
cudaError_t launch_calib(const CalibArgs &a);
cudaError_t launch_kv_calib(const KvCalibArgs &a);
cudaError_t launch_kv_quant(const KvArgs &a);
cudaError_t launch_dequant(const DequantArgs &a);
cudaError_t launch_kv_append(const KvAppendArgs &a);
cudaError_t launch_cluster_params(const float *mx, const float *mn, int C, const int32_t *labels, int g, int bits,
                                  float *scale, int32_t *zero, int *err, cudaStream_t stream);
cudaError_t launch_explicit_reorder(const XrArgs &a);
cudaError_t launch_kv_attention(const KvAttnArgs &a);
cudaError_t launch_kv_quant_reordered(const KvReorderedArgs &a);
// (H, D, g) that the cluster-ordered K/V kernel takes, with its tables within max_smem
bool kv_quant_reordered_supported(int H, int D, int g, int max_smem);
cudaError_t launch_linear_prepare(const LinPrepArgs &a);
cudaError_t launch_reordered_linear(const LinArgs &a);
// largest number of cache positions one decode-attention call reads (its scores stay in shared
// memory)
constexpr int64_t KV_ATTN_MAX_L = 16384;
cudaError_t launch_kmeans(const KmArgs &a);
size_t kmeans_ws_bytes(int C, int g);
// (C, g) within the limits and the fused KMeans kernel's shared memory within max_smem
bool kmeans_supported(int C, int g, int max_smem);
// the sticky device error word of the current device (nullptr if it cannot be looked up)
int *device_error_word();

}  // namespace rptq
