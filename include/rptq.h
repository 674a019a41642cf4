/*
 * rptq.h -- C ABI of librptq.so: the RPTQ data path on NVIDIA B200 (sm_100a).
 *
 * RPTQ (reorder-based post-training quantization) quantizes LLM activations per cluster of
 * channels.  Sources, cited by page title and the part of the page:
 *  [RPTQ-art]  "基于重排序的新量化方法RPTQ：实现大型语言模型的 3 比特量化":
 *              Fig. 1 caption (one (max, min) point per activation channel); the text after
 *              Fig. 2 (calibrate per-channel max/min, KMeans into g clusters, reorder so that a
 *              cluster's channels are adjacent, one scale s and zero point z per cluster); the
 *              text after Fig. 3 (LayerNorm changed to emit the reordered activations, so no
 *              explicit reorder runs); the results paragraph (K/V cache quantized alone:
 *              W4A4KV, W4A3KV, W3A3KV) and the closing memory paragraph.
 *  [Houmo-art] RPTQ / PB-LLM article, section "RPTQ：量化激活通道的新思路" (3-bit activations;
 *              reorder removed by operator fusion).
 *  [Basics]    quantization-basics article (gitcode.csdn.net), section 一 (scale = float
 *              range / integer range), 1.1 (static ranges, outliers clamped), 1.3 (zero point,
 *              dequantization S(Wq - Z)), 1.4 (granularity).
 *
 * Conventions for every entry point
 *  - Tensor arguments are DEVICE pointers on the current CUDA device, owned by the caller,
 *    never freed or retained by the library.  Tensors are dense, row-major, and their base
 *    addresses must be 16-byte aligned (what cudaMalloc and torch allocations give).
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream) and is
 *    asynchronous: outputs are valid once the stream has been synchronised.
 *  - Arguments are validated on the host before anything is launched; an invalid call
 *    returns a negative status and launches nothing.  No C++ exception crosses the ABI.
 *  - Kernels never trap.  Conditions only the device can see (a cluster id outside [0, g), an
 *    R entry outside [0, C), a bounded wait that ran out) set a sticky device error word and
 *    the kernel carries on with safe values; read and clear it with rptq_device_error().
 *  - Calls that touch the same output buffers must not overlap on the GPU.
 *  - Per-device facts are looked up at a device's first call and kept for the process: the SM
 *    count, the shared-memory limit, the error word's address, each kernel's raised
 *    shared-memory limit and its occupancy.  A process that resets a device (cudaDeviceReset)
 *    must not call the library on that device afterwards.
 *  - Empty problems (no rows, no positions) are valid: nothing is launched (see each call).
 *
 * Notation: T tokens, C channels, g clusters, b = bits (3 or 4), qmax = 2^b - 1.
 *
 * Packed code layout (the pages only name 3- and 4-bit codes; this is the library's layout):
 *   a row of C codes takes C*b/8 bytes (C must be a multiple of 8);
 *   b = 4: code 2i -> low nibble of byte i, code 2i+1 -> high nibble;
 *   b = 3: codes 8m..8m+7 -> bytes 3m..3m+2; code 8m+k at bits [3k, 3k+3) of the
 *          little-endian 24-bit word byte0 | byte1 << 8 | byte2 << 16.
 */
#ifndef RPTQ_H_
#define RPTQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared here so that this header needs no CUDA header. */
typedef struct CUstream_st *rptq_stream_t;

/* Status codes. */
#define RPTQ_OK 0
#define RPTQ_ERR_INVALID_ARG (-1) /* null / misaligned pointer, bad size or range */
#define RPTQ_ERR_UNSUPPORTED (-2) /* bits not 3/4, C not a multiple of 8, C too large, dtype */
#define RPTQ_ERR_WORKSPACE (-3)   /* workspace pointer null or smaller than required */
#define RPTQ_ERR_CUDA (-4)        /* a CUDA runtime call or a launch failed */
#define RPTQ_ERR_DEVICE (-5)      /* the device error word was set (see rptq_device_error) */

/* Element types. */
#define RPTQ_F32 0
#define RPTQ_F16 1
#define RPTQ_BF16 2

/* Code layouts for rptq_dequant. */
#define RPTQ_LAYOUT_ROWS 0 /* [rows, C], column j in cluster col_cluster[j] */
#define RPTQ_LAYOUT_BHSD 1 /* [B, H, S, D] packed along D, channel c = h*D + d */

/* Largest channel count C (and H*D) any entry point accepts. */
#define RPTQ_MAX_CHANNELS 16384
/* Largest cluster count g. */
#define RPTQ_MAX_CLUSTERS 512

/* Human-readable text of a status code (static storage, never NULL). */
const char *rptq_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int rptq_version(void);

/*
 * Device error word.  Waits for `stream` to finish, stores the sticky device error word of
 * the current device in *code (0 = none; otherwise a bit set of RPTQ_DEVERR_* values) and
 * clears it.  Returns RPTQ_OK, or RPTQ_ERR_CUDA if the synchronisation or copy failed.
 */
#define RPTQ_DEVERR_CLUSTER_ID 1 /* a cluster id was outside [0, g); cluster 0 was used */
#define RPTQ_DEVERR_REORDER 2    /* an R entry was outside [0, C) */
#define RPTQ_DEVERR_TIMEOUT 4    /* a bounded wait on an asynchronous copy ran out */
int rptq_device_error(rptq_stream_t stream, int *code);

/*
 * Calibration statistics: per-channel maximum and minimum over T tokens.
 * [RPTQ-art] text after Fig. 2 and Fig. 1 caption.  The statistic is taken on the tensor
 * that will be quantized: with gamma != NULL it is LayerNorm(x) (the activation path),
 * otherwise x itself (the K/V path).
 *   x        [T, C] of `dtype` (RPTQ_F32 / RPTQ_F16 / RPTQ_BF16).
 *   gamma, beta  fp32 [C] in the original channel order, or both NULL.
 *   eps      LayerNorm epsilon (added to the biased variance); ignored without gamma.
 *   ch_max, ch_min  fp32 [C] outputs.  accumulate = 0 overwrites them; accumulate = 1 folds
 *            this batch into the values already there (calibrate in chunks).
 * In raw mode (gamma == NULL) the results are exact (bit-identical to a CPU max/min).
 * LayerNorm mode computes the normalisation in fp32 (single-pass moments with an exact
 * two-pass fallback for rows whose mean is large against their spread).
 * T == 0 is valid (no work; with accumulate = 0 the outputs become -inf / +inf).
 */
int rptq_calib_minmax(const void *x, int dtype, int64_t T, int C, const float *gamma,
                      const float *beta, float eps, float *ch_max, float *ch_min,
                      int accumulate, rptq_stream_t stream);

/*
 * Calibration statistics of a K or V cache in its attention layout: kv is [B, H, S, D] of
 * `dtype`, channel c = h*D + d, and the max / min of every channel are taken over the B*S
 * tokens (exact, like raw-mode rptq_calib_minmax).  ch_max, ch_min: fp32 [H*D].
 * accumulate as in rptq_calib_minmax.  D must be a multiple of 8, D <= 2048, H*D <=
 * RPTQ_MAX_CHANNELS.  [RPTQ-art] results paragraph (K/V cache quantized per cluster) with the
 * calibration of the text after Fig. 2.
 */
int rptq_kv_calib_minmax(const void *kv, int dtype, int B, int H, int64_t S, int D, float *ch_max,
                         float *ch_min, int accumulate, rptq_stream_t stream);

/* Workspace bytes rptq_kmeans needs for C points and g clusters (0 for invalid sizes). */
size_t rptq_kmeans_workspace_size(int C, int g);

/*
 * KMeans on the C points (ch_max[c], ch_min[c]), then the reorder index and the per-cluster
 * quantization parameters.  [RPTQ-art] text after Fig. 2 (KMeans on the (max, min) points,
 * same-cluster channels placed together, per-cluster s and z); [Basics] sections 一, 1.3.
 * Fixed readings (deterministic, identical on every run):
 *   - points are (double)ch_max[c], (double)ch_min[c];
 *   - init: channels sorted by (max, min, index) ascending; centroid k = point at sorted
 *     position floor((2k+1) C / (2g));
 *   - `iters` rounds of (assign, update) then a final assign; assign = argmin of the fp64
 *     squared distance dx*dx + dy*dy (no fused multiply-add), ties to the lowest k;
 *     update = mean of the members; an empty cluster keeps its centroid.  The loop stops
 *     early once an assignment repeats the previous one (provably the same result);
 *   - R: stable counting sort of the channels by label (clusters in label order, channels
 *     ascending inside each cluster);
 *   - cluster range M_k = max of members' ch_max, m_k = min of members' ch_min;
 *     scale s_k = (M_k - m_k) / qmax and zero z_k = rint(-m_k / s_k), fp32 IEEE divides,
 *     round-half-to-even, z not clamped; M_k == m_k gives s_k = max(|m_k|, |M_k|) / qmax
 *     (1 / qmax if both are 0); an empty cluster gets s = 1, z = 0.
 * Inputs: 1 <= g <= min(C, RPTQ_MAX_CLUSTERS), 1 <= C <= RPTQ_MAX_CHANNELS, iters >= 0,
 * bits in {3, 4}, finite statistics.
 * Outputs (device): labels int32[C]; centroids fp64[g][2] as (max, min); R int32[C]
 * (R[j] = channel stored at column j); col_cluster int32[C] (= labels[R[j]], non-decreasing);
 * offsets int32[g+1] (first stored column of each cluster, offsets[g] = C); scale fp32[g];
 * zero int32[g].
 * workspace: device buffer of at least rptq_kmeans_workspace_size(C, g) bytes, owned by the
 * caller; its contents need no initialisation and are garbage afterwards.
 */
int rptq_kmeans(const float *ch_max, const float *ch_min, int C, int g, int iters, int bits,
                int32_t *labels, double *centroids, int32_t *R, int32_t *col_cluster,
                int32_t *offsets, float *scale, int32_t *zero, void *workspace,
                size_t workspace_bytes, rptq_stream_t stream);

/*
 * Allocation-free variant of rptq_kmeans (the pages have no counterpart: this is a library
 * convenience).  Same arguments, outputs and results as rptq_kmeans, without the workspace:
 * the scratch is a fixed 2 MiB array inside the library's device image, which every GPU that
 * loads the library holds until the process exits.  For callers that cannot allocate device
 * memory while running (a plugin whose host owns all GPU memory, a serving loop that forbids
 * cudaMalloc / cudaFree after start-up); the call itself allocates nothing.
 *   - (C, g) needing more than 2 MiB of scratch is refused with RPTQ_ERR_UNSUPPORTED (every
 *     C <= RPTQ_MAX_CHANNELS with g <= RPTQ_MAX_CLUSTERS fits, so this does not happen within
 *     the library's limits);
 *   - all calls on a device share the scratch: calls whose kernels may overlap on the GPU
 *     race and can give wrong results, so order them (one stream, or events);
 *   - the scratch keeps the last call's contents; each call re-initialises what it reads;
 *   - the first call on a device looks up the scratch's device address (and the device's
 *     properties) with that device current; make that first call before any stream capture.
 */
#define RPTQ_KMEANS_NOALLOC_SCRATCH_BYTES (2u << 20)
int rptq_kmeans_noalloc(const float *ch_max, const float *ch_min, int C, int g, int iters,
                        int bits, int32_t *labels, double *centroids, int32_t *R,
                        int32_t *col_cluster, int32_t *offsets, float *scale, int32_t *zero,
                        rptq_stream_t stream);

/*
 * Per-cluster scale and zero point for FIXED clusters from per-channel statistics: the parameter
 * step of rptq_kmeans alone.  With statistics of the batch being quantized (rptq_calib_minmax on
 * it) this gives dynamic per-batch cluster ranges ([Basics] 1.1: static ranges come from
 * calibration data, dynamic ones from the data at hand; [RPTQ-art] text after Fig. 2: one scale
 * and zero point per cluster of channels); the clusters, R and col_cluster stay those of the
 * offline calibration, and the codes follow with rptq_ln_reorder_quant.
 *   ch_max, ch_min  fp32 [C];  labels  int32 [C] (the cluster of each channel, rptq_kmeans's
 *   labels);  scale, zero  fp32 / int32 [g] outputs, computed exactly as rptq_kmeans does:
 *   M_k = max of members' ch_max, m_k = min of members' ch_min, s_k = (M_k - m_k) / qmax,
 *   z_k = rint(-m_k / s_k) (fp32 IEEE, half-to-even; M_k == m_k and empty clusters as there).
 * A label outside [0, g) is reported in the device error word and the channel is skipped.
 */
int rptq_cluster_params(const float *ch_max, const float *ch_min, int C, const int32_t *labels,
                        int g, int bits, float *scale, int32_t *zero, rptq_stream_t stream);

/*
 * Reorder-fused LayerNorm with per-cluster quantization: the runtime activation path.
 * [RPTQ-art] text after Fig. 3 (the LayerNorm itself emits channels in cluster order, so no
 * reordered copy of x is ever stored); text after Fig. 2 (per-cluster s, z); [Houmo-art]
 * (reorder fused away, 3-bit activations); [Basics] 1.1 (static range: out-of-range values
 * clamp), 1.3 (q = round(y / s) + z).
 * For every token t, with y = LayerNorm(x[t]) over the C channels in the ORIGINAL order
 * (mean, biased variance, eps, gamma, beta):
 *   stored column j holds channel R[j]; k = col_cluster[j];
 *   code[t][j] = clamp(rint(y[R[j]] / scale[k]) + zero[k], 0, qmax)  (half-to-even),
 *   ln_out[t][j] = y[R[j]] rounded to `dtype`.
 *   x            [T, C] of `dtype`.
 *   gamma, beta  fp32 [C], original channel order.
 *   R, col_cluster  int32 [C] from rptq_kmeans.  R must be a permutation of [0, C): entries
 *                outside [0, C) are reported and skipped; repeated entries are not detected.
 *   scale, zero  fp32 [g], int32 [g]; g is the length of these tables.
 *   codes        uint8 [T, C*bits/8] packed codes in stored order, or NULL.
 *   ln_out       [T, C] of `dtype`, stored order, or NULL.  At least one of codes / ln_out.
 * T == 0 is valid: nothing is launched and x, codes and ln_out may all be NULL.
 * Codes are computed in fp32 and may differ from an exact-arithmetic reference by one step
 * where y / scale lies within fp32 rounding of a half-integer.
 */
int rptq_ln_reorder_quant(const void *x, int dtype, int64_t T, int C, const float *gamma,
                          const float *beta, float eps, const int32_t *R,
                          const int32_t *col_cluster, const float *scale, const int32_t *zero,
                          int g, int bits, uint8_t *codes, void *ln_out, rptq_stream_t stream);

/*
 * The offline LayerNorm rewrite as data: [RPTQ-art] text after Fig. 3 (the LayerNorm is changed
 * once, offline, so that it emits the reordered, quantized activations) folded with the text
 * after Fig. 2 (one (s, z) per cluster).  For every channel c, with j its stored column
 * (R[j] = c) and k = col_cluster[j], the plan holds the code-buffer offset of j and the affine
 * coefficients A_c = gamma_c / (s_k qmax), B_c = beta_c / (s_k qmax) + z_k / qmax (fp64,
 * rounded to fp32 once) with which rptq_ln_reorder_quant computes the codes; with the plan the
 * fused kernel does not rebuild these tables in every CTA.
 *   plan  device buffer of rptq_ln_quant_plan_bytes(C) bytes, 16-byte aligned, written here
 *         (layout: uint32 offset[C], float A[C], float B[C]; to be read only by
 *         rptq_ln_reorder_quant_planned).
 * Arguments as in rptq_ln_reorder_quant.  An R entry outside [0, C) or a cluster id outside
 * [0, g) sets the device error word (the channel keeps offset 0, A = B = 0, resp. uses
 * cluster 0).
 */
size_t rptq_ln_quant_plan_bytes(int C);
int rptq_ln_quant_plan(const float *gamma, const float *beta, const int32_t *R,
                       const int32_t *col_cluster, const float *scale, const int32_t *zero, int C,
                       int g, int bits, void *plan, rptq_stream_t stream);

/*
 * rptq_ln_reorder_quant (codes only) from a plan: the same codes, bit for bit, as
 * rptq_ln_reorder_quant with the arguments the plan was made from.  `bits` must be the plan's.
 * Shapes: those for which rptq_ln_reorder_quant uses its direct kernel -- C a multiple of 32 with
 * a thread split of the row (every OPT hidden size 768 .. 12288 qualifies); others return
 * RPTQ_ERR_UNSUPPORTED.  T == 0 is valid: nothing is launched.
 */
int rptq_ln_reorder_quant_planned(const void *x, int dtype, int64_t T, int C, float eps,
                                  const void *plan, int bits, uint8_t *codes, rptq_stream_t stream);

/*
 * K/V cache quantization with per-cluster parameters ([RPTQ-art] results paragraph:
 * W4A4KV / W4A3KV / W3A3KV quantize the key and value caches alone).
 * k, v: [B, H, S, D] of `dtype` (either may be NULL, not both); channel c = h*D + d.
 * cluster_k / cluster_v: int32 [H*D] cluster id of each channel in its NATURAL order (the
 * `labels` output of rptq_kmeans run on that tensor's statistics); the cache layout is kept,
 * so no reorder applies.  scale_*, zero_*: fp32 / int32 [g].
 *   code = clamp(rint(x / s) + z, 0, qmax), packed along D:
 *   k_codes / v_codes uint8 [B, H, S, D*bits/8].
 * D must be a multiple of 8 and H*D <= RPTQ_MAX_CHANNELS.  B == 0 or S == 0 is valid: nothing
 * is launched and no pointer is read (any of them may be NULL).
 */
int rptq_kv_quant(const void *k, const void *v, int dtype, int B, int H, int64_t S, int D,
                  const int32_t *cluster_k, const float *scale_k, const int32_t *zero_k,
                  const int32_t *cluster_v, const float *scale_v, const int32_t *zero_v, int g,
                  int bits, uint8_t *k_codes, uint8_t *v_codes, rptq_stream_t stream);

/*
 * Decode-time K/V append: the new tokens of one step quantized into preallocated caches.
 * [RPTQ-art] results paragraph (K/V cache quantized per cluster: W4A4KV / W4A3KV / W3A3KV) and
 * closing memory paragraph (the cache dominates memory at large batch x sequence).
 *   k_new, v_new  [B, H, s_len, D] of `dtype` (either may be NULL, not both), channel c = h*D + d.
 *   k_cache, v_cache  uint8 [B, H, S_max, D*bits/8] packed caches (rptq_kv_quant's layout);
 *                positions s_begin .. s_begin + s_len - 1 of every (b, h) receive the codes of
 *                the new tokens, computed exactly as rptq_kv_quant computes them; every other
 *                byte is left as it is.
 *   cluster_*, scale_*, zero_*: as in rptq_kv_quant (the calibration of that tensor).
 * s_begin + s_len must not exceed S_max (RPTQ_ERR_INVALID_ARG).  D must be a multiple of 8,
 * H*D <= RPTQ_MAX_CHANNELS.  B == 0 or s_len == 0 is valid: nothing is launched and no pointer
 * is read.
 */
int rptq_kv_append(const void *k_new, const void *v_new, int dtype, int B, int H, int64_t s_len,
                   int D, int64_t S_max, int64_t s_begin, const int32_t *cluster_k,
                   const float *scale_k, const int32_t *zero_k, const int32_t *cluster_v,
                   const float *scale_v, const int32_t *zero_v, int g, int bits,
                   uint8_t *k_cache, uint8_t *v_cache, rptq_stream_t stream);

/*
 * The K or V cache stored in cluster order: the layout variant of the cache beside
 * rptq_kv_quant's kept [B, H, S, D] layout ([RPTQ-art] text after Fig. 2: the channels of one
 * cluster placed side by side, one s and z per cluster; results paragraph: the K/V cache
 * quantized per cluster).  For every token (b, s) the C = H*D channels (c = h*D + d) are
 * gathered through the reorder index and quantized per cluster:
 *   codes[b][s] = pack over j of clamp(rint(kv[b, h, s, d] / s_k) + z_k, 0, qmax),
 *                 c = R[j] = h*D + d, k = col_cluster[j],
 * the same codes as rptq_kv_quant channel for channel (the same quotient, rounding and clamp),
 * in the row layout of the activation codes, so rptq_dequant's rows layout reads them back with
 * col_cluster.
 *   kv     [B, H, S, D] of `dtype` (RPTQ_F32 / RPTQ_F16 / RPTQ_BF16), 16-byte aligned.
 *   R, col_cluster  int32 [C] (rptq_kmeans's outputs for this cache); scale fp32 [g], zero int32 [g].
 *   codes  uint8 [B, S, C*bits/8] output, 16-byte aligned.
 * D a multiple of 8, C a multiple of 32 and at most RPTQ_MAX_CHANNELS (RPTQ_ERR_UNSUPPORTED
 * otherwise); B == 0 or S == 0 is valid: nothing is launched.  An R entry outside [0, C) or a
 * cluster id outside [0, g) is reported in the device error word (the codes are then undefined,
 * every store stays inside `codes`).
 */
int rptq_kv_quant_cluster_ordered(const void *kv, int dtype, int B, int H, int64_t S, int D,
                                  const int32_t *R, const int32_t *col_cluster, const float *scale,
                                  const int32_t *zero, int g, int bits, uint8_t *codes,
                                  rptq_stream_t stream);

/*
 * One decode step of attention over the packed caches, dequantizing every code in registers
 * as it is read (value = s_k * (q - z_k) in fp32, the value rptq_dequant writes): the consumer
 * of the quantized K/V cache ([RPTQ-art] results and closing memory paragraphs).  For every
 * (b, h): score_s = scale * sum_d q[b,h,d] K[b,h,s,d] for s < L, p = softmax(score),
 * out[b,h,d] = sum_s p_s V[b,h,s,d].
 *   q    fp32 [B, H, D] (one query per (b, h)).   out  fp32 [B, H, D].
 *   k_cache, v_cache  uint8 [B, H, S_max, D*bits/8]; positions 0 .. L-1 are read.
 *   cluster_*, scale_*, zero_*: the caches' calibrations (channel c = h*D + d).
 *   scale  > 0, or 0 for 1 / sqrt(D).
 * D must be a power of two in [8, 256]; 1 <= L <= S_max and L <= 16384 (the scores of a (b, h)
 * stay in shared memory).  Arithmetic in fp32 (fma dot products, expf, the sums in a fixed
 * order).  B == 0 is valid: nothing is launched.
 */
int rptq_kv_decode_attention(const float *q, int B, int H, int D, const uint8_t *k_cache,
                             const uint8_t *v_cache, int64_t S_max, int64_t L,
                             const int32_t *cluster_k, const float *scale_k, const int32_t *zero_k,
                             const int32_t *cluster_v, const float *scale_v, const int32_t *zero_v,
                             int g, int bits, float scale, float *out, rptq_stream_t stream);

/*
 * Offline weight preparation for the linear layer that reads the reordered activations.
 * [RPTQ-art] Fig. 3 caption and the text after it: the weights of the layer after the reordered
 * LayerNorm are permuted offline by the same reorder index, so that the layer consumes the
 * activations in cluster order and computes the same output; [Basics] sections 1.3 / 1.4: the
 * weights are 4-bit codes with one (s_w, z_w) per output row.
 *   w_codes   uint8 [N, C/2]: 4-bit weight codes in the ORIGINAL channel order (the packed
 *             layout above, b = 4); w_zero int32 [N]: row n's zero point z_w (its scale s_w is
 *             applied by rptq_reordered_linear and is not needed here).
 *   R, col_cluster, scale, zero, g: the activation calibration (rptq_kmeans's outputs).
 *   w_prep    fp16 [N, C] (output): the prepared operand, in cluster order, with the folded
 *             activation scale: B[n][j] = RN16(RN32(s_k * (w[n][R[j]] - z_w[n])) / lambda[n]),
 *             k = col_cluster[j], its columns interleaved inside each group of 8 as the GEMM
 *             decodes them (stored column 8m + 2i holds j = 8m + i, 8m + 2i + 1 holds
 *             j = 8m + 4 + i, i < 4).
 *   w_bias    fp32 [N] (output): sum_j z_k B[n][j] (summed in fp64, rounded once).
 *   w_lambda  fp32 [N] (output): the power of two that puts max_j |B[n][j]| in [2^14, 2^15)
 *             (1 for an all-zero row).
 * C a multiple of 64 in [64, RPTQ_MAX_CHANNELS], N >= 1, 1 <= g <= C; w_codes and w_prep
 * 16-byte aligned.  An R entry outside [0, C) or a cluster id outside [0, g) sets the device
 * error word (entry 0 / cluster 0 is used instead).
 */
int rptq_linear_prepare(const uint8_t *w_codes, const int32_t *w_zero, int N, int C,
                        const int32_t *R, const int32_t *col_cluster, const float *scale,
                        const int32_t *zero, int g, void *w_prep, float *w_bias, float *w_lambda,
                        rptq_stream_t stream);

/*
 * The reordered low-bit linear layer (W4A4 / W4A3, [RPTQ-art] results paragraph) on the tensor
 * cores: for token t and output n,
 *   out[t][n] = sum_j s_k (q[t][j] - z_k) * s_w[n] (w[n][R[j]] - z_w[n])
 *             = s_w[n] lambda[n] (sum_j q[t][j] B[n][j] - w_bias[n]),
 * with q the packed cluster-ordered activation codes (rptq_ln_reorder_quant's output).
 *   codes     uint8 [T, C*bits/8], bits 3 or 4.
 *   w_prep, w_bias, w_lambda: rptq_linear_prepare's outputs for this calibration; w_scale the
 *             weights' per-row scales.
 *   out       fp32 [T, N].
 * The codes go to the tensor core as exact fp16 integers and the products are accumulated in
 * fp32 (tcgen05.mma kind::f16, 128 x 256 output tiles).  C a multiple of 64 in
 * [64, RPTQ_MAX_CHANNELS], N in [1, 65535 * 256].  T == 0 is valid: nothing is launched.  A bounded
 * wait that runs out sets RPTQ_DEVERR_TIMEOUT (the output is then undefined).
 */
int rptq_reordered_linear(const uint8_t *codes, int64_t T, int C, int bits, const void *w_prep,
                          const float *w_bias, const float *w_lambda, const float *w_scale, int N,
                          float *out, rptq_stream_t stream);

/*
 * Dequantization, [Basics] section 1.3: value = s_k * (q - z_k), computed in fp32 (one
 * rounding) and rounded to out_dtype.
 *   layout RPTQ_LAYOUT_ROWS: codes [n0, n1*bits/8] with n0 = rows, n1 = C; cluster[j] is the
 *          cluster of column j (col_cluster from rptq_kmeans); S and D are ignored.
 *   layout RPTQ_LAYOUT_BHSD: codes [n0, n1, S, D*bits/8] with n0 = B, n1 = H; cluster[c] is
 *          the cluster of channel c = h*D + d.
 *   out: same shape with unpacked values of out_dtype.
 * n0 == 0 (or S == 0 for BHSD) is valid: nothing is launched and codes / out may be NULL.
 */
int rptq_dequant(const uint8_t *codes, int layout, int64_t n0, int n1, int64_t S, int D,
                 const int32_t *cluster, const float *scale, const int32_t *zero, int g,
                 int bits, void *out, int out_dtype, rptq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* RPTQ_H_ */
