/*
 * rptq_oracle.c -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.
 *
 * A plain, slow, single-threaded CPU statement of what the RPTQ data path computes.
 * Only the test suite, the smoke check and the bench's CPU-baseline / reference legs may
 * load it.  It shares no source, header, table or helper with the CUDA library, and it
 * never reads anything the CUDA library produced.  Floating point is IEEE fp64 unless a
 * step fixes fp32; build with `-O2 -ffp-contract=off` and without fast-math so that no
 * multiply-add is fused and every operation rounds exactly as written.
 *
 * Sources, cited by page title and the part of the page:
 *  [RPTQ-art]  "基于重排序的新量化方法RPTQ：实现大型语言模型的 3 比特量化" (m.zhengruan.com).
 *              Fig. 1 caption: one (max, min) point per activation channel.
 *              Text after Fig. 2: calibrate per-channel max/min, KMeans into g clusters on those
 *              points, place same-cluster channels next to each other, one scale s and zero
 *              point z per cluster.
 *              Text after Fig. 3: LayerNorm is changed to emit the reordered activations
 *              directly (no explicit reorder); results paragraph: K/V cache quantized alone
 *              (W4A4KV, W4A3KV, W3A3KV).
 *  [Houmo-art] RPTQ / PB-LLM article, section "RPTQ：量化激活通道的新思路": 3-bit activations,
 *              reorder avoided by operator fusion.
 *  [Basics]    Quantization-basics article (gitcode.csdn.net): section 一 "量化的概念"
 *              (uniform scale = float range / integer range), section 1.1 "dynamic和static"
 *              (static ranges profiled offline; outliers clamped to the profiled range),
 *              section 1.3 "symmetric和asymmetric" (zero point Z, dequantization S(Wq - Z)),
 *              section 1.4 "granularity" (per-tensor, per-channel).
 *
 * Where the pages leave a step open, the reading taken is stated beside the step.
 * Every function here is pinned by tests/test_oracle_*.py against closed forms, brute
 * force, library routines or hand-computed values.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------ */
/* 1. Calibration: per-channel max and min over the calibration tokens.                  */
/*    [RPTQ-art] text after Fig. 2; the points plotted in Fig. 1.                         */
/*    x is row-major [T x C] fp32 (fp16/bf16 inputs are widened exactly before the call). */
/*    accumulate = 0 starts from the first row, 1 folds into the values already in mx/mn. */
/* ------------------------------------------------------------------------------------ */
void orc_minmax(const float *x, int64_t T, int C, float *mx, float *mn, int accumulate)
{
    for (int c = 0; c < C; ++c) {
        float hi = accumulate ? mx[c] : -INFINITY;
        float lo = accumulate ? mn[c] : INFINITY;
        for (int64_t t = 0; t < T; ++t) {
            float v = x[t * (int64_t)C + c];
            if (v > hi) hi = v;
            if (v < lo) lo = v;
        }
        mx[c] = hi;
        mn[c] = lo;
    }
}

/* ------------------------------------------------------------------------------------ */
/* 2. LayerNorm of one row, fp64.  The pages give no formula (the Fig. 3 text only says  */
/*    LayerNorm is modified to emit reordered output).  Reading: the standard LayerNorm   */
/*    of OPT-style models: mean, biased variance (two passes), eps added to the variance, */
/*    per-channel affine gamma, beta in the ORIGINAL channel order.                       */
/* ------------------------------------------------------------------------------------ */
static void ln_row(const float *xr, int C, const float *gamma, const float *beta, double eps,
                   double *y)
{
    double sum = 0.0;
    for (int c = 0; c < C; ++c) sum += (double)xr[c];
    double mean = sum / (double)C;
    double ss = 0.0;
    for (int c = 0; c < C; ++c) {
        double d = (double)xr[c] - mean;
        ss += d * d;
    }
    double var = ss / (double)C;
    double denom = sqrt(var + eps);
    for (int c = 0; c < C; ++c) {
        double xhat = ((double)xr[c] - mean) / denom;
        y[c] = xhat * (double)gamma[c] + (double)beta[c];
    }
}

/* LayerNorm of a [T x C] matrix.  y64 (unrounded) and y32 (rounded to fp32) are optional. */
void orc_layernorm(const float *x, int64_t T, int C, const float *gamma, const float *beta,
                   double eps, double *y64, float *y32)
{
    double *y = (double *)malloc(sizeof(double) * (size_t)C);
    for (int64_t t = 0; t < T; ++t) {
        ln_row(x + t * (int64_t)C, C, gamma, beta, eps, y);
        for (int c = 0; c < C; ++c) {
            if (y64) y64[t * (int64_t)C + c] = y[c];
            if (y32) y32[t * (int64_t)C + c] = (float)y[c];
        }
    }
    free(y);
}

/* Calibration statistics of the LayerNorm output (the tensor the runtime path quantizes),
 * taken on the fp32-rounded LayerNorm values.  Same accumulate convention as orc_minmax. */
void orc_minmax_ln(const float *x, int64_t T, int C, const float *gamma, const float *beta,
                   double eps, float *mx, float *mn, int accumulate)
{
    double *y = (double *)malloc(sizeof(double) * (size_t)C);
    if (!accumulate) {
        for (int c = 0; c < C; ++c) {
            mx[c] = -INFINITY;
            mn[c] = INFINITY;
        }
    }
    for (int64_t t = 0; t < T; ++t) {
        ln_row(x + t * (int64_t)C, C, gamma, beta, eps, y);
        for (int c = 0; c < C; ++c) {
            float v = (float)y[c];
            if (v > mx[c]) mx[c] = v;
            if (v < mn[c]) mn[c] = v;
        }
    }
    free(y);
}

/* ------------------------------------------------------------------------------------ */
/* 3. KMeans on the 2-D points P_c = (max_c, min_c).  [RPTQ-art] text after Fig. 2 names  */
/*    KMeans, g and the points; everything else is a reading:                             */
/*    - init: sort channels by (max, then min, then index) ascending; centroid k is the   */
/*      point at sorted position floor((2k+1)*C / (2g))  (deterministic quantile init);   */
/*    - assign: squared Euclidean distance dx*dx + dy*dy in fp64 (no fused multiply-add); */
/*      ties go to the lowest cluster index;                                              */
/*    - update: centroid = mean of its members (members summed in ascending channel       */
/*      order); an empty cluster keeps its previous centroid;                             */
/*    - exactly `iters` rounds of (assign, update), then one final assign.                */
/* ------------------------------------------------------------------------------------ */
typedef struct {
    double mx, mn;
    int c;
} key_t_;

static int key_cmp(const void *a, const void *b)
{
    const key_t_ *p = (const key_t_ *)a, *q = (const key_t_ *)b;
    if (p->mx < q->mx) return -1;
    if (p->mx > q->mx) return 1;
    if (p->mn < q->mn) return -1;
    if (p->mn > q->mn) return 1;
    return (p->c > q->c) - (p->c < q->c);
}

/* Quantile initialisation alone (exposed so tests can pin it). */
int orc_kmeans_init(const float *mx, const float *mn, int C, int g, double *cent)
{
    if (g < 1 || g > C) return -1;
    key_t_ *keys = (key_t_ *)malloc(sizeof(key_t_) * (size_t)C);
    for (int c = 0; c < C; ++c) {
        keys[c].mx = (double)mx[c];
        keys[c].mn = (double)mn[c];
        keys[c].c = c;
    }
    qsort(keys, (size_t)C, sizeof(key_t_), key_cmp);
    for (int k = 0; k < g; ++k) {
        int64_t pos = ((int64_t)(2 * k + 1) * (int64_t)C) / (2 * (int64_t)g);
        cent[2 * k + 0] = keys[pos].mx;
        cent[2 * k + 1] = keys[pos].mn;
    }
    free(keys);
    return 0;
}

/* One assignment pass; returns the number of labels that changed. */
int orc_kmeans_assign(const float *mx, const float *mn, int C, int g, const double *cent,
                      int32_t *labels)
{
    int changed = 0;
    for (int c = 0; c < C; ++c) {
        double px = (double)mx[c], py = (double)mn[c];
        int best = 0;
        double bestd = 0.0;
        for (int k = 0; k < g; ++k) {
            double dx = px - cent[2 * k + 0];
            double dy = py - cent[2 * k + 1];
            double d = dx * dx + dy * dy;
            if (k == 0 || d < bestd) {
                bestd = d;
                best = k;
            }
        }
        if (labels[c] != best) ++changed;
        labels[c] = best;
    }
    return changed;
}

/* One update pass: mean of the members, summed in ascending channel order. */
void orc_kmeans_update(const float *mx, const float *mn, int C, int g, const int32_t *labels,
                       double *cent)
{
    for (int k = 0; k < g; ++k) {
        double sx = 0.0, sy = 0.0;
        int64_t n = 0;
        for (int c = 0; c < C; ++c) {
            if (labels[c] != k) continue;
            sx += (double)mx[c];
            sy += (double)mn[c];
            ++n;
        }
        if (n > 0) {
            cent[2 * k + 0] = sx / (double)n;
            cent[2 * k + 1] = sy / (double)n;
        }
    }
}

int orc_kmeans(const float *mx, const float *mn, int C, int g, int iters, int32_t *labels,
               double *cent)
{
    if (g < 1 || g > C || iters < 0) return -1;
    if (orc_kmeans_init(mx, mn, C, g, cent) != 0) return -1;
    for (int c = 0; c < C; ++c) labels[c] = -1;
    for (int it = 0; it < iters; ++it) {
        orc_kmeans_assign(mx, mn, C, g, cent, labels);
        orc_kmeans_update(mx, mn, C, g, labels, cent);
    }
    orc_kmeans_assign(mx, mn, C, g, cent, labels);
    return 0;
}

/* ------------------------------------------------------------------------------------ */
/* 4. Reorder index.  [RPTQ-art] text after Fig. 2 (same-cluster channels placed next to */
/*    each other) and Fig. 3 (reorder indices R1..R5).  Reading: clusters in label order,  */
/*    channels ascending inside a cluster (a stable counting sort).  R[j] = source channel */
/*    of stored column j; offsets[k] = first stored column of cluster k (offsets[g] = C);  */
/*    col_cluster[j] = label of R[j].                                                      */
/* ------------------------------------------------------------------------------------ */
void orc_reorder(const int32_t *labels, int C, int g, int32_t *R, int32_t *col_cluster,
                 int32_t *offsets)
{
    for (int k = 0; k <= g; ++k) offsets[k] = 0;
    for (int c = 0; c < C; ++c) offsets[labels[c] + 1] += 1;
    for (int k = 0; k < g; ++k) offsets[k + 1] += offsets[k];
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)(g > 0 ? g : 1));
    for (int k = 0; k < g; ++k) fill[k] = offsets[k];
    for (int c = 0; c < C; ++c) {
        int j = fill[labels[c]]++;
        R[j] = c;
        col_cluster[j] = labels[c];
    }
    free(fill);
}

/* ------------------------------------------------------------------------------------ */
/* 5. Per-cluster quantization parameters.  [RPTQ-art] text after Fig. 2 (one s and one  */
/*    z per cluster); [Basics] section 一 (scale = float range / integer range) and       */
/*    section 1.3 (zero point).  Readings:                                                */
/*    - cluster range: M = max of the members' max, m = min of the members' min;          */
/*    - s = (M - m) / qmax and z = rint(-m / s), both in fp32, round-half-to-even;        */
/*    - z is NOT clamped to [0, qmax] (stored as int32) and the range is NOT widened to   */
/*      contain 0;                                                                        */
/*    - degenerate cluster (M == m): s = max(|m|, |M|) / qmax, or 1 / qmax when that is 0; */
/*    - empty cluster: s = 1, z = 0 (never referenced).                                   */
/* ------------------------------------------------------------------------------------ */
void orc_cluster_params(const float *mx, const float *mn, const int32_t *labels, int C, int g,
                        int bits, float *s, int32_t *z)
{
    const float qmax = (float)((1 << bits) - 1);
    for (int k = 0; k < g; ++k) {
        int any = 0;
        float M = 0.0f, m = 0.0f;
        for (int c = 0; c < C; ++c) {
            if (labels[c] != k) continue;
            if (!any || mx[c] > M) M = mx[c];
            if (!any || mn[c] < m) m = mn[c];
            any = 1;
        }
        if (!any) {
            s[k] = 1.0f;
            z[k] = 0;
            continue;
        }
        float scale;
        if (M == m) {
            float r = fabsf(m) > fabsf(M) ? fabsf(m) : fabsf(M);
            if (r == 0.0f) r = 1.0f;
            scale = r / qmax;
        } else {
            float range = M - m;
            scale = range / qmax;
        }
        float ratio = -m / scale;
        s[k] = scale;
        z[k] = (int32_t)rintf(ratio);
    }
}

/* ------------------------------------------------------------------------------------ */
/* 6. Asymmetric uniform quantization of one value with its cluster's (s, z).             */
/*    [Basics] section 1.3: real value = S * (q - Z), so q = round(v / S) + Z; section    */
/*    1.1: a static range clips values outside it.  Reading: q = clamp(rint(v/s) + z, 0,  */
/*    qmax), fp32 divide, round-half-to-even, z added as an integer after rounding.       */
/* ------------------------------------------------------------------------------------ */
static int quant_one(float v, float s, int32_t z, int qmax)
{
    float t = v / s;
    /* rintf(t) is an integer-valued float; widening to double and adding z is exact for
       every finite t, and the clamp then cannot overflow an integer type. */
    double q = (double)rintf(t) + (double)z;
    if (q < 0.0) q = 0.0;
    if (q > (double)qmax) q = (double)qmax;
    return (int)q;
}

/* Unpacked codes of a [rows x C] matrix whose column j belongs to cluster col_cluster[j]. */
void orc_quantize(const float *y, int64_t rows, int C, const int32_t *col_cluster,
                  const float *s, const int32_t *z, int bits, uint8_t *q)
{
    const int qmax = (1 << bits) - 1;
    for (int64_t t = 0; t < rows; ++t)
        for (int j = 0; j < C; ++j) {
            int k = col_cluster[j];
            q[t * (int64_t)C + j] = (uint8_t)quant_one(y[t * (int64_t)C + j], s[k], z[k], qmax);
        }
}

/* ------------------------------------------------------------------------------------ */
/* 7. Packing (the pages only say 3- and 4-bit codes).  Reading, per row:                 */
/*    4 bits: code 2i in the low nibble of byte i, code 2i+1 in the high nibble;          */
/*    3 bits: each group of 8 codes fills 3 bytes; code k of the group sits at bits       */
/*    [3k, 3k+3) of the little-endian 24-bit word b0 | b1<<8 | b2<<16.                    */
/*    Row pitch = C*bits/8 bytes (C a multiple of 8).                                     */
/* ------------------------------------------------------------------------------------ */
void orc_pack(const uint8_t *q, int64_t rows, int C, int bits, uint8_t *out)
{
    const int64_t pitch = (int64_t)C * bits / 8;
    for (int64_t t = 0; t < rows; ++t) {
        const uint8_t *qr = q + t * (int64_t)C;
        uint8_t *o = out + t * pitch;
        if (bits == 4) {
            for (int i = 0; i < C / 2; ++i)
                o[i] = (uint8_t)((qr[2 * i] & 15) | ((qr[2 * i + 1] & 15) << 4));
        } else {
            for (int gidx = 0; gidx < C / 8; ++gidx) {
                uint32_t w = 0;
                for (int k = 0; k < 8; ++k) w |= (uint32_t)(qr[8 * gidx + k] & 7) << (3 * k);
                o[3 * gidx + 0] = (uint8_t)(w & 0xff);
                o[3 * gidx + 1] = (uint8_t)((w >> 8) & 0xff);
                o[3 * gidx + 2] = (uint8_t)((w >> 16) & 0xff);
            }
        }
    }
}

void orc_unpack(const uint8_t *packed, int64_t rows, int C, int bits, uint8_t *q)
{
    const int64_t pitch = (int64_t)C * bits / 8;
    for (int64_t t = 0; t < rows; ++t) {
        const uint8_t *p = packed + t * pitch;
        uint8_t *qr = q + t * (int64_t)C;
        if (bits == 4) {
            for (int i = 0; i < C / 2; ++i) {
                qr[2 * i] = p[i] & 15;
                qr[2 * i + 1] = (p[i] >> 4) & 15;
            }
        } else {
            for (int gidx = 0; gidx < C / 8; ++gidx) {
                uint32_t w = (uint32_t)p[3 * gidx] | ((uint32_t)p[3 * gidx + 1] << 8) |
                             ((uint32_t)p[3 * gidx + 2] << 16);
                for (int k = 0; k < 8; ++k) qr[8 * gidx + k] = (uint8_t)((w >> (3 * k)) & 7);
            }
        }
    }
}

/* ------------------------------------------------------------------------------------ */
/* 8. Dequantization, [Basics] section 1.3: value = s * (q - z), fp32 (one rounding).     */
/*    Row layout [rows x C] with per-column cluster ids.                                  */
/* ------------------------------------------------------------------------------------ */
void orc_dequant(const uint8_t *q, int64_t rows, int C, const int32_t *col_cluster,
                 const float *s, const int32_t *z, float *out)
{
    for (int64_t t = 0; t < rows; ++t)
        for (int j = 0; j < C; ++j) {
            int k = col_cluster[j];
            float diff = (float)((int32_t)q[t * (int64_t)C + j] - z[k]);
            out[t * (int64_t)C + j] = s[k] * diff;
        }
}

/* ------------------------------------------------------------------------------------ */
/* 9. The runtime activation path written UNFUSED, as its definition: LayerNorm in the    */
/*    original channel order, rounded to fp32, then an explicit gather through R          */
/*    (stored column j takes channel R[j]), then per-cluster quantization, then packing.  */
/*    [RPTQ-art] text after Fig. 3: the fused kernel must produce exactly this without    */
/*    ever materialising the reordered tensor.                                            */
/*    packed (rows * C*bits/8 bytes), ln32 and ln64 ([T x C], stored order) are optional. */
/* ------------------------------------------------------------------------------------ */
void orc_ln_reorder_quant(const float *x, int64_t T, int C, const float *gamma,
                          const float *beta, double eps, const int32_t *R,
                          const int32_t *col_cluster, const float *s, const int32_t *z, int bits,
                          uint8_t *packed, float *ln32, double *ln64)
{
    double *y = (double *)malloc(sizeof(double) * (size_t)C);
    float *g32 = (float *)malloc(sizeof(float) * (size_t)C);
    uint8_t *q = (uint8_t *)malloc((size_t)C);
    const int64_t pitch = (int64_t)C * bits / 8;
    for (int64_t t = 0; t < T; ++t) {
        ln_row(x + t * (int64_t)C, C, gamma, beta, eps, y);
        for (int j = 0; j < C; ++j) {
            g32[j] = (float)y[R[j]];
            if (ln32) ln32[t * (int64_t)C + j] = g32[j];
            if (ln64) ln64[t * (int64_t)C + j] = y[R[j]];
        }
        if (packed) {
            orc_quantize(g32, 1, C, col_cluster, s, z, bits, q);
            orc_pack(q, 1, C, bits, packed + t * pitch);
        }
    }
    free(y);
    free(g32);
    free(q);
}

/* ------------------------------------------------------------------------------------ */
/* 10. K/V cache quantization ([RPTQ-art] results paragraph: W4A4KV / W4A3KV / W3A3KV).   */
/*     Reading: K (or V) is [B, H, S, D]; its channel is c = h*D + d, clustered over the   */
/*     H*D channels with its own calibration; the layout stays [B, H, S, D] and codes are  */
/*     packed along D (row pitch D*bits/8 bytes per (b, h, s)).                           */
/* ------------------------------------------------------------------------------------ */
void orc_kv_quant(const float *kv, int64_t B, int H, int64_t S, int D, const int32_t *col_cluster,
                  const float *s, const int32_t *z, int bits, uint8_t *packed)
{
    const int qmax = (1 << bits) - 1;
    const int64_t pitch = (int64_t)D * bits / 8;
    uint8_t *q = (uint8_t *)malloc((size_t)D);
    for (int64_t b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int64_t t = 0; t < S; ++t) {
                int64_t row = (b * H + h) * S + t;
                const float *xr = kv + row * D;
                for (int d = 0; d < D; ++d) {
                    int k = col_cluster[h * D + d];
                    q[d] = (uint8_t)quant_one(xr[d], s[k], z[k], qmax);
                }
                orc_pack(q, 1, D, bits, packed + row * pitch);
            }
    free(q);
}

/* Dequantization of a packed [B, H, S, D] cache (channel c = h*D + d). */
void orc_kv_dequant(const uint8_t *packed, int64_t B, int H, int64_t S, int D,
                    const int32_t *col_cluster, const float *s, const int32_t *z, int bits,
                    float *out)
{
    const int64_t pitch = (int64_t)D * bits / 8;
    uint8_t *q = (uint8_t *)malloc((size_t)D);
    for (int64_t b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int64_t t = 0; t < S; ++t) {
                int64_t row = (b * H + h) * S + t;
                orc_unpack(packed + row * pitch, 1, D, bits, q);
                for (int d = 0; d < D; ++d) {
                    int k = col_cluster[h * D + d];
                    float diff = (float)((int32_t)q[d] - z[k]);
                    out[row * D + d] = s[k] * diff;
                }
            }
    free(q);
}
