/*
 * rptq_baseline.h -- baselines of librptq.so, kept for measurement, not for use: paths that the
 * RPTQ method exists to avoid, built with the same care as the product kernels so that what
 * the product saves can be measured on the same GPU.  Same conventions as rptq.h.
 */
#ifndef RPTQ_BASELINE_H_
#define RPTQ_BASELINE_H_

#include <stdint.h>

#include "rptq.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * The explicit reorder that RPTQ's fused LayerNorm removes ([RPTQ-art], the paragraph before
 * Fig. 3's text: reordering the channels at run time moves every channel and costs time and
 * memory; the text after Fig. 3: the LayerNorm itself emits cluster order instead).  Three
 * kernels with two materialised fp32 intermediates:
 *   y[t][c]  = LayerNorm(x[t])[c]          (original channel order)
 *   y_reordered[t][j] = y[t][R[j]]         (the explicit gather through R)
 *   codes[t] = clamp(rint(y_reordered[t][j] / scale[k]) + zero[k], 0, qmax), k = col_cluster[j]
 * Arguments as in rptq_ln_reorder_quant; y and y_reordered are caller-owned fp32 [T, C]
 * buffers (their contents are outputs too).  The codes are those of rptq_ln_reorder_quant's
 * definition.  All pointers 16-byte aligned, R and col_cluster included; 8*C bytes must fit in
 * one CTA's shared memory.  T == 0 is valid: nothing is launched.
 */
int rptq_baseline_explicit_reorder_quant(const void *x, int dtype, int64_t T, int C,
                                         const float *gamma, const float *beta, float eps,
                                         const int32_t *R, const int32_t *col_cluster,
                                         const float *scale, const int32_t *zero, int g, int bits,
                                         float *y, float *y_reordered, uint8_t *codes,
                                         rptq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* RPTQ_BASELINE_H_ */
