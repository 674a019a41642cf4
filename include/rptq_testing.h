/*
 * rptq_testing.h -- test hooks of librptq.so.  They are not part of the RPTQ data path and the
 * pages have no counterpart for them; they exist so that tests can check, on the GPU, pieces of
 * arithmetic and failure handling that the entry points of rptq.h cannot expose on their own.
 * Same conventions as rptq.h (device pointers, asynchronous on `stream`, status codes).
 */
#ifndef RPTQ_TESTING_H_
#define RPTQ_TESTING_H_

#include <stdint.h>

#include "rptq.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * The quotient the K/V quantizer forms for a value x and a cluster scale s: a correctly rounded
 * x / s from r = RN(1 / s) and one fused-multiply-add correction (P. Markstein, 2000), in the
 * packed two-lane form of the kernels.  q[i] = quotient(x[i], s) for i < n.
 *   x, q  fp32 [n], device.   s  finite and > 0.
 * Errors: RPTQ_ERR_INVALID_ARG (s not finite or not positive, n < 0, NULL pointers with n > 0),
 * RPTQ_ERR_CUDA (launch failed).  n == 0 launches nothing.
 */
int rptq_testing_kv_quotient(const float *x, int64_t n, float s, float *q, rptq_stream_t stream);

/*
 * Failure-detection hook of the KMeans kernel (rptq_kmeans, rptq_kmeans_noalloc) on the current
 * device: every wait of its cross-CTA exchange and of its grid barrier gives up after
 * `limit_ns` nanoseconds (0 = the default, 2 s), sets RPTQ_DEVERR_TIMEOUT in the device error
 * word and stops waiting for the rest of the call; with withhold_cta >= 0, CTA number
 * `withhold_cta` leaves out its first Lloyd record, so the other CTAs' waits for it run out
 * (every wait still ends, after the limit).  -1 restores normal operation.  The setting stays
 * until changed.  Synchronous (copies to device symbols).  Errors: RPTQ_ERR_INVALID_ARG
 * (withhold_cta < -1), RPTQ_ERR_CUDA.
 */
int rptq_testing_kmeans_wait(unsigned long long limit_ns, int withhold_cta);

#ifdef __cplusplus
}
#endif

#endif /* RPTQ_TESTING_H_ */
