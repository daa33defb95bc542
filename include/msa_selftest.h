/*
 * msa_selftest.h — self-test hooks of libmsa's internal device arithmetic.
 * Not part of the routed step: the pages have no counterpart. They exist so that
 * tests can check a device function on its own, over its whole domain, instead
 * of only through the outputs of the kernel that uses it.
 */
#ifndef MSA_SELFTEST_H_
#define MSA_SELFTEST_H_

#include <stdint.h>

#include "msa.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Evaluates, for i < n, y_poly[i] = the polynomial 2^x that the tcgen05 prefill
 * kernel uses for part of its softmax exponentials (range reduction to the
 * nearest integer n, a Remez cubic for 2^f on [-1/2, 1/2], n added to the
 * exponent; x clamped to [-125, 64] first), and y_lib[i] = CUDA's exp2f(x[i]).
 * x, y_poly, y_lib: device fp32 [n], caller-owned. Asynchronous on `stream`.
 * MSA_ERR_INVALID_ARG for a NULL pointer or n outside [1, 2^30]; MSA_ERR_CUDA
 * if the launch fails. */
msa_status msa_selftest_exp2_poly(const float* x, float* y_poly, float* y_lib, int64_t n, void* stream);

/* The document selection on its own: for each of `rows` rows of n fp32 scores
 * (device, [rows][n], row-major), the k largest, ranked by score (descending) and,
 * between equal scores, by index (ascending); scores compare through the IEEE
 * total order of their bits (-0 below +0). idx[r][i] = the index in row r of
 * rank i; top_scores[r][i] its score (or NULL). idx, top_scores: device,
 * caller-owned [rows][k]. path 0 runs the kernel msa_route uses for this shape,
 * 1 the block-per-row radix select (any n, k <= 64), 2 the warp-per-row select
 * (n <= 2048, k <= 32). Asynchronous on `stream`. MSA_ERR_INVALID_ARG for a NULL
 * scores or idx, rows < 1, n < 1, k outside [1, min(n, 64)], or a path that does
 * not take the shape; MSA_ERR_CUDA if the launch fails. */
msa_status msa_selftest_topk(const float* scores, int32_t rows, int32_t n, int32_t k, int32_t* idx,
                             float* top_scores, int32_t path, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MSA_SELFTEST_H_ */
