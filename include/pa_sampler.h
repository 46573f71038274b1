/*
 * pa_sampler.h -- C ABI of the fused next-token sampler.
 *
 * Source: "vLLM 基本原理", section "FlashInfer 采样器": the logits a step
 * produces go through temperature scaling, Top-K, Top-P and a random draw;
 * a fused kernel does all of it without sorting the logits and is
 * statistically equivalent to the sort-based sampler.
 *
 * For row r with logits x (vocab entries), T = temperature[r], K = top_k[r],
 * P = top_p[r], u = uniform[r]:
 *   - T <= 0 (or NaN): the largest logit, lowest index among equals.
 *   - otherwise p_i ∝ exp(x_i / T);
 *     0 < K < vocab: keep the tokens whose logit is at least the K-th largest
 *     (ties with it are all kept);
 *     P < 1: of those, keep the tokens in decreasing logit order until their
 *     probability reaches P of what Top-K kept, plus every token tied with the
 *     last one;
 *     the token is the first kept one, in vocabulary order, whose cumulative
 *     kept probability exceeds u (inverse-CDF sampling; u outside [0, 1) is
 *     taken as 0).
 * Probabilities are computed in fp32 and summed exactly in 32.32 fixed point,
 * so a row's result depends only on its inputs.  Logits must be finite or
 * -inf; NaN logits are never drawn.
 *
 *   logits       fp32 [num_rows][row_stride], device; row_stride >= vocab
 *                (any stride: the kernel reads single floats).
 *   temperature, top_p  fp32 [num_rows], device.
 *   top_k        int32 [num_rows], device (<= 0 or >= vocab: no Top-K).
 *   uniform      fp32 [num_rows], device: the caller's uniform numbers.
 *   tokens       int32 [num_rows], device, out.
 * Asynchronous on `stream`; PA_ERR_ARG on bad sizes, NULL or misaligned pointers.
 */
#ifndef PA_SAMPLER_H_
#define PA_SAMPLER_H_

#include "pa.h"

#ifdef __cplusplus
extern "C" {
#endif

PA_API int pa_sample(const float* logits, int64_t row_stride, int32_t num_rows, int32_t vocab,
                     const float* temperature, const int32_t* top_k, const float* top_p,
                     const float* uniform, int32_t* tokens, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_SAMPLER_H_ */
