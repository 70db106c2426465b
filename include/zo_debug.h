/*
 * zo_debug.h - diagnostic entry point of libzo.so (see zo.h for conventions).
 *
 * zo_debug_cell_preact runs the first step (t = 0) of the perturbed forward
 * for layer 0 only and returns the cell pre-activations instead of updating
 * the state: for probe-sign ps = 2 i + s (s = 0: +eps, 1: -eps) of probes
 * probe0 .. probe0 + n_probes - 1 and batch row b < batch,
 *   preact_dev[(ps * max_batch + b) * 4H + r] =
 *       x_b . (W_1 + (+-eps) P_i)[r, :E] + (b_1 + (+-eps) p_i)[r]
 * with x_b the perturbed embedding row of tokens[b, 0] (the review's
 * L(Theta +- eps p_i) forward, "What carries the argument"; recurrent input
 * h_{-1} = 0).  Only contexts of dtype ZO_DTYPE_BF16 (the tensor-core cell)
 * are accepted; n_probes must not exceed the context's chunk.
 *   preact_dev  fp32 [2 n_probes x max_batch x 4H], device, caller-owned.
 * Async on `stream`; returns ZO_ERR_UNSUPPORTED for fp32 contexts.
 */
#ifndef ZO_DEBUG_H_
#define ZO_DEBUG_H_

#include "zo.h"

#ifdef __cplusplus
extern "C" {
#endif

ZO_API int zo_debug_cell_preact(zo_ctx* ctx, const float* theta_dev, uint64_t step_seed,
                                int32_t probe0, int32_t n_probes, float eps,
                                const int32_t* tokens_dev, int32_t batch, int32_t seq,
                                float* preact_dev, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ZO_DEBUG_H_ */
