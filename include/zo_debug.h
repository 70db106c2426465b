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

/*
 * zo_debug_cell_stall exercises the bounded device waits (every mbarrier wait
 * of the tensor-core kernels gives up after a time limit, latches
 * ZO_ERR_TIMEOUT in the context's error word and returns).  It launches one
 * tensor-core kernel on the context's own buffers with every wait bounded by
 * wait_ns and with a producer that issues no copy, so no stage ever fills:
 *   kind 0  the CTA-pair cell step of layer 0 (tcgen05.mma.cta_group::2);
 *   kind 1  the single-CTA output layer + cross-entropy (cta_group::1).
 * All waits run out, the CTAs free their tensor memory and return; no copy and
 * no MMA is ever in flight, and the context stays usable.  zo_sync_status()
 * then returns ZO_ERR_TIMEOUT (and clears it).  Only ZO_DTYPE_BF16 contexts
 * (else ZO_ERR_UNSUPPORTED); wait_ns in [1e3, 1e10] ns (else
 * ZO_ERR_INVALID_ARG).  Nothing the caller owns is written.  Async on `stream`.
 */
ZO_API int zo_debug_cell_stall(zo_ctx* ctx, int32_t kind, uint64_t wait_ns, void* stream);

/*
 * zo_debug_cell_variant selects, for the ZO_DTYPE_BF16 context's later calls,
 * how the tensor-core cell GEMMs form the weights at Theta +- eps p_i
 * (alex-wiki "Method"; pith.science review, "What carries the argument") and
 * on which tile form they run.  Every variant computes the same forward; they
 * differ in rounding and speed.  Operand forms:
 *   perturbed operand  B = bf16(bf16(W) +- bf16(eps) p), the bf16 tile of W
 *                      staged in shared memory by TMA and perturbed there;
 *   exact eps          G = A bf16(W)^T + A (+-bf16(eps) p)^T, the two products
 *                      accumulated in fp32: the perturbation is not lost in
 *                      the rounding of bf16(W) +- eps; twice the MMA work;
 *   direct W           as the perturbed operand, but the generator warps read
 *                      the bf16 rows of W from global memory into registers
 *                      and store the perturbed tile themselves.
 * Tile forms: single CTA (256 batch rows as two M = 128 MMAs per K slice on
 * one B, one accumulator) or CTA pair (tcgen05.mma.cta_group::2, M = 256, two
 * accumulators, each CTA loading and perturbing half of B).
 *   ZO_CELL_SINGLE (0, default)  perturbed operand, single CTA
 *   ZO_CELL_SINGLE_EXACT_EPS (1) exact eps, single CTA
 *   ZO_CELL_PAIR (2)             perturbed operand, CTA pair
 *   ZO_CELL_PAIR_EXACT_EPS (3)   exact eps, CTA pair
 *   ZO_CELL_PAIR_DIRECT_W (4)    direct W, CTA pair
 *   ZO_CELL_SINGLE_EPI8 (5)      perturbed operand, single CTA, with four
 *                                generator warps (two W rows a thread) and
 *                                eight epilogue warps (two per TMEM lane
 *                                quadrant, half the units each)
 * Embedding rows and biases are perturbed in fp32 in every variant.  Returns
 * ZO_ERR_UNSUPPORTED for ZO_DTYPE_FP32 contexts, ZO_ERR_INVALID_ARG for an
 * unknown variant.  Synchronous, host only.
 */
#define ZO_CELL_SINGLE 0
#define ZO_CELL_SINGLE_EXACT_EPS 1
#define ZO_CELL_PAIR 2
#define ZO_CELL_PAIR_EXACT_EPS 3
#define ZO_CELL_PAIR_DIRECT_W 4
#define ZO_CELL_SINGLE_EPI8 5
ZO_API int zo_debug_cell_variant(zo_ctx* ctx, int32_t variant);

ZO_API int zo_debug_cell_preact(zo_ctx* ctx, const float* theta_dev, uint64_t step_seed,
                                int32_t probe0, int32_t n_probes, float eps,
                                const int32_t* tokens_dev, int32_t batch, int32_t seq,
                                float* preact_dev, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ZO_DEBUG_H_ */
