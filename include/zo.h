/*
 * zo.h - C ABI of the B200 (sm_100a) hot path of central-difference
 * random-vector gradient estimation (CD-RGE) for multi-layer LSTMs.
 *
 * Method ("Scaling Recurrent Neural Networks to a Billion Parameters with
 * Zero-Order Optimization", Chaubard & Kochenderfer, arXiv 2505.17852):
 *   pith.science review, "What carries the argument":
 *     Theta' = Theta - 1/(2 n_pert) * sum_i (L(Theta + eps p_i) - L(Theta - eps p_i)) p_i,
 *     p_i Rademacher in {-1,+1}^d, step size eta tied to eps.
 *   alex-wiki source page, "Method":
 *     g_hat = 1/K sum_i (L(theta + eps u_i) - L(theta - eps u_i)) / (2 eps) u_i,
 *     with reconstructible random seeds and chunked perturbations.
 *
 * One update is three stream-ordered calls:
 *   zo_probe_losses  -> L+_i, L-_i for every probe     (complete perturbed forwards)
 *   zo_coeffs        -> c_i = eta (L+_i - L-_i) / (2 eps n_pert)
 *   zo_update        -> theta_j -= sum_i c_i p_ij      (probes replayed from the seed)
 *
 * Conventions shared by every call:
 *   - Every call returns an int status (ZO_OK = 0, else a ZO_ERR_* code).  No
 *     C++ exception crosses this interface.  Argument errors are detected on
 *     the host before anything is launched and nothing is written.
 *   - Calls that take a `stream` (a cudaStream_t passed as void*, NULL = the
 *     legacy default stream) only enqueue work on it: they never synchronise.
 *     Errors found by kernels (token out of range, non-finite loss, a bounded
 *     wait that gave up) are latched in a device word of the context and
 *     returned by zo_sync_status().
 *   - Pointers named *_dev are device pointers owned by the caller (allocated
 *     with cudaMalloc, or torch tensors' data_ptr()); pointers named *_host are
 *     host pointers.  The library never frees caller memory.
 *   - A context is bound to the device that was current at zo_create() and is
 *     not thread-safe: serialise calls that use the same context.
 *
 * Parameter layout (flat fp32 vector theta, length d_pad): segments in the
 * order E[V x E]; for each layer l: W_l[4H x (in_l + H)] (row blocks for the
 * gates i, f, g, o; columns [input | recurrent]; in_1 = E, in_l = H), b_l[4H];
 * W_out[V x H]; b_out[V].  Row-major, each segment starting on a multiple of
 * 128 elements, gaps zero.  zo_param_layout() returns the offsets.
 *
 * Probe signs: p_ij = +1 or -1 from bit (e >> 1) + 16 (e & 1), e = j & 31, of
 * word (j >> 5) & 3 of Philox4x32-10 (Salmon et al., SC'11) with key
 * (seed lo, seed hi) and counter (q lo, q hi, i, 0), q = j >> 7.  Bit 1 = -1.
 */
#ifndef ZO_H_
#define ZO_H_

#include <stdint.h>

#if defined(__GNUC__)
#define ZO_API __attribute__((visibility("default")))
#else
#define ZO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define ZO_OK               0
#define ZO_ERR_INVALID_ARG  1  /* bad argument; nothing was launched            */
#define ZO_ERR_CUDA         2  /* a CUDA runtime call failed                    */
#define ZO_ERR_OOM          3  /* device allocation failed (zo_create only)     */
#define ZO_ERR_UNSUPPORTED  4  /* shape outside what this build supports        */
#define ZO_ERR_TIMEOUT      5  /* a bounded device wait gave up (kernel returned) */
#define ZO_ERR_NONFINITE    6  /* a loss or coefficient was NaN/Inf; theta kept  */
#define ZO_ERR_BOUNDS       7  /* token outside [0,V) or target outside [-1,V)  */
#define ZO_ERR_NO_DEVICE    8  /* no CUDA device / not an sm_100 device         */

/* ---- model description ------------------------------------------------- */
#define ZO_DTYPE_FP32 0  /* fp32 operands on CUDA cores (small models)            */
#define ZO_DTYPE_BF16 1  /* bf16 operands, fp32 accumulate, fp32 master theta     */

typedef struct zo_model_spec {
  int32_t vocab;        /* V: token vocabulary (>= 2)                           */
  int32_t embed;        /* E: embedding width                                   */
  int32_t hidden;       /* H: LSTM hidden width                                 */
  int32_t layers;       /* L: stacked LSTM layers (1..8)                        */
  int32_t dtype;        /* ZO_DTYPE_FP32 or ZO_DTYPE_BF16                       */
  int32_t max_batch;    /* largest batch any call will pass                     */
  int32_t max_seq;      /* largest sequence length any call will pass           */
  int32_t chunk;        /* probes evaluated together per pass; 0 = automatic    */
} zo_model_spec;

typedef struct zo_ctx zo_ctx;

/* Create a context on the current device.  Validates the spec, allocates the
 * chunk workspace (recurrent state for 2*chunk perturbed copies) and, for
 * ZO_DTYPE_BF16, the bf16 shadow of theta.  Synchronous.  On error *out is
 * NULL and nothing stays allocated. */
ZO_API int zo_create(const zo_model_spec* spec, zo_ctx** out);

/* Release everything the context allocated (synchronises the device first). */
ZO_API int zo_destroy(zo_ctx* ctx);

/* Flat layout of theta.  d_pad = length of theta; d_real = number of real
 * parameters.  seg_offset/seg_numel (capacity *n_seg on input, may be NULL)
 * receive each segment's offset and element count; *n_seg returns the count
 * (2 + 2L). */
ZO_API int zo_param_layout(const zo_ctx* ctx, int64_t* d_pad, int64_t* d_real,
                    int64_t* seg_offset, int64_t* seg_numel, int32_t* n_seg);

/* Chunk size the context uses (probes per pass) and its workspace bytes. */
ZO_API int zo_workspace_info(const zo_ctx* ctx, int32_t* chunk, int64_t* workspace_bytes);

/* Per-probe central-difference losses (pith.science review, "What carries the
 * argument": two complete forwards per probe).
 *   theta_dev   fp32 [d_pad]; read only.
 *   step_seed   probe seed of this update; probe i is (step_seed, i).
 *   n_pert      number of probes (>= 1).
 *   eps         perturbation radius (finite, > 0).
 *   tokens_dev  int32 [batch x seq] row-major, values in [0, V).
 *   targets_dev int32 [batch x seq], values in [0, V) or -1 (not scored).
 *   loss_plus_dev, loss_minus_dev  fp32 [n_pert]: L(theta +- eps p_i), the
 *               mean softmax cross-entropy over scored positions (0 if none).
 * Probes are processed in chunks of zo_workspace_info()'s chunk; the model is
 * never copied per probe.  Async on `stream`. */
ZO_API int zo_probe_losses(zo_ctx* ctx, const float* theta_dev, uint64_t step_seed, int32_t n_pert,
                    float eps, const int32_t* tokens_dev, const int32_t* targets_dev,
                    int32_t batch, int32_t seq, float* loss_plus_dev, float* loss_minus_dev,
                    void* stream);

/* As zo_probe_losses; if row_loss_dev is not NULL it also receives, for each
 * probe i, sign s (0 = +eps, 1 = -eps) and batch row b, the sum over scored
 * steps of that row's cross-entropy: row_loss_dev[(2 i + s) * batch + b]
 * (fp32, [n_pert x 2 x batch]). */
ZO_API int zo_probe_losses_ex(zo_ctx* ctx, const float* theta_dev, uint64_t step_seed, int32_t n_pert,
                       float eps, const int32_t* tokens_dev, const int32_t* targets_dev,
                       int32_t batch, int32_t seq, float* loss_plus_dev, float* loss_minus_dev,
                       float* row_loss_dev, void* stream);

/* Losses of the probe slice probe_begin .. probe_begin + n_probes - 1 only,
 * written to loss_plus_dev[i], loss_minus_dev[i] (fp32 [n_probes]); probe
 * probe_begin + i is exactly probe probe_begin + i of zo_probe_losses.  This
 * is the unit of the probe-parallel scheme of the pith.science review ("What
 * carries the argument": workers each compute a few perturbed losses and only
 * scalar losses travel): each process evaluates one slice and the slices'
 * losses are gathered before zo_coeffs.  Other arguments and behaviour as
 * zo_probe_losses.  Async on `stream`. */
ZO_API int zo_probe_losses_slice(zo_ctx* ctx, const float* theta_dev, uint64_t step_seed,
                                 int32_t probe_begin, int32_t n_probes, float eps,
                                 const int32_t* tokens_dev, const int32_t* targets_dev,
                                 int32_t batch, int32_t seq, float* loss_plus_dev,
                                 float* loss_minus_dev, void* stream);

/* Coefficients c_i = eta (L+_i - L-_i) / (2 eps n_pert) (alex-wiki "Method";
 * eta = eps gives the review's 1/(2 n_pert) factor).  fp32 [n_pert] in and
 * out, device.  A non-finite input latches ZO_ERR_NONFINITE and writes NaN
 * for that coefficient, which zo_update then refuses.  Async. */
ZO_API int zo_coeffs(zo_ctx* ctx, const float* loss_plus_dev, const float* loss_minus_dev,
              int32_t n_pert, float eps, float eta, float* coeffs_dev, void* stream);

/* L(theta): the mean cross-entropy of the unperturbed forward over the scored
 * targets of tokens_dev / targets_dev (int32 [batch x seq], device), written
 * to loss_dev (one fp32, device).  It runs the probe-loss path for one probe
 * at radius 0, so both of its signs are exactly L(theta); the baseline that a
 * forward difference subtracts, and an exact evaluation loss.  Argument
 * checks and device errors as zo_probe_losses.  Async. */
ZO_API int zo_loss(zo_ctx* ctx, const float* theta_dev, const int32_t* tokens_dev,
                   const int32_t* targets_dev, int32_t batch, int32_t seq, float* loss_dev,
                   void* stream);

/* Forward-difference coefficients c_i = eta (L+_i - L0) / (eps n_pert), with
 * L0 = L(theta) from zo_loss (one fp32, device): the one-sided estimator
 * g_hat = 1/n sum_i (L(theta + eps p_i) - L(theta)) / eps p_i, applied by
 * zo_update like the central coefficients.  Over an antithetic probe set
 * {p_i, -p_i} it equals the central difference (review, "Circularity Check":
 * Appendix C).  Non-finite inputs as in zo_coeffs.  Async. */
ZO_API int zo_coeffs_forward(zo_ctx* ctx, const float* loss_plus_dev, const float* loss0_dev,
                             int32_t n_pert, float eps, float eta, float* coeffs_dev,
                             void* stream);

/* theta_j -= sum_i c_i p_ij for every real parameter j, probes replayed from
 * (step_seed, i) and never stored (review, "What carries the argument").
 * theta_dev is updated in place; padding stays zero.  For ZO_DTYPE_BF16 the
 * bf16 shadow is rewritten in the same pass.  If any coefficient is non-finite
 * theta is left unchanged and ZO_ERR_NONFINITE is latched.  n_pert is at
 * most ZO_MAX_UPDATE_PROBES (above 64 probes the kernel keeps 16 fp32 subset
 * sums per four probes in shared memory); larger counts return
 * ZO_ERR_INVALID_ARG.  Async. */
#define ZO_MAX_UPDATE_PROBES 8192
ZO_API int zo_update(zo_ctx* ctx, float* theta_dev, uint64_t step_seed, int32_t n_pert,
              const float* coeffs_dev, void* stream);

/* The bf16 shadow is reused by zo_probe_losses only when the previous
 * zo_update wrote it from the same theta pointer.  A caller that writes theta
 * by other means (loading a checkpoint, say) into that same buffer must call
 * this so that the next zo_probe_losses recasts it. */
ZO_API int zo_invalidate_shadow(zo_ctx* ctx);

/* One whole update from host buffers: copies tokens/targets (host, int32
 * [batch x seq]) to the device, runs zo_probe_losses, zo_coeffs (eta) and
 * zo_update on theta_dev, copies L+/L- back to the host buffers
 * loss_plus_host/loss_minus_host (fp32 [n_pert]) and synchronises `stream`.
 * Returns the first error, including latched device errors. */
ZO_API int zo_step_host(zo_ctx* ctx, float* theta_dev, uint64_t step_seed, int32_t n_pert, float eps,
                 float eta, const int32_t* tokens_host, const int32_t* targets_host,
                 int32_t batch, int32_t seq, float* loss_plus_host, float* loss_minus_host,
                 void* stream);

/* Synchronise `stream`, then return (and clear) the latched device error:
 * ZO_ERR_TIMEOUT, ZO_ERR_BOUNDS or ZO_ERR_NONFINITE, else ZO_OK. */
ZO_API int zo_sync_status(zo_ctx* ctx, void* stream);

/* Probe sign words (test hook for the sign generator of the review's p_i):
 * out_dev[4 k + w] = word w of Philox4x32-10 for block q0 + k of probe
 * `probe`, k < n_blocks.  uint32, device.  Async; needs no context. */
ZO_API int zo_sign_words(uint64_t step_seed, int32_t probe, int64_t q0, int64_t n_blocks,
                  uint32_t* out_dev, void* stream);

/* Per-kernel timing.  zo_profile(ctx, 1) starts recording a CUDA event pair
 * around every kernel the context launches (and clears earlier records);
 * zo_profile(ctx, 0) stops recording.  zo_profile_read() synchronises the
 * recorded events and returns, for one kernel kind, the number of launches,
 * their summed device time in ms, and the summed algorithmic work of those
 * launches: flops (2 per multiply-add of the plain dense forward the launch
 * computes) and bytes (the HBM bytes the launch must move at minimum).
 * Kinds: ZO_KIND_CELL - tensor-core cell GEMM (bf16) or the whole fp32
 * persistent forward; ZO_KIND_LOSS - output projection + cross-entropy;
 * ZO_KIND_UPDATE - the update; ZO_KIND_OTHER - everything else. */
#define ZO_KIND_CELL   0
#define ZO_KIND_LOSS   1
#define ZO_KIND_UPDATE 2
#define ZO_KIND_OTHER  3
ZO_API int zo_profile(zo_ctx* ctx, int32_t enable);
ZO_API int zo_profile_read(zo_ctx* ctx, int32_t kind, int64_t* launches, double* total_ms,
                           double* total_flops, double* total_bytes);

/* zo_probe_losses for a ZO_DTYPE_FP32 model without a context and without
 * allocating anything.  The paper has no counterpart: this exists for callers
 * that cannot call cudaMalloc at the point where they need the losses - code
 * running under a memory manager that owns the whole device heap, or a
 * latency-critical loop that must not take cudaMalloc's implicit device
 * synchronisation.  Arguments are those of zo_probe_losses (spec replaces the
 * context; its max_batch, max_seq and chunk fields are ignored).  Every probe
 * is evaluated in one pass; the per-row loss sums (2 x n_pert x batch floats)
 * live in a fixed device array of ZO_STATIC_SCRATCH_FLOATS floats that every
 * GPU loading the library keeps until exit.  Larger requests return
 * ZO_ERR_INVALID_ARG before anything is launched; models whose fp32 forward
 * does not fit one CTA's shared memory return ZO_ERR_UNSUPPORTED.
 * The first call on a device resolves that array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls share the array and it keeps the last
 * call's contents: calls that overlap on the GPU (two streams, or two host
 * threads) race and must be serialised by the caller.  Device-detected input
 * errors are not reported here (tokens are clamped, out-of-range targets are
 * not scored): validate tokens and targets beforehand.  No cudaMalloc,
 * cudaFree or allocating library routine is called.  Async on `stream`. */
#define ZO_STATIC_SCRATCH_FLOATS 65536
ZO_API int zo_probe_losses_static(const zo_model_spec* spec, const float* theta_dev,
                                  uint64_t step_seed, int32_t n_pert, float eps,
                                  const int32_t* tokens_dev, const int32_t* targets_dev,
                                  int32_t batch, int32_t seq, float* loss_plus_dev,
                                  float* loss_minus_dev, void* stream);

/* Human-readable name of a status code (static string). */
ZO_API const char* zo_status_string(int status);

/* Kernels this library launched since load (all entry points, all contexts). */
ZO_API int64_t zo_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* ZO_H_ */
