// Host-side internals shared by the library's translation units: the
// context, its workspace and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>
#include <vector>

#include "../../include/zo_debug.h"

namespace zo {

constexpr int kMaxLayersHost = 8;
constexpr int kMaxSegHost = 2 + 2 * kMaxLayersHost;

// Segment table in the flat parameter vector.
struct Segments {
  int n = 0;
  int64_t off[kMaxSegHost];
  int64_t numel[kMaxSegHost];
  int64_t d_pad = 0, d_real = 0;
  // indices into off/numel
  int E = 0, W[kMaxLayersHost], b[kMaxLayersHost], Wout = 0, bout = 0;
};

// Per-probe-sign perturbed copies of the small segments (bf16 path):
// embedding, cell biases, output weights and bias, fp32.
struct SmallLayout {
  int64_t E = 0, b[kMaxLayersHost], Wout = 0, bout = 0, stride = 0;  // float offsets
};

struct CellMaps {
  alignas(64) CUtensorMap x;                    // x_t            [P][B][E]  bf16
  alignas(64) CUtensorMap h[kMaxLayersHost][2];  // h_l (parity)   [P][B][H]  bf16
  alignas(64) CUtensorMap w[kMaxLayersHost];     // W_l shadow     [4H][in+H] bf16, 64-row box
  alignas(64) CUtensorMap wout;                  // W_out shadow   [V][H] bf16, 16-row box
};

}  // namespace zo

struct ZoProfRec {
  cudaEvent_t a = nullptr, b = nullptr;
  int kind = 0;
  double flops = 0, bytes = 0;
};

// Rows of the fp32 cell-state buffer per probe-sign: the batch rounded up to
// the 128-row blocks of its layout.  Within a block the state is stored four
// units at a time, row-minor ([unit/4][row][4]), so the 32 lanes of a warp,
// which hold 32 consecutive rows of one tensor-memory quadrant, read and write
// 512 contiguous bytes.  A layer whose input term comes from the vocabulary
// table keeps it row-major ([row][unit]).
inline int64_t cst_rows(int64_t B) { return (B + 127) / 128 * 128; }

struct zo_ctx {
  zo_model_spec spec;
  int device = 0;
  int sm_count = 0;
  zo::Segments seg;
  int chunk = 0;            // probes per pass
  int64_t ws_bytes = 0;
  unsigned* err = nullptr;  // device error word
  // bf16 path
  __nv_bfloat16* shadow = nullptr;
  const float* shadow_theta = nullptr;
  bool shadow_fresh = false;
  zo::SmallLayout small;
  float* small_p = nullptr;      // [2*chunk][small.stride]
  __nv_bfloat16* x = nullptr;    // [2*chunk][B][E]
  __nv_bfloat16* h = nullptr;    // [L][2][2*chunk][B][H]
  float* cst = nullptr;          // [L][2*chunk][cst_rows(B)*H]: [Bpad/128][H/4][128][4], or
                                 // [B][H] for a layer fed by the vocabulary table
  zo::CellMaps* maps = nullptr;  // host copy of the tensor maps
  // vocabulary table of the first layer's input term (bf16 path, wide
  // embeddings): vt[ps][v][4H] = E'_ps[v] (W_0x +- eps P)^T, built once per chunk
  float* vt = nullptr;
  bool vocab = false;
  // how the cell GEMMs form the perturbed operand (ZO_CELL_*, include/zo_debug.h)
  int cell_variant = 0;
  // both paths
  float* rowloss = nullptr;      // [2*chunk][B]
  // zo_step_host staging (device)
  int32_t* tok = nullptr;
  int32_t* tgt = nullptr;
  float* lp = nullptr;
  float* lm = nullptr;
  float* coef = nullptr;
  int n_stage = 0;               // capacity of lp/lm/coef
  float* l0m = nullptr;          // zo_loss: the second sign's copy of L(theta)
  int fp32_bb = 1;               // rows per CTA of the fp32 forward
  size_t fp32_smem = 0;
  int fp32_wide_np = 0;          // probes per CTA of the probe-column fp32 forward (0: unused)
  float* wt = nullptr;           // its transposed weight copies
  // per-launch timing (zo_profile)
  bool prof_on = false;
  std::vector<ZoProfRec> prof;
  size_t prof_used = 0;
};

namespace zo {

extern std::atomic<int64_t> g_launches;
inline void count_launch(int n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// ---- launchers (each returns cudaGetLastError() after enqueueing) ----
cudaError_t launch_sign_words(uint64_t seed, int probe, int64_t q0, int64_t n, uint32_t* out,
                              cudaStream_t st);
cudaError_t launch_cast_shadow(const float* theta, __nv_bfloat16* shadow, int64_t d_pad,
                               cudaStream_t st);
cudaError_t launch_coeffs(const float* lp, const float* lm, int n, float eps, float eta,
                          float* out, unsigned* err, cudaStream_t st);
cudaError_t launch_coeffs_forward(const float* lp, const float* l0, int n, float eps, float eta,
                                  float* out, unsigned* err, cudaStream_t st);
cudaError_t launch_update(const zo_ctx* ctx, float* theta, uint64_t seed, int n,
                          const float* coeffs, __nv_bfloat16* shadow, cudaStream_t st);
cudaError_t launch_fp32_forward(const zo_ctx* ctx, const float* theta, uint64_t seed, int probe0,
                                int nprobe, float eps, const int32_t* tokens,
                                const int32_t* targets, int B, int T, cudaStream_t st);
cudaError_t launch_reduce_losses(const zo_ctx* ctx, const int32_t* targets, int B, int T,
                                 int probe0, int nprobe, float* lp, float* lm, float* row_out,
                                 cudaStream_t st);
// bf16 path
cudaError_t launch_perturb_small(const zo_ctx* ctx, const float* theta, uint64_t seed, int probe0,
                                 int nprobe, float eps, cudaStream_t st);
cudaError_t launch_gather_x(const zo_ctx* ctx, const int32_t* tokens, int t, int B, int T,
                            int nprobe, cudaStream_t st);
// wait_ns bounds every mbarrier wait of the launch; stall = 1 (a test hook)
// makes the producer issue nothing, so every wait runs out and the kernel
// latches ZO_ERR_TIMEOUT with no copy or MMA in flight
constexpr uint64_t kDefaultWaitNs = 2000000000ull;
cudaError_t launch_loss_tc(const zo_ctx* ctx, const int32_t* targets, int t, int B, int T,
                           int nprobe, int probe0, uint64_t seed, float eps, cudaStream_t st,
                           uint64_t wait_ns = kDefaultWaitNs, int stall = 0);
cudaError_t launch_cell_tc(const zo_ctx* ctx, int layer, int t, int B, int nprobe, int probe0,
                           uint64_t seed, float eps, float* raw_out, const int32_t* tokens, int T,
                           bool vocab, cudaStream_t st, uint64_t wait_ns = kDefaultWaitNs,
                           int stall = 0);
// vocabulary table (rows kVocabRows per probe-sign) and the first step of
// layer 0 from it
constexpr int kVocabRows = 64;
cudaError_t launch_vocab_table(const zo_ctx* ctx, int nprobe, int probe0, uint64_t seed, float eps,
                               cudaStream_t st);
cudaError_t launch_vocab_first(const zo_ctx* ctx, const int32_t* tokens, int B, int T, int nprobe,
                               cudaStream_t st);
cudaError_t launch_vocab_x(const zo_ctx* ctx, int nprobe, cudaStream_t st);
bool make_cell_maps(zo_ctx* ctx);
void layout_of(const zo_model_spec& sp, Segments& s);
// probe-column fp32 forward: probes per CTA that fit `limit` bytes of shared
// memory (0 if the shape is not supported), its workspace and shared memory
int fp32_wide_probes(const zo_model_spec& s, size_t limit, int64_t* wt_floats, size_t* smem);
cudaError_t launch_fp32_wide(const zo_ctx* ctx, const float* theta, uint64_t seed, int probe0,
                             int nprobe, float eps, const int32_t* tokens, const int32_t* targets,
                             int B, int T, cudaStream_t st);
// shared memory of the per-probe fp32 forward for bb batch rows per CTA
size_t fp32_smem_bytes(const zo_model_spec& s, int bb, int64_t d_pad);

}  // namespace zo
