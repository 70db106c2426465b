// C ABI of the CD-RGE hot path: context and workspace, argument checks, the
// probe-chunk scheduler ("chunked ... perturbations", alex-wiki "Method") and
// the update driver.  Every kernel runs on the caller's stream; nothing here
// synchronises except zo_create, zo_destroy, zo_step_host and zo_sync_status.
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <new>

#include "../../include/zo_debug.h"
#include "zo_common.cuh"
#include "zo_internal.h"

namespace zo {
std::atomic<int64_t> g_launches{0};
}  // namespace zo

using namespace zo;

namespace {

inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Host-side fault injection for tests, read from the environment at every
// call: ZO_FAULT=alloc makes zo_create's device allocations fail (it returns
// ZO_ERR_OOM and keeps nothing allocated); ZO_FAULT=launch makes the
// probe-loss, coefficient and update calls return ZO_ERR_CUDA before they
// enqueue anything.  No device-side fault is ever injected.
bool injected(const char* what) {
  const char* f = getenv("ZO_FAULT");
  return f && strcmp(f, what) == 0;
}

#define ZO_CUDA(call)                      \
  do {                                     \
    cudaError_t e_ = (call);               \
    if (e_ != cudaSuccess) return ZO_ERR_CUDA; \
  } while (0)

void build_segments(const zo_model_spec& sp, Segments& s) {
  int64_t off = 0;
  s.n = 0;
  s.d_real = 0;
  auto add = [&](int64_t numel) {
    s.off[s.n] = off;
    s.numel[s.n] = numel;
    s.d_real += numel;
    off += numel;
    off = (off + 127) / 128 * 128;
    return s.n++;
  };
  const int64_t V = sp.vocab, E = sp.embed, H = sp.hidden;
  s.E = add(V * E);
  for (int l = 0; l < sp.layers; ++l) {
    const int64_t in_l = l == 0 ? E : H;
    s.W[l] = add(4 * H * (in_l + H));
    s.b[l] = add(4 * H);
  }
  s.Wout = add(V * H);
  s.bout = add(V);
  s.d_pad = off;
}

int64_t align4(int64_t x) { return (x + 3) / 4 * 4; }

// Event pair around one launch when profiling is on.  Returns the record
// index or -1.
int prof_begin(zo_ctx* c, cudaStream_t st, int kind, double flops, double bytes) {
  if (!c->prof_on) return -1;
  if (c->prof_used == c->prof.size()) {
    ZoProfRec r;
    if (cudaEventCreate(&r.a) != cudaSuccess || cudaEventCreate(&r.b) != cudaSuccess) return -1;
    c->prof.push_back(r);
  }
  ZoProfRec& r = c->prof[c->prof_used];
  r.kind = kind;
  r.flops = flops;
  r.bytes = bytes;
  cudaEventRecord(r.a, st);
  return (int)c->prof_used++;
}

void prof_end(zo_ctx* c, cudaStream_t st, int idx) {
  if (idx >= 0) cudaEventRecord(c->prof[idx].b, st);
}

// Run `launch` (a lambda returning cudaError_t) between profiling events.
template <class F>
cudaError_t timed(zo_ctx* c, cudaStream_t st, int kind, double flops, double bytes, F&& launch) {
  const int idx = prof_begin(c, st, kind, flops, bytes);
  cudaError_t e = launch();
  prof_end(c, st, idx);
  return e;
}

void free_ctx(zo_ctx* c) {
  if (!c) return;
  cudaFree(c->err);
  cudaFree(c->shadow);
  cudaFree(c->small_p);
  cudaFree(c->x);
  cudaFree(c->h);
  cudaFree(c->cst);
  cudaFree(c->rowloss);
  cudaFree(c->tok);
  cudaFree(c->tgt);
  cudaFree(c->lp);
  cudaFree(c->lm);
  cudaFree(c->coef);
  cudaFree(c->wt);
  cudaFree(c->vt);
  cudaFree(c->l0m);
  for (auto& r : c->prof) {
    if (r.a) cudaEventDestroy(r.a);
    if (r.b) cudaEventDestroy(r.b);
  }
  delete c->maps;
  delete c;
}

bool bf16_shape_ok(const zo_model_spec& s) {
  // tcgen05 cell GEMM: K tiles of 64 over the input and recurrent widths, N
  // tiles of 4 gates x 64 units, V <= 64 logits per row in the loss kernel.
  return s.embed % 64 == 0 && s.hidden % 64 == 0 && s.vocab <= 64;
}

}  // namespace

namespace zo {
// The flat parameter layout of a spec (the same one zo_create builds).
void layout_of(const zo_model_spec& sp, Segments& s) { build_segments(sp, s); }
}  // namespace zo

extern "C" {

const char* zo_status_string(int st) {
  switch (st) {
    case ZO_OK: return "ok";
    case ZO_ERR_INVALID_ARG: return "invalid argument";
    case ZO_ERR_CUDA: return "CUDA runtime error";
    case ZO_ERR_OOM: return "out of device memory";
    case ZO_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case ZO_ERR_TIMEOUT: return "device wait timed out";
    case ZO_ERR_NONFINITE: return "non-finite loss or coefficient";
    case ZO_ERR_BOUNDS: return "token or target out of range";
    case ZO_ERR_NO_DEVICE: return "no sm_100 CUDA device";
    default: return "unknown status";
  }
}

int64_t zo_kernel_launches(void) { return g_launches.load(); }

int zo_create(const zo_model_spec* spec, zo_ctx** out) {
  if (!out) return ZO_ERR_INVALID_ARG;
  *out = nullptr;
  if (!spec) return ZO_ERR_INVALID_ARG;
  const zo_model_spec s = *spec;
  if (s.vocab < 2 || s.embed < 1 || s.hidden < 1 || s.layers < 1 || s.layers > kMaxLayersHost ||
      s.max_batch < 1 || s.max_seq < 1 || s.chunk < 0 ||
      (s.dtype != ZO_DTYPE_FP32 && s.dtype != ZO_DTYPE_BF16))
    return ZO_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ZO_ERR_NO_DEVICE;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return ZO_ERR_NO_DEVICE;
  if (prop.major != 10) return ZO_ERR_NO_DEVICE;
  if (s.dtype == ZO_DTYPE_BF16 && !bf16_shape_ok(s)) return ZO_ERR_UNSUPPORTED;

  zo_ctx* c = new (std::nothrow) zo_ctx();
  if (!c) return ZO_ERR_OOM;
  c->spec = s;
  c->device = dev;
  c->sm_count = prop.multiProcessorCount;
  build_segments(s, c->seg);
  const int64_t B = s.max_batch, E = s.embed, H = s.hidden, V = s.vocab, L = s.layers;
  int rc = ZO_OK;
  const bool fail_alloc = injected("alloc");
  auto alloc = [&](void** p, size_t bytes) {
    if (rc != ZO_OK) return;
    if (fail_alloc) {
      rc = ZO_ERR_OOM;
      return;
    }
    if (cudaMalloc(p, bytes) != cudaSuccess) {
      cudaGetLastError();
      rc = ZO_ERR_OOM;
    } else {
      c->ws_bytes += (int64_t)bytes;
    }
  };
  alloc((void**)&c->err, sizeof(unsigned));
  if (rc == ZO_OK) cudaMemset(c->err, 0, sizeof(unsigned));
  alloc((void**)&c->l0m, sizeof(float));
  alloc((void**)&c->tok, sizeof(int32_t) * B * s.max_seq);
  alloc((void**)&c->tgt, sizeof(int32_t) * B * s.max_seq);

  if (s.dtype == ZO_DTYPE_FP32) {
    // rows per CTA: the smallest power of two >= min(B, 8) whose state fits
    // (the probe's sign words for all d_pad parameters live in shared memory)
    const int64_t dp = c->seg.d_pad;
    int bb = 8;
    while (bb > 1 && (bb / 2 >= B || fp32_smem_bytes(s, bb, dp) > 200 * 1024)) bb /= 2;
    if (fp32_smem_bytes(s, bb, dp) > 200 * 1024) {
      free_ctx(c);
      return ZO_ERR_UNSUPPORTED;
    }
    c->fp32_bb = bb;
    c->fp32_smem = fp32_smem_bytes(s, bb, dp);
    // probe-column forward (several probes share each weight load) where the
    // shape and shared memory allow; it needs a transposed copy of W
    int64_t wt_floats = 0;
    size_t wide_smem = 0;
    const int wnp = fp32_wide_probes(s, 220 * 1024, &wt_floats, &wide_smem);
    if (wnp > 0) {
      alloc((void**)&c->wt, sizeof(float) * (size_t)wt_floats);
      c->fp32_wide_np = wnp;
    }
    c->chunk = s.chunk > 0 ? s.chunk : 4096;
    alloc((void**)&c->rowloss, sizeof(float) * 2 * (size_t)c->chunk * B);
  } else {
    SmallLayout& sl = c->small;
    int64_t o = 0;
    sl.E = o;
    o += align4(V * E);
    for (int l = 0; l < L; ++l) {
      sl.b[l] = o;
      o += align4(4 * H);
    }
    sl.Wout = o;
    o += align4(V * H);
    sl.bout = o;
    o += align4(V);
    sl.stride = o;
    // the first layer's input term from a per-chunk vocabulary table where the
    // embedding is wide enough that the table's gather (16 B per gate row and
    // batch row) costs less than the input K stages it replaces (2 E flops),
    // and the vocabulary rows fit one 256-row tile of the x buffer
    c->vocab = E >= 512 && B >= 256;
    const int64_t per_ps = 2 * B * E + L * 2 * B * H * 2 + L * cst_rows(B) * H * 4 + sl.stride * 4 + B * 4 +
                           (c->vocab ? (int64_t)kVocabRows * 4 * H * 4 : 0);
    int chunk = s.chunk;
    if (chunk == 0) {
      size_t fr = 0, tot = 0;
      cudaMemGetInfo(&fr, &tot);
      const int64_t budget = (int64_t)(fr * 0.4);
      chunk = 64;
      while (chunk > 1 && 2 * chunk * per_ps > budget) chunk /= 2;
    }
    c->chunk = chunk;
    const int64_t P = 2 * (int64_t)chunk;
    alloc((void**)&c->shadow, sizeof(__nv_bfloat16) * c->seg.d_pad);
    alloc((void**)&c->small_p, sizeof(float) * P * sl.stride);
    alloc((void**)&c->x, sizeof(__nv_bfloat16) * P * B * E);
    alloc((void**)&c->h, sizeof(__nv_bfloat16) * L * 2 * P * B * H);
    alloc((void**)&c->cst, sizeof(float) * L * P * cst_rows(B) * H);
    alloc((void**)&c->rowloss, sizeof(float) * P * B);
    if (c->vocab) alloc((void**)&c->vt, sizeof(float) * P * kVocabRows * 4 * H);
    if (rc == ZO_OK && !make_cell_maps(c)) rc = ZO_ERR_CUDA;
  }
  if (rc == ZO_OK && cudaDeviceSynchronize() != cudaSuccess) rc = ZO_ERR_CUDA;
  if (rc != ZO_OK) {
    free_ctx(c);
    return rc;
  }
  *out = c;
  return ZO_OK;
}

int zo_destroy(zo_ctx* ctx) {
  if (!ctx) return ZO_ERR_INVALID_ARG;
  cudaDeviceSynchronize();
  free_ctx(ctx);
  return ZO_OK;
}

int zo_param_layout(const zo_ctx* ctx, int64_t* d_pad, int64_t* d_real, int64_t* seg_offset,
                    int64_t* seg_numel, int32_t* n_seg) {
  if (!ctx) return ZO_ERR_INVALID_ARG;
  if (d_pad) *d_pad = ctx->seg.d_pad;
  if (d_real) *d_real = ctx->seg.d_real;
  if (n_seg) {
    const int cap = *n_seg;
    for (int i = 0; i < ctx->seg.n && i < cap; ++i) {
      if (seg_offset) seg_offset[i] = ctx->seg.off[i];
      if (seg_numel) seg_numel[i] = ctx->seg.numel[i];
    }
    *n_seg = ctx->seg.n;
  }
  return ZO_OK;
}

int zo_workspace_info(const zo_ctx* ctx, int32_t* chunk, int64_t* workspace_bytes) {
  if (!ctx) return ZO_ERR_INVALID_ARG;
  if (chunk) *chunk = ctx->chunk;
  if (workspace_bytes) *workspace_bytes = ctx->ws_bytes;
  return ZO_OK;
}

int zo_invalidate_shadow(zo_ctx* ctx) {
  if (!ctx) return ZO_ERR_INVALID_ARG;
  ctx->shadow_fresh = false;
  return ZO_OK;
}

// Losses of probes probe_begin .. probe_begin + n_pert - 1 (the probes' signs
// use their global index), written to loss_plus[i], loss_minus[i] for
// i < n_pert.
// radius0: the unperturbed forward (zo_loss), eps must be 0.
static int probe_losses_range(zo_ctx* ctx, const float* theta, uint64_t seed, int32_t probe_begin,
                              int32_t n_pert, float eps, const int32_t* tokens,
                              const int32_t* targets, int32_t batch, int32_t seq, float* loss_plus,
                              float* loss_minus, float* row_loss, void* stream,
                              bool radius0 = false) {
  if (!ctx || !theta || !tokens || !targets || !loss_plus || !loss_minus) return ZO_ERR_INVALID_ARG;
  if (n_pert < 1 || probe_begin < 0 || (int64_t)probe_begin + n_pert > INT32_MAX ||
      !(radius0 ? eps == 0.f : (eps > 0.f && isfinite(eps))))
    return ZO_ERR_INVALID_ARG;
  if (batch < 1 || batch > ctx->spec.max_batch || seq < 1 || seq > ctx->spec.max_seq)
    return ZO_ERR_INVALID_ARG;
  if (injected("launch")) return ZO_ERR_CUDA;
  cudaStream_t st = S(stream);
  const int B = batch, T = seq;
  const int64_t Vv = ctx->spec.vocab, Ee = ctx->spec.embed, Hh = ctx->spec.hidden;
  double fwd_macs = (double)Vv * Hh;  // multiply-adds per token of the plain forward
  for (int l = 0; l < ctx->spec.layers; ++l) fwd_macs += 4.0 * Hh * ((l == 0 ? Ee : Hh) + Hh);
  if (ctx->spec.dtype == ZO_DTYPE_FP32) {
    for (int p0 = 0; p0 < n_pert; p0 += ctx->chunk) {
      const int np = n_pert - p0 < ctx->chunk ? n_pert - p0 : ctx->chunk;
      const double fl = 2.0 * 2 * np * (double)B * T * fwd_macs;
      ZO_CUDA(timed(ctx, st, ZO_KIND_CELL, fl, 0.0, [&] {
        return ctx->fp32_wide_np
                   ? launch_fp32_wide(ctx, theta, seed, probe_begin + p0, np, eps, tokens, targets,
                                      B, T, st)
                   : launch_fp32_forward(ctx, theta, seed, probe_begin + p0, np, eps, tokens,
                                         targets, B, T, st);
      }));
      ZO_CUDA(timed(ctx, st, ZO_KIND_OTHER, 0.0, 0.0, [&] {
        return launch_reduce_losses(ctx, targets, B, T, p0, np, loss_plus, loss_minus, row_loss, st);
      }));
    }
    return ZO_OK;
  }
  if (!ctx->shadow_fresh || ctx->shadow_theta != theta) {
    ZO_CUDA(timed(ctx, st, ZO_KIND_OTHER, 0.0, 6.0 * ctx->seg.d_pad,
                  [&] { return launch_cast_shadow(theta, ctx->shadow, ctx->seg.d_pad, st); }));
    ctx->shadow_theta = theta;
    ctx->shadow_fresh = true;
  }
  const int L = ctx->spec.layers;
  for (int p0 = 0; p0 < n_pert; p0 += ctx->chunk) {
    const int np = n_pert - p0 < ctx->chunk ? n_pert - p0 : ctx->chunk;
    const double P = 2.0 * np;
    ZO_CUDA(timed(ctx, st, ZO_KIND_OTHER, 0.0, 0.0,
                  [&] { return launch_perturb_small(ctx, theta, seed, probe_begin + p0, np, eps, st); }));
    ZO_CUDA(cudaMemsetAsync(ctx->rowloss, 0, sizeof(float) * 2 * np * ctx->spec.max_batch, st));
    const bool vocab = ctx->vocab;
    if (vocab) {
      // executed flops: the 256-row tile over the vocabulary rows
      const double fl = 2.0 * P * 256.0 * Ee * 4.0 * Hh * ((ctx->cell_variant == ZO_CELL_SINGLE_EXACT_EPS || ctx->cell_variant == ZO_CELL_PAIR_EXACT_EPS) ? 2.0 : 1.0);
      ZO_CUDA(timed(ctx, st, ZO_KIND_OTHER, 0.0, 0.0, [&] { return launch_vocab_x(ctx, np, st); }));
      ZO_CUDA(timed(ctx, st, ZO_KIND_CELL, fl, 0.0, [&] {
        return launch_vocab_table(ctx, np, probe_begin + p0, seed, eps, st);
      }));
    }
    for (int t = 0; t < T; ++t) {
      if (!vocab)
        ZO_CUDA(timed(ctx, st, ZO_KIND_OTHER, 0.0, P * B * Ee * 2.0,
                      [&] { return launch_gather_x(ctx, tokens, t, B, T, np, st); }));
      for (int l = 0; l < L; ++l) {
        if (vocab && l == 0 && t == 0) {
          ZO_CUDA(timed(ctx, st, ZO_KIND_OTHER, 0.0, 0.0,
                        [&] { return launch_vocab_first(ctx, tokens, B, T, np, st); }));
          continue;
        }
        const double Kin = (vocab && l == 0) ? 0.0 : (double)(l == 0 ? Ee : Hh);
        const double Krun = Kin + (t == 0 ? 0.0 : (double)Hh);
        // executed flops (twice over with the separate +-eps P product)
        const double fl = 2.0 * P * B * Krun * 4.0 * Hh * ((ctx->cell_variant == ZO_CELL_SINGLE_EXACT_EPS || ctx->cell_variant == ZO_CELL_PAIR_EXACT_EPS) ? 2.0 : 1.0);
        ZO_CUDA(timed(ctx, st, ZO_KIND_CELL, fl, 0.0, [&] {
          return launch_cell_tc(ctx, l, t, B, np, probe_begin + p0, seed, eps, nullptr, tokens, T,
                                vocab, st);
        }));
      }
      ZO_CUDA(timed(ctx, st, ZO_KIND_LOSS, 2.0 * P * B * Hh * Vv, P * B * Hh * 2.0, [&] {
        return launch_loss_tc(ctx, targets, t, B, T, np, probe_begin + p0, seed, eps, st);
      }));
    }
    ZO_CUDA(timed(ctx, st, ZO_KIND_OTHER, 0.0, 0.0, [&] {
      return launch_reduce_losses(ctx, targets, B, T, p0, np, loss_plus, loss_minus, row_loss, st);
    }));
  }
  return ZO_OK;
}

int zo_probe_losses_ex(zo_ctx* ctx, const float* theta, uint64_t seed, int32_t n_pert, float eps,
                       const int32_t* tokens, const int32_t* targets, int32_t batch, int32_t seq,
                       float* loss_plus, float* loss_minus, float* row_loss, void* stream) {
  return probe_losses_range(ctx, theta, seed, 0, n_pert, eps, tokens, targets, batch, seq,
                            loss_plus, loss_minus, row_loss, stream);
}

int zo_probe_losses_slice(zo_ctx* ctx, const float* theta, uint64_t seed, int32_t probe_begin,
                          int32_t n_probes, float eps, const int32_t* tokens,
                          const int32_t* targets, int32_t batch, int32_t seq, float* loss_plus,
                          float* loss_minus, void* stream) {
  return probe_losses_range(ctx, theta, seed, probe_begin, n_probes, eps, tokens, targets, batch,
                            seq, loss_plus, loss_minus, nullptr, stream);
}

int zo_probe_losses(zo_ctx* ctx, const float* theta, uint64_t seed, int32_t n_pert, float eps,
                    const int32_t* tokens, const int32_t* targets, int32_t batch, int32_t seq,
                    float* loss_plus, float* loss_minus, void* stream) {
  return zo_probe_losses_ex(ctx, theta, seed, n_pert, eps, tokens, targets, batch, seq, loss_plus,
                            loss_minus, nullptr, stream);
}

int zo_coeffs(zo_ctx* ctx, const float* lp, const float* lm, int32_t n, float eps, float eta,
              float* coeffs, void* stream) {
  if (!ctx || !lp || !lm || !coeffs || n < 1) return ZO_ERR_INVALID_ARG;
  if (!(eps > 0.f) || !isfinite(eps) || !isfinite(eta)) return ZO_ERR_INVALID_ARG;
  if (injected("launch")) return ZO_ERR_CUDA;
  ZO_CUDA(timed(ctx, S(stream), ZO_KIND_OTHER, 0.0, 0.0, [&] {
    return launch_coeffs(lp, lm, n, eps, eta, coeffs, ctx->err, S(stream));
  }));
  return ZO_OK;
}

int zo_loss(zo_ctx* ctx, const float* theta, const int32_t* tokens, const int32_t* targets,
            int32_t batch, int32_t seq, float* loss, void* stream) {
  if (!ctx || !loss) return ZO_ERR_INVALID_ARG;
  return probe_losses_range(ctx, theta, 0, 0, 1, 0.f, tokens, targets, batch, seq, loss, ctx->l0m,
                            nullptr, stream, true);
}

int zo_coeffs_forward(zo_ctx* ctx, const float* lp, const float* l0, int32_t n, float eps,
                      float eta, float* coeffs, void* stream) {
  if (!ctx || !lp || !l0 || !coeffs || n < 1) return ZO_ERR_INVALID_ARG;
  if (!(eps > 0.f) || !isfinite(eps) || !isfinite(eta)) return ZO_ERR_INVALID_ARG;
  ZO_CUDA(timed(ctx, S(stream), ZO_KIND_OTHER, 0.0, 0.0, [&] {
    return launch_coeffs_forward(lp, l0, n, eps, eta, coeffs, ctx->err, S(stream));
  }));
  return ZO_OK;
}

int zo_update(zo_ctx* ctx, float* theta, uint64_t seed, int32_t n, const float* coeffs,
              void* stream) {
  if (!ctx || !theta || !coeffs || n < 1 || n > ZO_MAX_UPDATE_PROBES) return ZO_ERR_INVALID_ARG;
  if (injected("launch")) return ZO_ERR_CUDA;
  __nv_bfloat16* sh = ctx->spec.dtype == ZO_DTYPE_BF16 ? ctx->shadow : nullptr;
  const double bytes = (double)ctx->seg.d_pad * (sh ? 10.0 : 8.0);
  ZO_CUDA(timed(ctx, S(stream), ZO_KIND_UPDATE, 0.0, bytes,
                [&] { return launch_update(ctx, theta, seed, n, coeffs, sh, S(stream)); }));
  if (sh) {
    ctx->shadow_theta = theta;
    ctx->shadow_fresh = true;
  }
  return ZO_OK;
}

int zo_sync_status(zo_ctx* ctx, void* stream) {
  if (!ctx) return ZO_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return ZO_ERR_CUDA;
  unsigned w = 0;
  if (cudaMemcpy(&w, ctx->err, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess)
    return ZO_ERR_CUDA;
  if (w) {
    if (cudaMemset(ctx->err, 0, sizeof(unsigned)) != cudaSuccess) return ZO_ERR_CUDA;
  }
  if (w & kErrTimeout) return ZO_ERR_TIMEOUT;
  if (w & kErrBounds) return ZO_ERR_BOUNDS;
  if (w & kErrNonfinite) return ZO_ERR_NONFINITE;
  return ZO_OK;
}

int zo_step_host(zo_ctx* ctx, float* theta, uint64_t seed, int32_t n, float eps, float eta,
                 const int32_t* tokens_h, const int32_t* targets_h, int32_t batch, int32_t seq,
                 float* lp_h, float* lm_h, void* stream) {
  if (!ctx || !theta || !tokens_h || !targets_h || !lp_h || !lm_h || n < 1)
    return ZO_ERR_INVALID_ARG;
  if (batch < 1 || batch > ctx->spec.max_batch || seq < 1 || seq > ctx->spec.max_seq)
    return ZO_ERR_INVALID_ARG;
  if (!(eps > 0.f) || !isfinite(eps) || !isfinite(eta)) return ZO_ERR_INVALID_ARG;
  cudaStream_t st = S(stream);
  if (n > ctx->n_stage) {
    cudaStreamSynchronize(st);
    cudaFree(ctx->lp);
    cudaFree(ctx->lm);
    cudaFree(ctx->coef);
    ctx->lp = ctx->lm = ctx->coef = nullptr;
    ctx->n_stage = 0;
    if (cudaMalloc(&ctx->lp, sizeof(float) * n) != cudaSuccess ||
        cudaMalloc(&ctx->lm, sizeof(float) * n) != cudaSuccess ||
        cudaMalloc(&ctx->coef, sizeof(float) * n) != cudaSuccess) {
      cudaGetLastError();
      return ZO_ERR_OOM;
    }
    ctx->n_stage = n;
  }
  const size_t tb = sizeof(int32_t) * (size_t)batch * seq;
  ZO_CUDA(cudaMemcpyAsync(ctx->tok, tokens_h, tb, cudaMemcpyHostToDevice, st));
  ZO_CUDA(cudaMemcpyAsync(ctx->tgt, targets_h, tb, cudaMemcpyHostToDevice, st));
  int rc = zo_probe_losses(ctx, theta, seed, n, eps, ctx->tok, ctx->tgt, batch, seq, ctx->lp,
                           ctx->lm, stream);
  if (rc) return rc;
  rc = zo_coeffs(ctx, ctx->lp, ctx->lm, n, eps, eta, ctx->coef, stream);
  if (rc) return rc;
  rc = zo_update(ctx, theta, seed, n, ctx->coef, stream);
  if (rc) return rc;
  ZO_CUDA(cudaMemcpyAsync(lp_h, ctx->lp, sizeof(float) * n, cudaMemcpyDeviceToHost, st));
  ZO_CUDA(cudaMemcpyAsync(lm_h, ctx->lm, sizeof(float) * n, cudaMemcpyDeviceToHost, st));
  return zo_sync_status(ctx, stream);
}

int zo_sign_words(uint64_t seed, int32_t probe, int64_t q0, int64_t n_blocks, uint32_t* out,
                  void* stream) {
  if (!out || probe < 0 || q0 < 0 || n_blocks < 0) return ZO_ERR_INVALID_ARG;
  ZO_CUDA(launch_sign_words(seed, probe, q0, n_blocks, out, S(stream)));
  return ZO_OK;
}

int zo_profile(zo_ctx* ctx, int32_t enable) {
  if (!ctx) return ZO_ERR_INVALID_ARG;
  ctx->prof_on = enable != 0;
  if (enable) ctx->prof_used = 0;
  return ZO_OK;
}

int zo_profile_read(zo_ctx* ctx, int32_t kind, int64_t* launches, double* total_ms,
                    double* total_flops, double* total_bytes) {
  if (!ctx || kind < 0 || kind > ZO_KIND_OTHER) return ZO_ERR_INVALID_ARG;
  int64_t n = 0;
  double ms = 0, fl = 0, by = 0;
  for (size_t i = 0; i < ctx->prof_used; ++i) {
    const ZoProfRec& r = ctx->prof[i];
    if (r.kind != kind) continue;
    if (cudaEventSynchronize(r.b) != cudaSuccess) return ZO_ERR_CUDA;
    float e = 0.f;
    if (cudaEventElapsedTime(&e, r.a, r.b) != cudaSuccess) return ZO_ERR_CUDA;
    ++n;
    ms += e;
    fl += r.flops;
    by += r.bytes;
  }
  if (launches) *launches = n;
  if (total_ms) *total_ms = ms;
  if (total_flops) *total_flops = fl;
  if (total_bytes) *total_bytes = by;
  return ZO_OK;
}

int zo_debug_cell_variant(zo_ctx* ctx, int32_t variant) {
  if (!ctx || variant < ZO_CELL_SINGLE || variant > ZO_CELL_SINGLE_EPI8)
    return ZO_ERR_INVALID_ARG;
  if (ctx->spec.dtype != ZO_DTYPE_BF16) return ZO_ERR_UNSUPPORTED;
  ctx->cell_variant = variant;
  return ZO_OK;
}

int zo_debug_cell_stall(zo_ctx* ctx, int32_t kind, uint64_t wait_ns, void* stream) {
  if (!ctx || (kind != 0 && kind != 1) || wait_ns < 1000ull || wait_ns > 10000000000ull)
    return ZO_ERR_INVALID_ARG;
  if (ctx->spec.dtype != ZO_DTYPE_BF16) return ZO_ERR_UNSUPPORTED;
  cudaStream_t st = S(stream);
  const int B = ctx->spec.max_batch, T = ctx->spec.max_seq;
  if (kind == 0)
    ZO_CUDA(launch_cell_tc(ctx, 0, 1, B, 1, 0, 0, 1e-3f, nullptr, ctx->tok, T, false, st, wait_ns,
                           1));
  else
    ZO_CUDA(launch_loss_tc(ctx, ctx->tgt, 0, B, T, 1, 0, 0, 1e-3f, st, wait_ns, 1));
  return ZO_OK;
}

int zo_debug_cell_preact(zo_ctx* ctx, const float* theta, uint64_t seed, int32_t probe0,
                         int32_t n_probes, float eps, const int32_t* tokens, int32_t batch,
                         int32_t seq, float* preact, void* stream) {
  if (!ctx || !theta || !tokens || !preact || probe0 < 0 || n_probes < 1) return ZO_ERR_INVALID_ARG;
  if (ctx->spec.dtype != ZO_DTYPE_BF16) return ZO_ERR_UNSUPPORTED;
  if (n_probes > ctx->chunk || batch < 1 || batch > ctx->spec.max_batch || seq < 1 ||
      seq > ctx->spec.max_seq || !(eps > 0.f))
    return ZO_ERR_INVALID_ARG;
  cudaStream_t st = S(stream);
  ZO_CUDA(launch_cast_shadow(theta, ctx->shadow, ctx->seg.d_pad, st));
  ctx->shadow_theta = theta;
  ctx->shadow_fresh = true;
  ZO_CUDA(launch_perturb_small(ctx, theta, seed, probe0, n_probes, eps, st));
  ZO_CUDA(launch_gather_x(ctx, tokens, 0, batch, seq, n_probes, st));
  ZO_CUDA(launch_cell_tc(ctx, 0, 0, batch, n_probes, probe0, seed, eps, preact, tokens, seq, false,
                         st));
  return ZO_OK;
}

}  // extern "C"
