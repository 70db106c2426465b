// Small kernels of the perturbed forward: perturbed copies of the small
// segments, the embedding gather that builds the first layer's input, and the
// final per-probe loss reduction.  "Central-difference random-vector gradient estimation evaluates
// complete recurrent forwards at perturbed weights" (alex-wiki, "Method").
#include "zo_common.cuh"
#include "zo_internal.h"

namespace zo {

// ---------------------------------------------------------------------------
// Perturbed small segments: for every probe-sign ps = 2*ci + s of the chunk,
// small_p[ps] = theta_seg + (s ? -eps : +eps) * p_{probe0+ci} over the
// embedding, every cell bias, W_out and b_out (fp32).
// ---------------------------------------------------------------------------
struct SmallArgs {
  const float* theta;
  float* out;
  uint64_t seed;
  int probe0;
  int nprobe;
  float eps;
  int nparts;
  int64_t src[kMaxSeg];   // theta offset of each part
  int64_t dst[kMaxSeg];   // float offset inside one probe-sign's block
  int64_t len[kMaxSeg];
  int64_t stride;         // floats per probe-sign
  int64_t blocks_per_probe;
  int64_t part_blk0[kMaxSeg + 1];  // first 128-block index of each part (cumulative)
};

// One warp per 128-element block: every lane derives the block's sign words,
// lane l handles elements l, l + 32, l + 64 and l + 96 (coalesced rows).
__global__ void perturb_small_kernel(const SmallArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t total = a.blocks_per_probe * a.nprobe;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t t = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; t < total; t += warps) {
    const int ci = (int)(t / a.blocks_per_probe);
    int64_t rb = t - (int64_t)ci * a.blocks_per_probe;
    int part = 0;
    while (part + 1 < a.nparts && rb >= a.part_blk0[part + 1]) ++part;
    const int64_t kb = rb - a.part_blk0[part];               // block within part
    const int64_t j0 = a.src[part] + kb * 128;                // 128-aligned theta index
    const int64_t n = min((int64_t)128, a.len[part] - kb * 128);
    const uint4 w = sign_block(a.seed, (uint32_t)(a.probe0 + ci), (uint64_t)(j0 >> 7));
    float* op = a.out + (int64_t)(2 * ci) * a.stride + a.dst[part] + kb * 128;
    float* om = op + a.stride;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = lane + 32 * q;
      if (e < n) {
        const float th = a.theta[j0 + e];
        const float d = sign_bit(w, j0 + e) ? -a.eps : a.eps;
        op[e] = th + d;
        om[e] = th - d;
      }
    }
  }
}

cudaError_t launch_perturb_small(const zo_ctx* ctx, const float* theta, uint64_t seed, int probe0,
                                 int nprobe, float eps, cudaStream_t st) {
  const Segments& s = ctx->seg;
  const SmallLayout& sl = ctx->small;
  const int L = ctx->spec.layers;
  SmallArgs a;
  a.theta = theta;
  a.out = ctx->small_p;
  a.seed = seed;
  a.probe0 = probe0;
  a.nprobe = nprobe;
  a.eps = eps;
  int np = 0;
  auto add = [&](int seg, int64_t dst) {
    a.src[np] = s.off[seg];
    a.dst[np] = dst;
    a.len[np] = s.numel[seg];
    ++np;
  };
  add(s.E, sl.E);
  for (int l = 0; l < L; ++l) add(s.b[l], sl.b[l]);
  add(s.Wout, sl.Wout);
  add(s.bout, sl.bout);
  a.nparts = np;
  int64_t cum = 0;
  for (int i = 0; i < np; ++i) {
    a.part_blk0[i] = cum;
    cum += (a.len[i] + 127) / 128;
  }
  a.part_blk0[np] = cum;
  a.blocks_per_probe = cum;
  a.stride = sl.stride;
  const int64_t total = cum * nprobe;       // one warp per block, 8 warps per CTA
  int64_t grid = (total + 7) / 8;
  if (grid > 16 * (int64_t)ctx->sm_count) grid = 16 * (int64_t)ctx->sm_count;
  perturb_small_kernel<<<(int)grid, 256, 0, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Vocabulary rows of the first layer's input: x[ps][v][:] = bf16(E'_ps[v][:])
// for every token v (the A operand of the vocabulary-table launch).
// ---------------------------------------------------------------------------
__global__ void vocab_x_kernel(const float* __restrict__ small_p, int64_t stride, int64_t offE,
                               int Bmax, int E, int V, int P, __nv_bfloat16* __restrict__ x) {
  const int e2 = E / 2;
  const int64_t total = (int64_t)P * V * e2;
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < total;
       k += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(k % e2);
    const int64_t pv = k / e2;
    const int v = (int)(pv % V);
    const int ps = (int)(pv / V);
    const float2 u =
        reinterpret_cast<const float2*>(small_p + ps * stride + offE + (int64_t)v * E)[c];
    reinterpret_cast<__nv_bfloat162*>(x + ((int64_t)ps * Bmax + v) * E)[c] =
        __floats2bfloat162_rn(u.x, u.y);
  }
}

// The cell epilogue's approximations (tanh.approx), so that t = 0 from the
// vocabulary table matches what the tensor-core epilogue computes.
__device__ __forceinline__ float tanh_ap(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float sigmoid_ap(float x) { return fmaf(0.5f, tanh_ap(0.5f * x), 0.5f); }

// Layer 0 at t = 0 from the vocabulary table: h_{-1} = c_{-1} = 0, so the
// pre-activations are the table row of the token plus the bias.
__global__ void vocab_first_kernel(const float* __restrict__ vt, int vtrows,
                                   const float* __restrict__ small_p, int64_t stride,
                                   int64_t offb, const int32_t* __restrict__ tokens, int T, int B,
                                   int Bmax, int H, int V, int P, float* __restrict__ cst,
                                   __nv_bfloat16* __restrict__ hout, unsigned* err) {
  const int64_t total = (int64_t)P * B * H;
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < total;
       k += (int64_t)gridDim.x * blockDim.x) {
    const int u = (int)(k % H);
    const int64_t pb = k / H;
    const int b = (int)(pb % B);
    const int ps = (int)(pb / B);
    int tok = tokens[(int64_t)b * T];
    if (tok < 0 || tok >= V) {
      latch(err, kErrBounds);
      tok = 0;
    }
    const float* tr = vt + ((int64_t)ps * vtrows + tok) * 4 * H;
    const float* bias = small_p + ps * stride + offb;
    const float ig = sigmoid_ap(tr[u] + bias[u]);
    const float gg = tanh_ap(tr[2 * H + u] + bias[2 * H + u]);
    const float og = sigmoid_ap(tr[3 * H + u] + bias[3 * H + u]);
    const float c = ig * gg;
    const int64_t o = ((int64_t)ps * Bmax + b) * H + u;
    cst[o] = c;   // row-major, as the table-fed layer's cell step reads it
    hout[o] = __float2bfloat16_rn(og * tanh_ap(c));
  }
}

cudaError_t launch_vocab_first(const zo_ctx* ctx, const int32_t* tokens, int B, int T, int nprobe,
                               cudaStream_t st) {
  const zo_model_spec& s = ctx->spec;
  const int P = 2 * nprobe, H = s.hidden;
  const int64_t total = (int64_t)P * B * H;
  int64_t grid = (total + 255) / 256;
  if (grid > (int64_t)ctx->sm_count * 16) grid = (int64_t)ctx->sm_count * 16;
  vocab_first_kernel<<<(int)grid, 256, 0, st>>>(ctx->vt, kVocabRows, ctx->small_p,
                                                ctx->small.stride, ctx->small.b[0], tokens, T, B,
                                                s.max_batch, H, s.vocab, P, ctx->cst,
                                                ctx->h /* layer 0, parity of t = 0 */, ctx->err);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_vocab_x(const zo_ctx* ctx, int nprobe, cudaStream_t st) {
  const zo_model_spec& s = ctx->spec;
  const int P = 2 * nprobe;
  const int64_t total = (int64_t)P * s.vocab * (s.embed / 2);
  int64_t grid = (total + 255) / 256;
  if (grid > (int64_t)ctx->sm_count * 16) grid = (int64_t)ctx->sm_count * 16;
  vocab_x_kernel<<<(int)grid, 256, 0, st>>>(ctx->small_p, ctx->small.stride, ctx->small.E,
                                            s.max_batch, s.embed, s.vocab, P, ctx->x);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// x_t[ps][b][:] = bf16(E_perturbed[ps][token[b, t]][:])  (first layer input)
// ---------------------------------------------------------------------------
__global__ void gather_x_kernel(const float* __restrict__ small_p, int64_t stride, int64_t offE,
                                const int32_t* __restrict__ tokens, int t, int B, int T, int Bmax,
                                int E, int V, int P, __nv_bfloat16* __restrict__ x,
                                unsigned* err) {
  const int e8 = E / 8;
  const int64_t total = (int64_t)P * B * e8;
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < total;
       k += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(k % e8);
    const int64_t pb = k / e8;
    const int b = (int)(pb % B);
    const int ps = (int)(pb / B);
    int tok = tokens[(int64_t)b * T + t];
    if (tok < 0 || tok >= V) {
      latch(err, kErrBounds);
      tok = 0;
    }
    const float4* src = reinterpret_cast<const float4*>(small_p + ps * stride + offE +
                                                        (int64_t)tok * E + 8 * c);
    const float4 u = src[0], v = src[1];
    __nv_bfloat162 q0 = __floats2bfloat162_rn(u.x, u.y), q1 = __floats2bfloat162_rn(u.z, u.w);
    __nv_bfloat162 q2 = __floats2bfloat162_rn(v.x, v.y), q3 = __floats2bfloat162_rn(v.z, v.w);
    uint4 o;
    o.x = *reinterpret_cast<uint32_t*>(&q0);
    o.y = *reinterpret_cast<uint32_t*>(&q1);
    o.z = *reinterpret_cast<uint32_t*>(&q2);
    o.w = *reinterpret_cast<uint32_t*>(&q3);
    reinterpret_cast<uint4*>(x + ((int64_t)ps * Bmax + b) * E)[c] = o;
  }
}

cudaError_t launch_gather_x(const zo_ctx* ctx, const int32_t* tokens, int t, int B, int T,
                            int nprobe, cudaStream_t st) {
  const int E = ctx->spec.embed;
  const int P = 2 * nprobe;
  const int64_t total = (int64_t)P * B * (E / 8);
  int64_t grid = (total + 255) / 256;
  if (grid > (int64_t)ctx->sm_count * 16) grid = (int64_t)ctx->sm_count * 16;
  gather_x_kernel<<<(int)grid, 256, 0, st>>>(ctx->small_p, ctx->small.stride, ctx->small.E,
                                             tokens, t, B, T, ctx->spec.max_batch, E,
                                             ctx->spec.vocab, P, ctx->x, ctx->err);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// L[ps] = sum_b rowloss[ps][b] / #scored; fixed-order tree reduction, one CTA
// per probe-sign.  Also copies the row sums out when asked.
// ---------------------------------------------------------------------------
__global__ void reduce_losses_kernel(const float* __restrict__ rowloss, int Bmax,
                                     const int32_t* __restrict__ targets, int B, int T, int V,
                                     int probe0, float* lp, float* lm, float* row_out,
                                     unsigned* err) {
  __shared__ double ssum[256];
  __shared__ int scount[256];
  const int ps = blockIdx.x;
  double s = 0.0;
  int cnt = 0;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const float v = rowloss[(int64_t)ps * Bmax + b];
    s += v;
    if (row_out) row_out[((int64_t)(2 * probe0) + ps) * B + b] = v;
  }
  for (int64_t k = threadIdx.x; k < (int64_t)B * T; k += blockDim.x) {
    const int tg = targets[k];
    cnt += (tg >= 0 && tg < V);
  }
  ssum[threadIdx.x] = s;
  scount[threadIdx.x] = cnt;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      ssum[threadIdx.x] += ssum[threadIdx.x + w];
      scount[threadIdx.x] += scount[threadIdx.x + w];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int n = scount[0];
    const float L = n > 0 ? (float)(ssum[0] / n) : 0.f;
    if (!isfinite(L)) latch(err, kErrNonfinite);
    const int i = probe0 + ps / 2;
    if (ps & 1)
      lm[i] = L;
    else
      lp[i] = L;
  }
}

cudaError_t launch_reduce_losses(const zo_ctx* ctx, const int32_t* targets, int B, int T,
                                 int probe0, int nprobe, float* lp, float* lm, float* row_out,
                                 cudaStream_t st) {
  reduce_losses_kernel<<<2 * nprobe, 256, 0, st>>>(ctx->rowloss, ctx->spec.max_batch, targets, B,
                                                   T, ctx->spec.vocab, probe0, lp, lm, row_out,
                                                   ctx->err);
  count_launch();
  return cudaGetLastError();
}

}  // namespace zo
