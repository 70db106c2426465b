// fp32 CUDA-core path for small models: one persistent CTA runs the whole
// sequence for one probe (both signs) and a slice of the batch, with the
// recurrent state in shared memory and the perturbed weights W +- eps P
// formed on the fly.  Every cell step is
//   G = [x_t | h_{t-1}] (W +- eps P)^T + (b +- eps p),
//   c_t = sigma(f) c_{t-1} + sigma(i) tanh(g),  h_t = sigma(o) tanh(c_t)
// (pith.science review, "What carries the argument": complete forwards at
// Theta +- eps p_i; cell and loss readings in the oracle's header).
//
// The probe's sign words for the whole parameter vector (d/8 bytes) are
// generated once per CTA into shared memory, so the timestep loop runs no
// Philox at all.  Weight rows are read by groups of 8 lanes (float4 each,
// 128 contiguous bytes per row), so every global load is coalesced; the two
// signs share each weight load and each sign word.
#include "zo_common.cuh"
#include "zo_internal.h"

namespace zo {

struct Fp32Args {
  const float* theta;
  uint64_t seed;
  int probe0;
  float eps;
  const int32_t* tokens;
  const int32_t* targets;
  int B, T, Bmax;
  int V, E, H, L;
  int64_t nblk;    // d_pad / 128
  int64_t offE, offW[kMaxLayers], offB[kMaxLayers], offWout, offBout;
  float* rowloss;  // [2*nprobe][Bmax]
  unsigned* err;
};

constexpr int kFpThreads = 256;

// Signed perturbation +-eps for element j from the shared sign words.
__device__ __forceinline__ float pert(const uint32_t* sw, int64_t j, float eps) {
  const uint32_t w = sw[j >> 5];
  const int e = (int)(j & 31);
  return flip_sign(eps, (w >> bit_pos(e)) << 31);
}

// Rows [0, R) of a perturbed matrix-vector product for BB batch rows and both
// signs.  Row r of the matrix starts at theta[j0 + r*K]; its first Kin entries
// multiply `in` ([2][BB][Kin] in shared memory) and the rest `rec`
// ([2][BB][K-Kin]).  out[s][b][r] = bias_s[r] + sum_k (W +- eps P)[r,k] a_s[b,k].
// 8 lanes per row, 4 rows per warp.  VEC: rows and both parts are 4-aligned.
template <int BB, bool VEC>
__device__ void perturbed_gemv(const Fp32Args& a, const uint32_t* sw, int64_t j0, int R, int K,
                               int Kin, const float* in, const float* rec, int64_t jbias,
                               float* out, int out_stride) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  const int l8 = lane & 7;
  const int Krec = K - Kin;
  const float eps = a.eps;
  for (int rb = warp * 4; rb < R; rb += nw * 4) {
    const int r = rb + (lane >> 3);
    const bool live = r < R;
    const int64_t jr = j0 + (int64_t)(live ? r : 0) * K;
    float ap[BB], am[BB];
#pragma unroll
    for (int b = 0; b < BB; ++b) ap[b] = am[b] = 0.f;
    if (live) {
      if (VEC) {
        for (int k = 4 * l8; k < K; k += 32) {
          const float4 w = __ldg(reinterpret_cast<const float4*>(a.theta + jr + k));
          const int64_t j = jr + k;
          const uint32_t s = sw[j >> 5] >> ((int)(j & 31) >> 1);
          const float d0 = flip_sign(eps, s << 31), d1 = flip_sign(eps, s << 15);
          const float d2 = flip_sign(eps, s << 30), d3 = flip_sign(eps, s << 14);
          const float* src;
          int ld, kk;
          if (k < Kin) {
            src = in;
            ld = Kin;
            kk = k;
          } else {
            src = rec;
            ld = Krec;
            kk = k - Kin;
          }
#pragma unroll
          for (int b = 0; b < BB; ++b) {
            const float4 xp = *reinterpret_cast<const float4*>(src + b * ld + kk);
            const float4 xm = *reinterpret_cast<const float4*>(src + (BB + b) * ld + kk);
            ap[b] = fmaf(w.x + d0, xp.x, ap[b]);
            ap[b] = fmaf(w.y + d1, xp.y, ap[b]);
            ap[b] = fmaf(w.z + d2, xp.z, ap[b]);
            ap[b] = fmaf(w.w + d3, xp.w, ap[b]);
            am[b] = fmaf(w.x - d0, xm.x, am[b]);
            am[b] = fmaf(w.y - d1, xm.y, am[b]);
            am[b] = fmaf(w.z - d2, xm.z, am[b]);
            am[b] = fmaf(w.w - d3, xm.w, am[b]);
          }
        }
      } else {
        for (int k = l8; k < K; k += 8) {
          const float w = __ldg(a.theta + jr + k);
          const float d = pert(sw, jr + k, eps);
          const float* src;
          int ld, kk;
          if (k < Kin) {
            src = in;
            ld = Kin;
            kk = k;
          } else {
            src = rec;
            ld = Krec;
            kk = k - Kin;
          }
#pragma unroll
          for (int b = 0; b < BB; ++b) {
            ap[b] = fmaf(w + d, src[b * ld + kk], ap[b]);
            am[b] = fmaf(w - d, src[(BB + b) * ld + kk], am[b]);
          }
        }
      }
    }
#pragma unroll
    for (int b = 0; b < BB; ++b) {
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) {
        ap[b] += __shfl_xor_sync(0xffffffffu, ap[b], o);
        am[b] += __shfl_xor_sync(0xffffffffu, am[b], o);
      }
    }
    if (live && l8 == 0) {
      const float bth = a.theta[jbias + r];
      const float bd = pert(sw, jbias + r, eps);
#pragma unroll
      for (int b = 0; b < BB; ++b) {
        out[b * out_stride + r] = ap[b] + (bth + bd);
        out[(BB + b) * out_stride + r] = am[b] + (bth - bd);
      }
    }
  }
}

template <int BB, bool VEC>
__global__ void __launch_bounds__(kFpThreads, BB <= 2 ? 4 : 2) fp32_forward_kernel(const Fp32Args a) {
  extern __shared__ __align__(16) float sm[];
  const int ci = blockIdx.x;
  const uint32_t probe = (uint32_t)(a.probe0 + ci);
  const int r0 = blockIdx.y * BB;
  const int nb = min(BB, a.B - r0);
  const int H = a.H, E = a.E, V = a.V, L = a.L;
  const int G4 = 4 * H;
  const int tid = threadIdx.x, nt = blockDim.x;
  uint32_t* sw = reinterpret_cast<uint32_t*>(sm);        // [nblk*4] sign words
  float* xin = sm + a.nblk * 4;                            // [2][BB][E]
  float* hs = xin + 2 * BB * E;                            // [L][2][BB][H]
  float* cs = hs + L * 2 * BB * H;                         // [L][2][BB][H]
  float* gs = cs + L * 2 * BB * H;                         // [2][BB][4H]
  float* lg = gs + 2 * BB * G4;                            // [2][BB][V]
  float* rl = lg + 2 * BB * V;                             // [2][BB]
  for (int64_t q = tid; q < a.nblk; q += nt)
    reinterpret_cast<uint4*>(sw)[q] = sign_block(a.seed, probe, (uint64_t)q);
  for (int i = tid; i < 2 * L * 2 * BB * H; i += nt) hs[i] = 0.f;  // hs, cs
  for (int i = tid; i < 2 * BB; i += nt) rl[i] = 0.f;
  __syncthreads();

  for (int t = 0; t < a.T; ++t) {
    for (int i = tid; i < BB * E; i += nt) {
      const int b = i / E, k = i % E;
      float vp = 0.f, vm = 0.f;
      if (b < nb) {
        int tok = a.tokens[(int64_t)(r0 + b) * a.T + t];
        if (tok < 0 || tok >= V) {
          latch(a.err, kErrBounds);
          tok = 0;
        }
        const int64_t j = a.offE + (int64_t)tok * E + k;
        const float d = pert(sw, j, a.eps);
        const float th = a.theta[j];
        vp = th + d;
        vm = th - d;
      }
      xin[b * E + k] = vp;
      xin[BB * E + b * E + k] = vm;
    }
    __syncthreads();
    for (int l = 0; l < L; ++l) {
      const int in_l = l == 0 ? E : H;
      const float* inp = l == 0 ? xin : hs + (l - 1) * 2 * BB * H;
      float* hl = hs + l * 2 * BB * H;
      float* cl = cs + l * 2 * BB * H;
      perturbed_gemv<BB, VEC>(a, sw, a.offW[l], G4, in_l + H, in_l, inp, hl, a.offB[l], gs, G4);
      __syncthreads();
      for (int i = tid; i < 2 * BB * H; i += nt) {
        const int sb = i / H, u = i % H;
        const float* G = gs + sb * G4;
        const float ig = sigmoid_acc(G[u]);
        const float fg = sigmoid_acc(G[H + u]);
        const float gg = tanhf(G[2 * H + u]);
        const float og = sigmoid_acc(G[3 * H + u]);
        const float c = fg * cl[sb * H + u] + ig * gg;
        cl[sb * H + u] = c;
        hl[sb * H + u] = og * tanhf(c);
      }
      __syncthreads();
    }
    const float* htop = hs + (L - 1) * 2 * BB * H;
    perturbed_gemv<BB, VEC>(a, sw, a.offWout, V, H, H, htop, htop, a.offBout, lg, V);
    __syncthreads();
    for (int i = tid; i < 2 * BB; i += nt) {
      const int b = i % BB;
      if (b < nb) {
        int tg = a.targets[(int64_t)(r0 + b) * a.T + t];
        if (tg >= V || tg < -1) {
          latch(a.err, kErrBounds);
          tg = -1;
        }
        if (tg >= 0) {
          const float* z = lg + i * V;
          float m = -INFINITY;
          for (int v = 0; v < V; ++v) m = fmaxf(m, z[v]);
          float s = 0.f;
          for (int v = 0; v < V; ++v) s += expf(z[v] - m);
          rl[i] += m + logf(s) - z[tg];
        }
      }
    }
    __syncthreads();
  }
  for (int i = tid; i < 2 * BB; i += nt) {
    const int s = i / BB, b = i % BB;
    if (b < nb) a.rowloss[(int64_t)(2 * ci + s) * a.Bmax + r0 + b] = rl[i];
  }
}

size_t fp32_smem_bytes(const zo_model_spec& s, int bb, int64_t d_pad) {
  const size_t E = s.embed, H = s.hidden, V = s.vocab, L = s.layers;
  return (size_t)(d_pad / 8) +
         sizeof(float) * (2 * bb * E + 4 * L * bb * H + 2 * bb * 4 * H + 2 * bb * V + 2 * bb);
}

template <int BB, bool VEC>
static cudaError_t launch_fp32_bb(const Fp32Args& a, int nprobe, size_t smem, cudaStream_t st) {
  cudaFuncSetAttribute(fp32_forward_kernel<BB, VEC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)smem);
  // ask for the largest shared-memory carveout so several CTAs share an SM
  cudaFuncSetAttribute(fp32_forward_kernel<BB, VEC>,
                       cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  int threads = 4 * a.H * 8 / 4;  // 8 lanes per row, 4 rows per warp
  threads = ((threads + 31) / 32) * 32;
  if (threads > kFpThreads) threads = kFpThreads;
  if (threads < 128) threads = 128;
  dim3 grid(nprobe, (a.B + BB - 1) / BB);
  fp32_forward_kernel<BB, VEC><<<grid, threads, smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

template <bool VEC>
static cudaError_t launch_fp32_vec(const Fp32Args& a, int bb, int nprobe, size_t smem,
                                   cudaStream_t st) {
  switch (bb) {
    case 1: return launch_fp32_bb<1, VEC>(a, nprobe, smem, st);
    case 2: return launch_fp32_bb<2, VEC>(a, nprobe, smem, st);
    case 4: return launch_fp32_bb<4, VEC>(a, nprobe, smem, st);
    default: return launch_fp32_bb<8, VEC>(a, nprobe, smem, st);
  }
}

cudaError_t launch_fp32_forward(const zo_ctx* ctx, const float* theta, uint64_t seed, int probe0,
                                int nprobe, float eps, const int32_t* tokens,
                                const int32_t* targets, int B, int T, cudaStream_t st) {
  const Segments& s = ctx->seg;
  Fp32Args a;
  a.theta = theta;
  a.seed = seed;
  a.probe0 = probe0;
  a.eps = eps;
  a.tokens = tokens;
  a.targets = targets;
  a.B = B;
  a.T = T;
  a.Bmax = ctx->spec.max_batch;
  a.V = ctx->spec.vocab;
  a.E = ctx->spec.embed;
  a.H = ctx->spec.hidden;
  a.L = ctx->spec.layers;
  a.nblk = s.d_pad / 128;
  a.offE = s.off[s.E];
  for (int l = 0; l < a.L; ++l) {
    a.offW[l] = s.off[s.W[l]];
    a.offB[l] = s.off[s.b[l]];
  }
  a.offWout = s.off[s.Wout];
  a.offBout = s.off[s.bout];
  a.rowloss = ctx->rowloss;
  a.err = ctx->err;
  const bool vec = (a.E % 4 == 0) && (a.H % 4 == 0);
  return vec ? launch_fp32_vec<true>(a, ctx->fp32_bb, nprobe, ctx->fp32_smem, st)
             : launch_fp32_vec<false>(a, ctx->fp32_bb, nprobe, ctx->fp32_smem, st);
}

}  // namespace zo
