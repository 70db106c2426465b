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

__device__ __forceinline__ float2 fma_f32x2(float2 a, float2 b, float2 c) {
  unsigned long long ar = *reinterpret_cast<unsigned long long*>(&a);
  unsigned long long br = *reinterpret_cast<unsigned long long*>(&b);
  unsigned long long cr = *reinterpret_cast<unsigned long long*>(&c);
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(ar), "l"(br), "l"(cr));
  return *reinterpret_cast<float2*>(&r);
}

__device__ __forceinline__ float2 add_f32x2(float2 a, float2 b) {
  unsigned long long ar = *reinterpret_cast<unsigned long long*>(&a);
  unsigned long long br = *reinterpret_cast<unsigned long long*>(&b);
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(ar), "l"(br));
  return *reinterpret_cast<float2*>(&r);
}

// Subset-sum tables for the probe term.  For the concatenated input
// a = [in | rec] of one step and every group g of 4 inputs (k = 4g..4g+3),
//   U[b][g][idx] = ( sum_k p_k a+_k,  -sum_k p_k a-_k )  over the group,
// where p_k = -1 for the elements whose bit is set in the 4-bit index idx
// (bit 0 <-> k = 4g, bit 1 <-> 4g+2, bit 2 <-> 4g+1, bit 3 <-> 4g+3: the order
// in which a sign word, shifted to the group, holds them at bits 0, 1, 16, 17).
// Then sum_k p_k a_k over a row is one table lookup per group.
constexpr int kUStride = 17;  // float2 per group (16 + 1 pad against bank conflicts)

template <int BB>
__device__ void build_tables(const float* in, int Kin, const float* rec, int Krec, float2* U) {
  const int G = (Kin + Krec) / 4;
  for (int e = threadIdx.x; e < BB * G * 16; e += blockDim.x) {
    const int idx = e & 15;
    const int g = (e >> 4) % G;
    const int b = (e >> 4) / G;
    const int k = 4 * g;
    float4 xp, xm;
    if (k < Kin) {
      xp = *reinterpret_cast<const float4*>(in + b * Kin + k);
      xm = *reinterpret_cast<const float4*>(in + (BB + b) * Kin + k);
    } else {
      xp = *reinterpret_cast<const float4*>(rec + b * Krec + k - Kin);
      xm = *reinterpret_cast<const float4*>(rec + (BB + b) * Krec + k - Kin);
    }
    const float s0 = (idx & 1) ? -1.f : 1.f, s2 = (idx & 2) ? -1.f : 1.f;
    const float s1 = (idx & 4) ? -1.f : 1.f, s3 = (idx & 8) ? -1.f : 1.f;
    const float up = s0 * xp.x + s1 * xp.y + s2 * xp.z + s3 * xp.w;
    const float um = s0 * xm.x + s1 * xm.y + s2 * xm.z + s3 * xm.w;
    U[(b * G + g) * kUStride + idx] = make_float2(up, -um);
  }
}

// Rows [0, R) of a perturbed matrix-vector product for BB batch rows and both
// signs.  Row r of the matrix starts at theta[j0 + r*K]; its first Kin entries
// multiply `in` ([2][BB][Kin] in shared memory) and the rest `rec`
// ([2][BB][K-Kin]).  out[s][b][r] = bias_s[r] + sum_k (W +- eps P)[r,k] a_s[b,k].
//
// VEC (rows and both parts 4-aligned): a lane is (k-slice l8 = lane & 7,
// row slot rs = lane >> 3) and owns rows rb + rs + 4m, m < RPL (2 when BB = 1,
// else 1); it walks the
// groups g = l8 + 8i of 4 inputs, loads the group's activations once and uses
// them for all its rows: W a+- with packed fp32x2 FMAs on (even, odd) pairs,
// eps P a+- from the subset-sum tables U.  Weight loads stay coalesced (8
// lanes x 16 B of one row).
// Otherwise: 8 lanes per row, one element per step, W +- eps p formed directly.
template <int BB, bool VEC>
__device__ void perturbed_gemv(const Fp32Args& a, const uint32_t* sw, int64_t j0, int R, int K,
                               int Kin, const float* in, const float* rec, const float2* U,
                               int64_t jbias, float* out, int out_stride) {
  constexpr int RPL = (VEC && BB == 1) ? 2 : 1;   // rows per lane
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  const int l8 = lane & 7;
  const int Krec = K - Kin;
  const float eps = a.eps;
  for (int rb = warp * 4 * RPL; rb < R; rb += nw * 4 * RPL) {
    float gp[RPL][BB], gm[RPL][BB];
    if (VEC) {
      const int G = K / 4, Gin = Kin / 4;
      float2 wp[RPL][BB], wm[RPL][BB], pe[RPL][BB];
      // row m of this lane: weights at wbase + roff[m] (float4 units), sign
      // word index wi[m] (+1 per step of 32 inputs), in-word shift sh[m]
      const float4* wbase = reinterpret_cast<const float4*>(a.theta + j0 + 4 * l8);
      int roff[RPL], wi[RPL], sh[RPL];
#pragma unroll
      for (int m = 0; m < RPL; ++m) {
        const int r = rb + (lane >> 3) + 4 * m;
        const int rr = r < R ? r : 0;
        roff[m] = rr * (K / 4);
        const int64_t jl = j0 + (int64_t)rr * K + 4 * l8;
        wi[m] = (int)(jl >> 5);
        sh[m] = (int)(jl & 31) >> 1;
#pragma unroll
        for (int b = 0; b < BB; ++b) wp[m][b] = wm[m][b] = pe[m][b] = make_float2(0.f, 0.f);
      }
      for (int g = l8; g < G; g += 8) {
        float4 xp[BB], xm[BB];
#pragma unroll
        for (int b = 0; b < BB; ++b) {
          const float* src = g < Gin ? in + b * Kin + 4 * g : rec + b * Krec + 4 * g - Kin;
          const int off = g < Gin ? BB * Kin : BB * Krec;
          xp[b] = *reinterpret_cast<const float4*>(src);
          xm[b] = *reinterpret_cast<const float4*>(src + off);
        }
#pragma unroll
        for (int m = 0; m < RPL; ++m) {
          const float4 w = __ldg(wbase + roff[m] + (g - l8));
          const uint32_t s = sw[wi[m] + ((g - l8) >> 3)] >> sh[m];
          const int idx = (int)((s & 3u) | ((s >> 14) & 12u));
#pragma unroll
          for (int b = 0; b < BB; ++b) {
            wp[m][b] = fma_f32x2(make_float2(w.x, w.y), make_float2(xp[b].x, xp[b].y), wp[m][b]);
            wp[m][b] = fma_f32x2(make_float2(w.z, w.w), make_float2(xp[b].z, xp[b].w), wp[m][b]);
            wm[m][b] = fma_f32x2(make_float2(w.x, w.y), make_float2(xm[b].x, xm[b].y), wm[m][b]);
            wm[m][b] = fma_f32x2(make_float2(w.z, w.w), make_float2(xm[b].z, xm[b].w), wm[m][b]);
            pe[m][b] = add_f32x2(pe[m][b], U[(b * G + g) * kUStride + idx]);
          }
        }
      }
#pragma unroll
      for (int m = 0; m < RPL; ++m)
#pragma unroll
        for (int b = 0; b < BB; ++b) {
          gp[m][b] = fmaf(eps, pe[m][b].x, wp[m][b].x + wp[m][b].y);
          gm[m][b] = fmaf(eps, pe[m][b].y, wm[m][b].x + wm[m][b].y);
        }
    } else {
      const int r = rb + (lane >> 3);
      const int64_t jr = j0 + (int64_t)(r < R ? r : 0) * K;
#pragma unroll
      for (int b = 0; b < BB; ++b) gp[0][b] = gm[0][b] = 0.f;
      if (r < R) {
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
            gp[0][b] = fmaf(w + d, src[b * ld + kk], gp[0][b]);
            gm[0][b] = fmaf(w - d, src[(BB + b) * ld + kk], gm[0][b]);
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < RPL; ++m) {
#pragma unroll
      for (int b = 0; b < BB; ++b) {
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) {
          gp[m][b] += __shfl_xor_sync(0xffffffffu, gp[m][b], o);
          gm[m][b] += __shfl_xor_sync(0xffffffffu, gm[m][b], o);
        }
      }
      const int r = rb + (lane >> 3) + 4 * m;
      if (r < R && l8 == 0) {
        const float bth = a.theta[jbias + r];
        const float bd = pert(sw, jbias + r, eps);
#pragma unroll
        for (int b = 0; b < BB; ++b) {
          out[b * out_stride + r] = gp[m][b] + (bth + bd);
          out[(BB + b) * out_stride + r] = gm[m][b] + (bth - bd);
        }
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
  float2* U = reinterpret_cast<float2*>(rl + ((2 * BB + 3) & ~3));  // [BB][Gmax][17] (VEC)
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
      if (VEC) {
        build_tables<BB>(inp, in_l, hl, H, U);
        __syncthreads();
      }
      perturbed_gemv<BB, VEC>(a, sw, a.offW[l], G4, in_l + H, in_l, inp, hl, U, a.offB[l], gs, G4);
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
    if (VEC) {
      build_tables<BB>(htop, H, htop, 0, U);
      __syncthreads();
    }
    perturbed_gemv<BB, VEC>(a, sw, a.offWout, V, H, H, htop, htop, U, a.offBout, lg, V);
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
  const size_t gmax = ((E > H ? E : H) + H) / 4;   // groups of the widest step input
  const size_t ufloats = (E % 4 == 0 && H % 4 == 0) ? 2 * bb * gmax * kUStride : 0;
  return (size_t)(d_pad / 8) +
         sizeof(float) * (2 * bb * E + 4 * L * bb * H + 2 * bb * 4 * H + 2 * bb * V +
                          ((2 * bb + 3) & ~3) + ufloats);
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
  // rows per CTA: the context's maximum, halved while probes x row blocks
  // leave SMs idle (a CTA's shared memory shrinks with its rows)
  int bb = ctx->fp32_bb;
  while (bb > 1 && (int64_t)nprobe * ((B + bb - 1) / bb) < ctx->sm_count) bb /= 2;
  const size_t smem = fp32_smem_bytes(ctx->spec, bb, s.d_pad);
  return vec ? launch_fp32_vec<true>(a, bb, nprobe, smem, st)
             : launch_fp32_vec<false>(a, bb, nprobe, smem, st);
}

}  // namespace zo
