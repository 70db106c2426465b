// fp32 CUDA-core path for small models: one persistent CTA runs the whole
// sequence for one probe (both signs) and a slice of the batch, with the
// recurrent state in shared memory and the perturbed weights W +- eps P
// formed on the fly from theta and the probe's Philox words.  Every cell
// step is G = [x_t | h_{t-1}] (W +- eps P)^T + (b +- eps p),
// c_t = sigma(f) c_{t-1} + sigma(i) tanh(g), h_t = sigma(o) tanh(c_t)
// (pith.science review, "What carries the argument": complete forwards at
// Theta +- eps p_i; cell and loss readings in the oracle's header).
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
  int64_t offE, offW[kMaxLayers], offB[kMaxLayers], offWout, offBout;
  float* rowloss;  // [2*nprobe][Bmax]
  unsigned* err;
};

// dot products of one weight row (K entries starting at theta[j0]) with the
// + and - activations of BB rows; the sign words are refreshed per 128-block.
template <int BB>
__device__ __forceinline__ void perturbed_row_dot(const Fp32Args& a, uint32_t probe, int64_t j0,
                                                  int K, const float* __restrict__ ap, int lda,
                                                  const float* __restrict__ am,
                                                  float (&accp)[BB], float (&accm)[BB]) {
  int64_t cur_q = -1;
  uint4 w = make_uint4(0, 0, 0, 0);
  for (int k = 0; k < K; ++k) {
    const int64_t j = j0 + k;
    const int64_t q = j >> 7;
    if (q != cur_q) {
      w = sign_block(a.seed, probe, (uint64_t)q);
      cur_q = q;
    }
    const float d = sign_bit(w, j) ? -a.eps : a.eps;
    const float th = __ldg(a.theta + j);
    const float wp = th + d, wm = th - d;
#pragma unroll
    for (int b = 0; b < BB; ++b) {
      accp[b] = fmaf(wp, ap[b * lda + k], accp[b]);
      accm[b] = fmaf(wm, am[b * lda + k], accm[b]);
    }
  }
}

template <int BB>
__global__ void fp32_forward_kernel(const Fp32Args a) {
  extern __shared__ float sm[];
  const int ci = blockIdx.x;
  const uint32_t probe = (uint32_t)(a.probe0 + ci);
  const int r0 = blockIdx.y * BB;
  const int nb = min(BB, a.B - r0);
  const int H = a.H, E = a.E, V = a.V, L = a.L;
  const int G4 = 4 * H;
  const int tid = threadIdx.x, nt = blockDim.x;
  float* xin = sm;                       // [2][BB][E]
  float* hs = xin + 2 * BB * E;          // [L][2][BB][H]
  float* cs = hs + L * 2 * BB * H;       // [L][2][BB][H]
  float* gs = cs + L * 2 * BB * H;       // [2][BB][4H]
  float* lg = gs + 2 * BB * G4;          // [2][BB][V]
  float* rl = lg + 2 * BB * V;           // [2][BB]
  for (int i = tid; i < 2 * L * 2 * BB * H + 2 * BB; i += nt) {
    if (i < 2 * L * 2 * BB * H)
      hs[i] = 0.f;  // hs and cs are contiguous
    else
      rl[i - 2 * L * 2 * BB * H] = 0.f;
  }
  __syncthreads();

  for (int t = 0; t < a.T; ++t) {
    // perturbed embedding rows
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
        const float d = sign_at(a.seed, probe, j) * a.eps;
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
      const int K = in_l + H;
      const float* inp = l == 0 ? xin : hs + (l - 1) * 2 * BB * H;  // [2][BB][in_l]
      float* hl = hs + l * 2 * BB * H;
      float* cl = cs + l * 2 * BB * H;
      for (int r = tid; r < G4; r += nt) {
        float accp[BB], accm[BB];
        {
          const int64_t jb = a.offB[l] + r;
          const float d = sign_at(a.seed, probe, jb) * a.eps;
          const float th = a.theta[jb];
#pragma unroll
          for (int b = 0; b < BB; ++b) {
            accp[b] = th + d;
            accm[b] = th - d;
          }
        }
        const int64_t jr = a.offW[l] + (int64_t)r * K;
        perturbed_row_dot<BB>(a, probe, jr, in_l, inp, in_l, inp + BB * in_l, accp, accm);
        perturbed_row_dot<BB>(a, probe, jr + in_l, H, hl, H, hl + BB * H, accp, accm);
#pragma unroll
        for (int b = 0; b < BB; ++b) {
          gs[b * G4 + r] = accp[b];
          gs[BB * G4 + b * G4 + r] = accm[b];
        }
      }
      __syncthreads();
      for (int i = tid; i < 2 * BB * H; i += nt) {
        const int sb = i / H, u = i % H;  // sb = s * BB + b
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
    // output projection
    const float* htop = hs + (L - 1) * 2 * BB * H;
    for (int v = tid; v < V; v += nt) {
      float accp[BB], accm[BB];
      {
        const int64_t jb = a.offBout + v;
        const float d = sign_at(a.seed, probe, jb) * a.eps;
        const float th = a.theta[jb];
#pragma unroll
        for (int b = 0; b < BB; ++b) {
          accp[b] = th + d;
          accm[b] = th - d;
        }
      }
      perturbed_row_dot<BB>(a, probe, a.offWout + (int64_t)v * H, H, htop, H, htop + BB * H,
                            accp, accm);
#pragma unroll
      for (int b = 0; b < BB; ++b) {
        lg[b * V + v] = accp[b];
        lg[BB * V + b * V + v] = accm[b];
      }
    }
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

size_t fp32_smem_bytes(const zo_model_spec& s, int bb) {
  const size_t E = s.embed, H = s.hidden, V = s.vocab, L = s.layers;
  return sizeof(float) * (2 * bb * E + 4 * L * bb * H + 2 * bb * 4 * H + 2 * bb * V + 2 * bb);
}

template <int BB>
static cudaError_t launch_fp32_bb(const Fp32Args& a, int nprobe, size_t smem, cudaStream_t st) {
  cudaFuncSetAttribute(fp32_forward_kernel<BB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)smem);
  int threads = 4 * a.H;
  threads = ((threads + 31) / 32) * 32;
  if (threads > 512) threads = 512;
  if (threads < 64) threads = 64;
  dim3 grid(nprobe, (a.B + BB - 1) / BB);
  fp32_forward_kernel<BB><<<grid, threads, smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
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
  a.offE = s.off[s.E];
  for (int l = 0; l < a.L; ++l) {
    a.offW[l] = s.off[s.W[l]];
    a.offB[l] = s.off[s.b[l]];
  }
  a.offWout = s.off[s.Wout];
  a.offBout = s.off[s.bout];
  a.rowloss = ctx->rowloss;
  a.err = ctx->err;
  const size_t smem = ctx->fp32_smem;
  switch (ctx->fp32_bb) {
    case 1: return launch_fp32_bb<1>(a, nprobe, smem, st);
    case 2: return launch_fp32_bb<2>(a, nprobe, smem, st);
    case 4: return launch_fp32_bb<4>(a, nprobe, smem, st);
    default: return launch_fp32_bb<8>(a, nprobe, smem, st);
  }
}

}  // namespace zo
