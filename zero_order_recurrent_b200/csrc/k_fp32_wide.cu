// fp32 CUDA-core forward with the probes across columns: one CTA runs the
// whole sequence of one batch row for NP probes, i.e. NC = 2 NP probe-sign
// columns (column 2p + s: probe p, sign + for s = 0, - for s = 1).  Every cell
// step is
//   G = [x_t | h_{t-1}] (W +- eps P)^T + (b +- eps p),
//   c_t = sigma(f) c_{t-1} + sigma(i) tanh(g),  h_t = sigma(o) tanh(c_t)
// (pith.science review, "What carries the argument": complete forwards at
// Theta +- eps p_i), evaluated as W a + eps (P a) per column:
//
//  * W a: lane L of a warp owns two adjacent rows of a 64-row block and walks
//    the inputs in steps of 32; each weight (read from a transposed copy of W,
//    so a warp's loads are one coalesced 256-byte row) feeds all NC columns
//    with packed fp32x2 FMAs, and the activations are shared-memory
//    broadcasts.  When a matrix has fewer row blocks than warps, the inputs
//    are split over warps and the partial sums added in shared memory.
//  * eps P a: subset-sum tables.  The inputs k = 8v + par + 2i (i < 4) of one
//    8-input block and parity par form a group; their signs sit in one nibble
//    of a sign word (elements 2m and 2m+1 are bits m and m+16), so a group's
//    4-bit pattern is a shift and a mask, and one lookup in that group's
//    16-entry table of signed sums replaces four sign applications.
//
// The probes' sign words are generated once per CTA (Philox) into shared
// memory, the weight-matrix words transposed to [input word][row] so that a
// warp reads its rows' words without bank conflicts; the timestep loop runs
// no Philox.
#include "zo_common.cuh"
#include "zo_internal.h"

namespace zo {

constexpr int kWideThreads = 256;
constexpr int kWideWarps = kWideThreads / 32;

struct WideMat {
  const float* wt;   // W^T [K][Rp], rows past R are zero
  int R, Rp, K, Kin; // rows, rows rounded up to 64, inputs, inputs from the first operand
  int64_t off;       // theta offset of W (row-major [R][K])
  int64_t offb;      // theta offset of the bias (R entries)
  int sw;            // word offset of W in a probe's transposed words ([K/32][Rp])
  int sb;            // word offset of the bias in a probe's small-segment words
};

struct WideArgs {
  const float* theta;
  uint64_t seed;
  int probe0, nprobe;
  float eps;
  const int32_t* tokens;
  const int32_t* targets;
  int B, T, Bmax;
  int V, E, H, L;
  int64_t offE;
  int sE;                          // word offset of E in the small-segment words
  WideMat m[kMaxLayers + 1];       // cells 0..L-1, then the output layer
  int nsmall;                      // small segments: E, b_0..b_{L-1}, b_out
  int64_t small_off[kMaxSeg], small_num[kMaxSeg];
  int small_base[kMaxSeg];
  int sw_words, small_words;       // per probe
  int gmax;                        // table groups of the widest matrix (K/4)
  int rmax;                        // rows of the gate / logit buffer
  int pmax;                        // floats of the partial-sum buffer
  float* rowloss;                  // [2*nprobe][Bmax]
  unsigned* err;
};

__device__ __forceinline__ float2 wfma2(float2 a, float2 b, float2 c) {
  unsigned long long ar = *reinterpret_cast<unsigned long long*>(&a);
  unsigned long long br = *reinterpret_cast<unsigned long long*>(&b);
  unsigned long long cr = *reinterpret_cast<unsigned long long*>(&c);
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(ar), "l"(br), "l"(cr));
  return *reinterpret_cast<float2*>(&r);
}

__device__ __forceinline__ float2 wadd2(float2 a, float2 b) {
  unsigned long long ar = *reinterpret_cast<unsigned long long*>(&a);
  unsigned long long br = *reinterpret_cast<unsigned long long*>(&b);
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(ar), "l"(br));
  return *reinterpret_cast<float2*>(&r);
}

// Rows split over (row block, input slice) warp assignments: the largest
// power-of-two number of input slices that keeps every warp busy and divides
// the input words.
__device__ __forceinline__ int input_slices(int nrb, int ws) {
  int ksn = 1;
  while (ksn * 2 * nrb <= kWideWarps && ws % (ksn * 2) == 0) ksn *= 2;
  return ksn;
}

// Sign bit of element e (segment-local) of a small segment whose words start
// at w.
__device__ __forceinline__ uint32_t small_bit(const uint32_t* w, int64_t e) {
  return (w[e >> 5] >> bit_pos((int)(e & 31))) & 1u;
}

// One matrix of a step for all columns: out[r][col] = bias_s[r] + sum_k
// (W +- eps P_p)[r,k] a_col[k], inputs a = [inA (Kin) | inB (K - Kin)] stored
// [k][NC].  Callers synchronise before (inputs complete, tables free).
template <int NP>
__device__ void wide_matrix(const WideArgs& a, const WideMat& M, const float* inA,
                            const float* inB, const uint32_t* swT, const uint32_t* sml,
                            float2* U, float* out, float* part) {
  constexpr int NC = 2 * NP;
  const int tid = threadIdx.x, nt = blockDim.x;
  const float eps = a.eps;
  const int Gn = M.K / 4;
  // subset-sum tables: one thread per (probe, group); entry idx holds
  // (sum_i s_i a+_{k_i}, -sum_i s_i a-_{k_i}), s_i = -1 where bit i of idx is set
  for (int e = tid; e < NP * Gn; e += nt) {
    const int p = e / Gn, g = e - p * Gn;
    const int k0 = (g >> 1) * 8 + (g & 1);
    float2 x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int k = k0 + 2 * i;
      const float* src = k < M.Kin ? inA + k * NC : inB + (k - M.Kin) * NC;
      x[i] = make_float2(src[2 * p], src[2 * p + 1]);
    }
    float2 T[16];
    T[0] = wadd2(wadd2(wadd2(x[0], x[1]), x[2]), x[3]);
#pragma unroll
    for (int idx = 1; idx < 16; ++idx) {
      const int lb = (idx & 1) ? 0 : (idx & 2) ? 1 : (idx & 4) ? 2 : 3;   // lowest set bit
      T[idx] = wfma2(make_float2(-2.f, -2.f), x[lb], T[idx & (idx - 1)]);
    }
    float2* dst = U + (size_t)(p * a.gmax + g) * 16;
#pragma unroll
    for (int idx = 0; idx < 16; ++idx) dst[idx] = make_float2(T[idx].x, -T[idx].y);
  }
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31;
  const int WS = M.K / 32, nrb = M.Rp / 64;
  const int ksn = input_slices(nrb, WS);
  const int wg = warp / ksn, ks = warp - wg * ksn, ngr = kWideWarps / ksn;
  const int wsn = WS / ksn;
  for (int rb = wg; rb < nrb; rb += ngr) {
    const int r0 = rb * 64 + 2 * lane;
    float2 accW[2][NP], pe[2][NP];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
#pragma unroll
      for (int p = 0; p < NP; ++p) accW[rr][p] = pe[rr][p] = make_float2(0.f, 0.f);
    for (int wsi = ks * wsn; wsi < (ks + 1) * wsn; ++wsi) {
      const int k0 = wsi * 32;
      const float* inp = k0 < M.Kin ? inA + k0 * NC : inB + (k0 - M.Kin) * NC;
      // weights of the 32 inputs for rows r0, r0 + 1 (in flight during the
      // probe term below)
      float2 wv[32];
      const float2* wsrc = reinterpret_cast<const float2*>(M.wt + (int64_t)k0 * M.Rp + r0);
#pragma unroll
      for (int i = 0; i < 32; ++i) wv[i] = __ldg(wsrc + (int64_t)i * (M.Rp / 2));
      uint2 wd[NP];
#pragma unroll
      for (int p = 0; p < NP; ++p)
        wd[p] = *reinterpret_cast<const uint2*>(swT + (size_t)p * a.sw_words + M.sw +
                                                (size_t)wsi * M.Rp + r0);
      // probe term: 8 groups (block v = gq >> 1, parity gq & 1)
#pragma unroll
      for (int gq = 0; gq < 8; ++gq) {
        const int sh = 4 * (gq >> 1) + 16 * (gq & 1);
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          const float2* tb = U + (size_t)(p * a.gmax + wsi * 8 + gq) * 16;
          pe[0][p] = wadd2(pe[0][p], tb[(wd[p].x >> sh) & 15u]);
          pe[1][p] = wadd2(pe[1][p], tb[(wd[p].y >> sh) & 15u]);
        }
      }
      // weight term
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float4* xr = reinterpret_cast<const float4*>(inp + i * NC);
        const float2 w0 = make_float2(wv[i].x, wv[i].x);
        const float2 w1 = make_float2(wv[i].y, wv[i].y);
#pragma unroll
        for (int c4 = 0; c4 < NC / 4; ++c4) {
          const float4 x = xr[c4];
          accW[0][2 * c4] = wfma2(w0, make_float2(x.x, x.y), accW[0][2 * c4]);
          accW[0][2 * c4 + 1] = wfma2(w0, make_float2(x.z, x.w), accW[0][2 * c4 + 1]);
          accW[1][2 * c4] = wfma2(w1, make_float2(x.x, x.y), accW[1][2 * c4]);
          accW[1][2 * c4 + 1] = wfma2(w1, make_float2(x.z, x.w), accW[1][2 * c4 + 1]);
        }
      }
    }
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int r = r0 + rr;
      if (ksn == 1) {
        if (r < M.R) {
          const float bth = a.theta[M.offb + r];
#pragma unroll
          for (int p = 0; p < NP; ++p) {
            const float bd = small_bit(sml + (size_t)p * a.small_words + M.sb, r) ? -eps : eps;
            out[r * NC + 2 * p] = fmaf(eps, pe[rr][p].x, accW[rr][p].x) + (bth + bd);
            out[r * NC + 2 * p + 1] = fmaf(eps, pe[rr][p].y, accW[rr][p].y) + (bth - bd);
          }
        }
      } else {
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          part[(ks * M.Rp + r) * NC + 2 * p] = fmaf(eps, pe[rr][p].x, accW[rr][p].x);
          part[(ks * M.Rp + r) * NC + 2 * p + 1] = fmaf(eps, pe[rr][p].y, accW[rr][p].y);
        }
      }
    }
  }
  if (ksn > 1) {
    __syncthreads();
    for (int i = tid; i < M.R * NC; i += nt) {
      const int r = i / NC, col = i - r * NC;
      const int p = col >> 1;
      float sum = 0.f;
      for (int s = 0; s < ksn; ++s) sum += part[(s * M.Rp + r) * NC + col];
      const float bth = a.theta[M.offb + r];
      const float bd = small_bit(sml + (size_t)p * a.small_words + M.sb, r) ? -eps : eps;
      out[i] = sum + ((col & 1) ? bth - bd : bth + bd);
    }
  }
  __syncthreads();
}

template <int NP>
__global__ void __launch_bounds__(kWideThreads, 1) fp32_wide_kernel(const WideArgs a) {
  constexpr int NC = 2 * NP;
  extern __shared__ __align__(16) uint32_t smw[];
  const int pc = blockIdx.x * NP;               // first probe of this CTA (launch-local)
  const int npv = min(NP, a.nprobe - pc);       // probes of the CTA inside the launch
  const int b = blockIdx.y;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int H = a.H, E = a.E, V = a.V, L = a.L;
  uint32_t* swT = smw;                                           // [NP][sw_words]
  uint32_t* sml = swT + (size_t)NP * a.sw_words;                 // [NP][small_words]
  float2* U = reinterpret_cast<float2*>(sml + (size_t)NP * a.small_words);  // [NP][gmax][16]
  float* xe = reinterpret_cast<float*>(U + (size_t)NP * a.gmax * 16);       // [E][NC]
  float* hs = xe + E * NC;                                       // [L][H][NC]
  float* cs = hs + L * H * NC;                                   // [L][H][NC]
  float* G = cs + L * H * NC;                                    // [rmax][NC]
  float* part = G + a.rmax * NC;                                 // [pmax]
  float* rl = part + a.pmax;                                     // [NC]

  // sign words: probes past the launch (npv < NP) run on a valid probe index
  // and are never written out
  for (int i = tid; i < NP * a.sw_words; i += nt) swT[i] = 0u;   // pad rows stay zero
  for (int i = tid; i < 2 * L * H * NC; i += nt) hs[i] = 0.f;    // hs, cs
  for (int i = tid; i < NC; i += nt) rl[i] = 0.f;
  __syncthreads();
  for (int mi = 0; mi <= L; ++mi) {
    const WideMat& M = a.m[mi];
    const int64_t nwords = (int64_t)M.R * M.K / 32;
    const int64_t nbl = (nwords + 3) / 4;
    for (int64_t e = tid; e < NP * nbl; e += nt) {
      const int p = (int)(e / nbl);
      const int64_t qi = e - p * nbl;
      const uint32_t probe = (uint32_t)(a.probe0 + pc + (p < npv ? p : 0));
      const uint4 w = sign_block(a.seed, probe, (uint64_t)(M.off / 128 + qi));
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t wl = qi * 4 + i;
        if (wl < nwords) {
          const int64_t el = wl * 32;
          const int r = (int)(el / M.K);
          const int kw = (int)(el - (int64_t)r * M.K) / 32;
          swT[(size_t)p * a.sw_words + M.sw + (size_t)kw * M.Rp + r] = word_of(w, i);
        }
      }
    }
  }
  for (int s = 0; s < a.nsmall; ++s) {
    const int64_t nwords = (a.small_num[s] + 31) / 32;
    const int64_t nbl = (nwords + 3) / 4;
    for (int64_t e = tid; e < NP * nbl; e += nt) {
      const int p = (int)(e / nbl);
      const int64_t qi = e - p * nbl;
      const uint32_t probe = (uint32_t)(a.probe0 + pc + (p < npv ? p : 0));
      const uint4 w = sign_block(a.seed, probe, (uint64_t)(a.small_off[s] / 128 + qi));
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t wl = qi * 4 + i;
        if (wl < nwords) sml[(size_t)p * a.small_words + a.small_base[s] + wl] = word_of(w, i);
      }
    }
  }
  __syncthreads();

  for (int t = 0; t < a.T; ++t) {
    int tok = a.tokens[(int64_t)b * a.T + t];
    if (tok < 0 || tok >= V) {
      if (tid == 0) latch(a.err, kErrBounds);
      tok = 0;
    }
    for (int i = tid; i < E * NC; i += nt) {
      const int k = i / NC, col = i - k * NC;
      const int p = col >> 1;
      const int64_t el = (int64_t)tok * E + k;
      const float d = small_bit(sml + (size_t)p * a.small_words + a.sE, el) ? -a.eps : a.eps;
      const float th = a.theta[a.offE + el];
      xe[i] = (col & 1) ? th - d : th + d;
    }
    __syncthreads();
    for (int l = 0; l < L; ++l) {
      const float* inA = l == 0 ? xe : hs + (l - 1) * H * NC;
      float* hl = hs + l * H * NC;
      float* cl = cs + l * H * NC;
      wide_matrix<NP>(a, a.m[l], inA, hl, swT, sml, U, G, part);
      for (int i = tid; i < H * NC; i += nt) {
        const int u = i / NC, col = i - u * NC;
        const float ig = sigmoid_acc(G[u * NC + col]);
        const float fg = sigmoid_acc(G[(H + u) * NC + col]);
        const float gg = tanhf(G[(2 * H + u) * NC + col]);
        const float og = sigmoid_acc(G[(3 * H + u) * NC + col]);
        const float c = fg * cl[i] + ig * gg;
        cl[i] = c;
        hl[i] = og * tanhf(c);
      }
      __syncthreads();
    }
    wide_matrix<NP>(a, a.m[L], hs + (L - 1) * H * NC, nullptr, swT, sml, U, G, part);
    // cross-entropy: warp w takes column w, lanes stride over the vocabulary
    int tg = a.targets[(int64_t)b * a.T + t];
    if (tg >= V || tg < -1) {
      if (tid == 0) latch(a.err, kErrBounds);
      tg = -1;
    }
    if (tg >= 0) {
      for (int col = warp; col < NC; col += kWideWarps) {
        float m = -INFINITY;
        for (int v = lane; v < V; v += 32) m = fmaxf(m, G[v * NC + col]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float s = 0.f;
        for (int v = lane; v < V; v += 32) s += expf(G[v * NC + col] - m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) rl[col] += m + logf(s) - G[tg * NC + col];
      }
    }
    __syncthreads();
  }
  for (int i = tid; i < NC; i += nt) {
    const int p = i >> 1, s = i & 1;
    if (p < npv) a.rowloss[(int64_t)(2 * (pc + p) + s) * a.Bmax + b] = rl[i];
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
namespace {

struct WidePlan {
  int R[kMaxLayers + 1], Rp[kMaxLayers + 1], K[kMaxLayers + 1], Kin[kMaxLayers + 1];
  int sw[kMaxLayers + 1];
  int64_t wt_off[kMaxLayers + 1];   // float offsets of W^T in the workspace
  int64_t wt_floats = 0;
  int sw_words = 0, small_words = 0, gmax = 0, rmax = 0, pmax = 0;
  int nsmall = 0;
};

int round_up(int x, int m) { return (x + m - 1) / m * m; }

bool plan_wide(const zo_model_spec& s, WidePlan& P) {
  const int E = s.embed, H = s.hidden, V = s.vocab, L = s.layers;
  if (E % 32 || H % 32 || L < 1 || L > kMaxLayers) return false;
  int64_t wt = 0;
  int sw = 0;
  for (int mi = 0; mi <= L; ++mi) {
    const bool out = mi == L;
    P.R[mi] = out ? V : 4 * H;
    P.Rp[mi] = round_up(P.R[mi], 64);
    P.K[mi] = out ? H : (mi == 0 ? E : H) + H;
    P.Kin[mi] = out ? H : (mi == 0 ? E : H);
    P.sw[mi] = sw;
    sw += P.K[mi] / 32 * P.Rp[mi];
    P.wt_off[mi] = wt;
    wt += (int64_t)P.K[mi] * P.Rp[mi];
    wt = (wt + 63) / 64 * 64;
    P.gmax = P.gmax > P.K[mi] / 4 ? P.gmax : P.K[mi] / 4;
    P.rmax = P.rmax > P.Rp[mi] ? P.rmax : P.Rp[mi];
  }
  P.wt_floats = wt;
  P.sw_words = sw;
  // small segments: E, b_0..b_{L-1}, b_out
  int sm = (V * E + 31) / 32;
  for (int l = 0; l < L; ++l) sm += (4 * H + 31) / 32;
  sm += (V + 31) / 32;
  P.small_words = round_up(sm, 4);
  P.nsmall = L + 2;
  return true;
}

// partial sums of the matrices whose rows leave warps idle
int partial_floats(const WidePlan& P, int L, int nc) {
  int pm = 0;
  for (int mi = 0; mi <= L; ++mi) {
    const int nrb = P.Rp[mi] / 64, ws = P.K[mi] / 32;
    int ksn = 1;
    while (ksn * 2 * nrb <= kWideWarps && ws % (ksn * 2) == 0) ksn *= 2;
    if (ksn > 1) pm = pm > ksn * P.Rp[mi] * nc ? pm : ksn * P.Rp[mi] * nc;
  }
  return pm;
}

size_t wide_smem(const zo_model_spec& s, const WidePlan& P, int np) {
  const int nc = 2 * np;
  const size_t words = (size_t)np * P.sw_words + (size_t)np * P.small_words;
  const size_t tables = (size_t)np * P.gmax * 16 * sizeof(float2);
  const size_t floats = (size_t)s.embed * nc + 2 * (size_t)s.layers * s.hidden * nc +
                        (size_t)P.rmax * nc + partial_floats(P, s.layers, nc) + nc;
  return words * 4 + tables + floats * 4;
}

}  // namespace

// W^T copy of one matrix: wt[k][r] = W[r][k] for r < R, zero for R <= r < Rp.
__global__ void wide_transpose_kernel(const float* __restrict__ w, int R, int K, int Rp,
                                      float* __restrict__ wt) {
  __shared__ float tile[32][33];
  const int k0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;   // 32 x 8
  for (int i = ty; i < 32; i += 8) {
    const int r = r0 + i, k = k0 + tx;
    tile[i][tx] = (r < R && k < K) ? w[(int64_t)r * K + k] : 0.f;
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int k = k0 + i, r = r0 + tx;
    if (k < K && r < Rp) wt[(int64_t)k * Rp + r] = tile[tx][i];
  }
}

int fp32_wide_probes(const zo_model_spec& s, size_t limit, int64_t* wt_floats, size_t* smem) {
  WidePlan P;
  if (!plan_wide(s, P)) return 0;
  for (int np = 4; np >= 2; np /= 2) {
    const size_t sm = wide_smem(s, P, np);
    if (sm <= limit) {
      if (wt_floats) *wt_floats = P.wt_floats;
      if (smem) *smem = sm;
      return np;
    }
  }
  return 0;
}

template <int NP>
static cudaError_t launch_wide_np(const WideArgs& a, size_t smem, cudaStream_t st) {
  cudaFuncSetAttribute(fp32_wide_kernel<NP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)smem);
  dim3 grid((a.nprobe + NP - 1) / NP, a.B);
  fp32_wide_kernel<NP><<<grid, kWideThreads, smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_fp32_wide(const zo_ctx* ctx, const float* theta, uint64_t seed, int probe0,
                             int nprobe, float eps, const int32_t* tokens, const int32_t* targets,
                             int B, int T, cudaStream_t st) {
  const zo_model_spec& sp = ctx->spec;
  const Segments& s = ctx->seg;
  WidePlan P;
  if (!plan_wide(sp, P) || ctx->fp32_wide_np < 2 || !ctx->wt) return cudaErrorInvalidValue;
  const int L = sp.layers;
  // W^T copies of theta's current weights
  for (int mi = 0; mi <= L; ++mi) {
    const int seg = mi == L ? s.Wout : s.W[mi];
    dim3 grid((P.K[mi] + 31) / 32, (P.Rp[mi] + 31) / 32);
    wide_transpose_kernel<<<grid, dim3(32, 8), 0, st>>>(theta + s.off[seg], P.R[mi], P.K[mi],
                                                       P.Rp[mi], ctx->wt + P.wt_off[mi]);
    count_launch();
  }
  WideArgs a;
  a.theta = theta;
  a.seed = seed;
  a.probe0 = probe0;
  a.nprobe = nprobe;
  a.eps = eps;
  a.tokens = tokens;
  a.targets = targets;
  a.B = B;
  a.T = T;
  a.Bmax = sp.max_batch;
  a.V = sp.vocab;
  a.E = sp.embed;
  a.H = sp.hidden;
  a.L = L;
  a.offE = s.off[s.E];
  int base = 0;
  a.nsmall = 0;
  auto add_small = [&](int seg) {
    a.small_off[a.nsmall] = s.off[seg];
    a.small_num[a.nsmall] = s.numel[seg];
    a.small_base[a.nsmall] = base;
    const int b0 = base;
    base += (int)((s.numel[seg] + 31) / 32);
    ++a.nsmall;
    return b0;
  };
  a.sE = add_small(s.E);
  for (int mi = 0; mi <= L; ++mi) {
    WideMat& M = a.m[mi];
    const int seg = mi == L ? s.Wout : s.W[mi];
    const int segb = mi == L ? s.bout : s.b[mi];
    M.wt = ctx->wt + P.wt_off[mi];
    M.R = P.R[mi];
    M.Rp = P.Rp[mi];
    M.K = P.K[mi];
    M.Kin = P.Kin[mi];
    M.off = s.off[seg];
    M.offb = s.off[segb];
    M.sw = P.sw[mi];
    M.sb = add_small(segb);
  }
  a.sw_words = P.sw_words;
  a.small_words = P.small_words;
  a.gmax = P.gmax;
  a.rmax = P.rmax;
  // four probes per CTA share each weight load best; with few probes (a slice
  // of a probe-parallel step, small tests) two per CTA keep more SMs busy
  int np = ctx->fp32_wide_np;
  if (np == 4 && (int64_t)((nprobe + 3) / 4) * B < (int64_t)ctx->sm_count * 3 / 4) np = 2;
  a.pmax = partial_floats(P, L, 2 * np);
  a.rowloss = ctx->rowloss;
  a.err = ctx->err;
  const size_t smem = wide_smem(sp, P, np);
  return np == 4 ? launch_wide_np<4>(a, smem, st) : launch_wide_np<2>(a, smem, st);
}

}  // namespace zo
