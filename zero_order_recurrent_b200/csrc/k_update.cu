// Coefficients and the seed-replayed update (pith.science review, "What
// carries the argument": Theta' = Theta - 1/(2 n_pert) sum_i (L+_i - L-_i) p_i;
// alex-wiki "Method": theta' = theta - eta g_hat), plus the probe-sign test
// hook and the bf16 shadow cast.
#include "zo_common.cuh"
#include "zo_internal.h"

namespace zo {

// ---------------------------------------------------------------------------
// Sign words (test hook)
// ---------------------------------------------------------------------------
__global__ void sign_words_kernel(uint64_t seed, uint32_t probe, int64_t q0, int64_t n,
                                  uint32_t* out) {
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < n;
       k += (int64_t)gridDim.x * blockDim.x) {
    const uint4 w = sign_block(seed, probe, (uint64_t)(q0 + k));
    reinterpret_cast<uint4*>(out)[k] = w;
  }
}

cudaError_t launch_sign_words(uint64_t seed, int probe, int64_t q0, int64_t n, uint32_t* out,
                              cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const int grid = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  sign_words_kernel<<<grid, 256, 0, st>>>(seed, (uint32_t)probe, q0, n, out);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// bf16 shadow of theta
// ---------------------------------------------------------------------------
__global__ void cast_shadow_kernel(const float4* __restrict__ th, uint2* __restrict__ sh,
                                   int64_t n4) {
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < n4;
       k += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = th[k];
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t*>(&a);
    o.y = *reinterpret_cast<uint32_t*>(&b);
    sh[k] = o;
  }
}

cudaError_t launch_cast_shadow(const float* theta, __nv_bfloat16* shadow, int64_t d_pad,
                               cudaStream_t st) {
  const int64_t n4 = d_pad / 4;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t grid = (n4 + 255) / 256;
  if (grid > (int64_t)sms * 8) grid = (int64_t)sms * 8;
  if (grid < 1) grid = 1;
  cast_shadow_kernel<<<(int)grid, 256, 0, st>>>(reinterpret_cast<const float4*>(theta),
                                                 reinterpret_cast<uint2*>(shadow), n4);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Coefficients c_i = eta (L+_i - L-_i) / (2 eps n_pert)
// ---------------------------------------------------------------------------
__global__ void coeffs_kernel(const float* lp, const float* lm, int n, float eps, float eta,
                              float* out, unsigned* err) {
  const float scale = eta / (2.f * eps * (float)n);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const float a = lp[i], b = lm[i];
    float c = (a - b) * scale;
    if (!isfinite(a) || !isfinite(b) || !isfinite(c)) {
      latch(err, kErrNonfinite);
      c = __int_as_float(0x7fc00000);
    }
    out[i] = c;
  }
}

cudaError_t launch_coeffs(const float* lp, const float* lm, int n, float eps, float eta,
                          float* out, unsigned* err, cudaStream_t st) {
  const int grid = (n + 255) / 256;
  coeffs_kernel<<<grid, 256, 0, st>>>(lp, lm, n, eps, eta, out, err);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Update.  One warp handles a span of S consecutive 128-element blocks.  In
// the sign phase the 32 lanes compute the Philox words of all (probe, block)
// pairs of the span and park them in shared memory; in the apply phase the
// warp walks the span block by block, lane L owning the float4 at 4L..4L+3,
// so every global access is a coalesced 512-byte row.  Probes are summed in
// fp32 groups of 8 and the groups in fp64, then theta is rounded once.  S is
// chosen on the host so that all probes fit one pass (S * probes <= 512
// words per warp) and the spans still fill the GPU; with more probes than
// that, successive passes re-read theta.
// ---------------------------------------------------------------------------
constexpr int kUpdWarps = 4;
constexpr int kUpdSlots = 512;   // uint4 sign-word slots per warp (8 KB)

struct UpdateArgs {
  float* theta;
  __nv_bfloat16* shadow;   // may be null
  const float* coeffs;
  uint64_t seed;
  int n;
  int64_t nblk;            // d_pad / 128
  int S;                   // blocks per span
  int pmax;                // probes per pass (pmax * S <= kUpdSlots)
  int nseg;
  int64_t seg_off[kMaxSeg];
  int64_t seg_end[kMaxSeg];
  unsigned* err;
};

// Packed fp32x2 add (sm_100): two independent round-to-nearest sums.
__device__ __forceinline__ float2 add_f32x2(float2 a, float2 b) {
  unsigned long long ar = *reinterpret_cast<unsigned long long*>(&a);
  unsigned long long br = *reinterpret_cast<unsigned long long*>(&b);
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(ar), "l"(br));
  return *reinterpret_cast<float2*>(&r);
}

// PP > 0: compile-time probes per pass (n <= PP, unused slots carry c = 0,
// whose +-0 terms leave every sum unchanged), coefficients in registers,
// S = 128 / PP blocks per span (PP * S = 128 sign blocks: four Philox calls
// per lane) and theta staged in two buffers: the next span's loads are in
// flight while the current span is applied.  Small spans keep the shared
// memory per warp at ~10 KB, so 20 warps share an SM.
// PP == 0: runtime n, S and passes, one staging buffer.
template <int PP>
__global__ void __launch_bounds__(kUpdWarps * 32) update_kernel(const UpdateArgs a) {
  constexpr int SC = PP > 0 ? (128 / PP < 32 ? 128 / PP : 32) : 1;
  constexpr int WSLOTS = PP > 0 ? PP * SC : kUpdSlots;   // sign-word slots per warp
  constexpr int NBUF = PP > 0 ? 2 : 1;
  extern __shared__ uint4 dyn[];
  const int ncap = PP > 0 ? PP : a.n;
  float* negc = reinterpret_cast<float*>(dyn);             // [ncap], padded to 4
  uint4* words_all = dyn + (ncap + 3) / 4;                  // [warps][WSLOTS]
  const int S = PP > 0 ? SC : a.S;
  float4* stage_all = reinterpret_cast<float4*>(words_all + kUpdWarps * WSLOTS);  // [warps][NBUF][S*32]
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < ncap; i += blockDim.x) {
    const float c = i < a.n ? a.coeffs[i] : 0.f;
    if (!isfinite(c)) bad = 1;
    negc[i] = -c;
  }
  __syncthreads();
  if (bad) {
    if (blockIdx.x == 0 && threadIdx.x == 0) latch(a.err, kErrNonfinite);
    return;
  }
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  uint4* words = words_all + warp * WSLOTS;
  const uint32_t* words32 = reinterpret_cast<const uint32_t*>(words);
  float4* stage = stage_all + warp * NBUF * S * 32;
  const int64_t nspan = (a.nblk + S - 1) / S;
  const int64_t gw = blockIdx.x * (int64_t)kUpdWarps + warp;
  const int64_t nw = (int64_t)gridDim.x * kUpdWarps;
  const int widx = lane >> 3;
  const int sh = 2 * (lane & 7);
  const float4* th4 = reinterpret_cast<const float4*>(a.theta);
  float ncr[PP > 0 ? PP : 1];
  if constexpr (PP > 0) {
#pragma unroll
    for (int i = 0; i < PP; ++i) ncr[i] = negc[i];
  }

  auto issue = [&](int64_t sp, float4* dstbuf) {
    const int64_t qq = sp * S;
    const int nn = (int)min((int64_t)S, a.nblk - qq);
    for (int it = 0; it < nn; ++it) {
      const uint32_t dst = (uint32_t)__cvta_generic_to_shared(dstbuf + it * 32 + lane);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst),
                   "l"(th4 + (qq + it) * 32 + lane)
                   : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  int buf = 0;
  if (PP > 0 && gw < nspan) issue(gw, stage);

  for (int64_t span = gw; span < nspan; span += nw, buf ^= (NBUF - 1)) {
    const int64_t q0 = span * S;
    const int nq = (int)min((int64_t)S, a.nblk - q0);
    float4* cur = stage + buf * S * 32;
    // segment of the span's first block; segments start on block boundaries
    int seg = 0;
    while (seg + 1 < a.nseg && q0 * 128 >= a.seg_off[seg + 1]) ++seg;
    const int pmax = PP > 0 ? PP : a.pmax;
    for (int p0 = 0; p0 < a.n; p0 += pmax) {
      const int np = min(pmax, a.n - p0);
      const bool last_pass = p0 + pmax >= a.n;
      if (PP == 0) {
        // theta loads land during the sign phase (a later pass re-reads what
        // this lane stored in the previous one)
        if (p0 > 0) __threadfence_block();
        issue(span, cur);
      }
      const int pairs = np * S;
#pragma unroll 4
      for (int t = lane; t < pairs; t += 32) {
        const int i = t / S, b = t - i * S;
        if (b < nq) words[t] = sign_block(a.seed, (uint32_t)(p0 + i), (uint64_t)(q0 + b));
      }
      if (PP > 0) {
        // next span's theta into the other buffer, then wait for this span's
        if (span + nw < nspan) issue(span + nw, stage + (buf ^ 1) * S * 32);
        else asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      } else {
        asm volatile("cp.async.wait_all;" ::: "memory");
      }
      __syncwarp();
      int sg = seg;
      for (int it = 0; it < nq; ++it) {
        const int64_t q = q0 + it;
        const float4 th = cur[it * 32 + lane];
        double acc0 = th.x, acc1 = th.y, acc2 = th.z, acc3 = th.w;
        const uint32_t* wcol = words32 + it * 4 + widx;
        if constexpr (PP > 0) {
#pragma unroll
          for (int g = 0; g < PP; g += 8) {
            float2 s01 = make_float2(0.f, 0.f), s23 = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = g; i < g + 8; ++i) {
              const uint32_t w = wcol[i * SC * 4] >> sh;
              s01 = add_f32x2(s01, make_float2(flip_sign(ncr[i], w << 31), flip_sign(ncr[i], w << 15)));
              s23 = add_f32x2(s23, make_float2(flip_sign(ncr[i], w << 30), flip_sign(ncr[i], w << 14)));
            }
            acc0 += s01.x;
            acc1 += s01.y;
            acc2 += s23.x;
            acc3 += s23.y;
          }
        } else {
          for (int g = 0; g < np; g += 8) {
            float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
            const int ge = min(g + 8, np);
#pragma unroll 8
            for (int i = g; i < ge; ++i) {
              const float nc = negc[p0 + i];
              const uint32_t w = wcol[i * S * 4] >> sh;
              s0 += flip_sign(nc, w << 31);
              s1 += flip_sign(nc, w << 15);
              s2 += flip_sign(nc, w << 30);
              s3 += flip_sign(nc, w << 14);
            }
            acc0 += s0;
            acc1 += s1;
            acc2 += s2;
            acc3 += s3;
          }
        }
        while (sg + 1 < a.nseg && q * 128 >= a.seg_off[sg + 1]) ++sg;
        const int64_t j = q * 128 + 4 * lane;
        const int64_t lim = a.seg_end[sg];
        float4 o;
        o.x = j + 0 < lim ? (float)acc0 : th.x;
        o.y = j + 1 < lim ? (float)acc1 : th.y;
        o.z = j + 2 < lim ? (float)acc2 : th.z;
        o.w = j + 3 < lim ? (float)acc3 : th.w;
        reinterpret_cast<float4*>(a.theta)[q * 32 + lane] = o;
        if (last_pass && a.shadow) {
          __nv_bfloat162 lo = __floats2bfloat162_rn(o.x, o.y);
          __nv_bfloat162 hi = __floats2bfloat162_rn(o.z, o.w);
          uint2 pk;
          pk.x = *reinterpret_cast<uint32_t*>(&lo);
          pk.y = *reinterpret_cast<uint32_t*>(&hi);
          reinterpret_cast<uint2*>(a.shadow)[q * 32 + lane] = pk;
        }
      }
      __syncwarp();
    }
  }
}

template <int PP>
static cudaError_t launch_update_pp(const UpdateArgs& a, int sm_count, cudaStream_t st) {
  const int ncap = PP > 0 ? PP : a.n;
  const size_t wslots = PP > 0 ? (size_t)PP * a.S : (size_t)kUpdSlots;
  const size_t smem = sizeof(uint4) * ((ncap + 3) / 4 + (size_t)kUpdWarps * wslots +
                                      (size_t)kUpdWarps * (PP > 0 ? 2 : 1) * a.S * 32);
  cudaFuncSetAttribute(update_kernel<PP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaFuncSetAttribute(update_kernel<PP>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  const int64_t nspan = (a.nblk + a.S - 1) / a.S;
  int64_t grid = (nspan + kUpdWarps - 1) / kUpdWarps;
  int per_sm = (int)((220 * 1024) / smem);
  if (per_sm < 1) per_sm = 1;
  if (per_sm > 8) per_sm = 8;
  const int64_t cap = (int64_t)sm_count * per_sm;
  if (grid > cap) grid = cap;
  update_kernel<PP><<<(int)grid, kUpdWarps * 32, smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_update(const zo_ctx* ctx, float* theta, uint64_t seed, int n,
                          const float* coeffs, __nv_bfloat16* shadow, cudaStream_t st) {
  UpdateArgs a;
  a.theta = theta;
  a.shadow = shadow;
  a.coeffs = coeffs;
  a.seed = seed;
  a.n = n;
  a.nblk = ctx->seg.d_pad / 128;
  a.nseg = ctx->seg.n;
  for (int s = 0; s < ctx->seg.n; ++s) {
    a.seg_off[s] = ctx->seg.off[s];
    a.seg_end[s] = ctx->seg.off[s] + ctx->seg.numel[s];
  }
  a.err = ctx->err;
  const int64_t want = (int64_t)ctx->sm_count * 16;   // spans that fill the GPU
  // compile-time probe counts for large models
  const int pp = n <= 16 ? 16 : n <= 32 ? 32 : n <= 64 ? 64 : 0;
  if (pp) {
    const int S = 128 / pp < 32 ? 128 / pp : 32;
    if ((a.nblk + S - 1) / S >= want) {
      a.S = S;
      a.pmax = pp;
      if (pp == 16) return launch_update_pp<16>(a, ctx->sm_count, st);
      if (pp == 32) return launch_update_pp<32>(a, ctx->sm_count, st);
      return launch_update_pp<64>(a, ctx->sm_count, st);
    }
  }
  // blocks per span: all probes in one pass if possible, and enough spans
  // to give every SM 16 warps of work
  int S = 32;
  while (S > 1 && S * n > kUpdSlots) S /= 2;
  while (S > 1 && (a.nblk + S - 1) / S < want) S /= 2;
  a.S = S;
  a.pmax = kUpdSlots / S < n ? kUpdSlots / S : n;
  return launch_update_pp<0>(a, ctx->sm_count, st);
}

}  // namespace zo
