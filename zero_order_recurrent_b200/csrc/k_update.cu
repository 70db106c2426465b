// Coefficients (central and forward-difference) and the seed-replayed update
// (pith.science review, "What carries the argument": Theta' = Theta -
// 1/(2 n_pert) sum_i (L+_i - L-_i) p_i; alex-wiki "Method": theta' = theta -
// eta g_hat), plus the probe-sign test hook and the bf16 shadow cast.
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

// Forward-difference coefficients c_i = eta (L+_i - L0) / (eps n_pert).
__global__ void coeffs_forward_kernel(const float* lp, const float* l0, int n, float eps,
                                      float eta, float* out, unsigned* err) {
  const float scale = eta / (eps * (float)n);
  const float b = *l0;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const float a = lp[i];
    float c = (a - b) * scale;
    if (!isfinite(a) || !isfinite(b) || !isfinite(c)) {
      latch(err, kErrNonfinite);
      c = __int_as_float(0x7fc00000);
    }
    out[i] = c;
  }
}

cudaError_t launch_coeffs_forward(const float* lp, const float* l0, int n, float eps, float eta,
                                  float* out, unsigned* err, cudaStream_t st) {
  const int grid = (n + 255) / 256;
  coeffs_forward_kernel<<<grid, 256, 0, st>>>(lp, l0, n, eps, eta, out, err);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Update with four-probe tables (up to 8 probes, and above 64 in passes of
// 16 groups; 9..64 probes take the eight-probe tables below).
// theta'_j = theta_j + sum_i (-c_i) p_ij is evaluated four probes at a time
// through subset-sum tables: for the probes 4g..4g+3 of group g,
//   T_g[s] = sum_{r<4} (-c_{4g+r}) (1 - 2 s_r),   s = 4-bit sign pattern,
// (16 entries, computed in fp64 and rounded once) so one shared-memory lookup
// replaces four sign applications.  The tables hold 16 consecutive words, one
// per bank, so a warp's lookups never conflict.
//
// One warp handles a span of S consecutive 128-element blocks.  Sign phase:
// lane t owns one (group, block) pair, computes its four probes' Philox
// blocks and transposes the bits so that each byte holds one parameter's
// 4-bit pattern, pre-shifted to a word offset (pattern << 2), and parks them
// in shared memory.  Apply phase: lane L owns the float4 at 4L..4L+3 of each
// block (coalesced 512-byte rows) and, per group, takes its four bytes with
// byte permutes and sums the four table entries per parameter in a pairwise
// tree.  theta is staged by cp.async in two buffers, so the next span's
// loads are in flight during this span's work.
// ---------------------------------------------------------------------------
constexpr int kUpdWarps = 4;
constexpr int kPairStride = 17;   // 8-byte units per (group, block) pair: 16 + 1 pad

struct UpdateArgs {
  float* theta;
  __nv_bfloat16* shadow;   // may be null
  const float* coeffs;
  uint64_t seed;
  int n;
  int ngroups;             // table groups (chunks * NG)
  int chunks;              // passes of NG groups over each span
  int64_t nblk;            // d_pad / 128
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

// Bits of a where m is set, bits of b elsewhere.
__device__ __forceinline__ uint32_t bit_select(uint32_t m, uint32_t a, uint32_t b) {
  return (a & m) | (b & ~m);
}

// Transposes four probes' sign words (A = probe 4g, ..., D = probe 4g+3; bit p
// = word position p) into eight index words: byte j of W[c] holds, at bits
// 2..5, the pattern (A,B,C,D)[c + 8j] as bits 0..3.  Two interleaving steps
// pair up bits and then bit pairs of the four words (nibble u of n_s holds
// position 4u + (0,2,1,3)[s]); the last step spreads the nibbles to bytes.
__device__ __forceinline__ void index_bytes(uint32_t A, uint32_t B, uint32_t C, uint32_t D,
                                            uint32_t (&W)[8]) {
  const uint32_t m1 = 0x55555555u, m2 = 0x33333333u, m4 = 0x3C3C3C3Cu;
  const uint32_t abe = bit_select(m1, A, B << 1), abo = bit_select(m1, A >> 1, B);
  const uint32_t cde = bit_select(m1, C, D << 1), cdo = bit_select(m1, C >> 1, D);
  const uint32_t n0 = bit_select(m2, abe, cde << 2), n1 = bit_select(m2, abe >> 2, cde);
  const uint32_t n2 = bit_select(m2, abo, cdo << 2), n3 = bit_select(m2, abo >> 2, cdo);
  W[0] = (n0 << 2) & m4;
  W[1] = (n2 << 2) & m4;
  W[2] = (n1 << 2) & m4;
  W[3] = (n3 << 2) & m4;
  W[4] = (n0 >> 2) & m4;
  W[5] = (n2 >> 2) & m4;
  W[6] = (n1 >> 2) & m4;
  W[7] = (n3 >> 2) & m4;
}

__device__ __forceinline__ float table_at(const float* t, uint32_t byte_off) {
  return *reinterpret_cast<const float*>(reinterpret_cast<const char*>(t) + byte_off);
}

// theta' of block q (lane: its float4): pads past the block's segment end
// keep theta, and the bf16 shadow gets the same values.  clean: the whole
// span lies inside one segment's real entries, so no block needs the segment
// search or the mask.
__device__ __forceinline__ void store_block(const UpdateArgs& a, int64_t q, int lane, int& sg,
                                            bool clean, float4 th, float4 o) {
  if (!clean) {
    while (sg + 1 < a.nseg && q * 128 >= a.seg_off[sg + 1]) ++sg;
    const int64_t lim = a.seg_end[sg];
    if (q * 128 + 128 > lim) {
      const int64_t j = q * 128 + 4 * lane;
      o.x = j + 0 < lim ? o.x : th.x;
      o.y = j + 1 < lim ? o.y : th.y;
      o.z = j + 2 < lim ? o.z : th.z;
      o.w = j + 3 < lim ? o.w : th.w;
    }
  }
  reinterpret_cast<float4*>(a.theta)[q * 32 + lane] = o;
  if (a.shadow) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(o.x, o.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(o.z, o.w);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&lo);
    pk.y = *reinterpret_cast<uint32_t*>(&hi);
    reinterpret_cast<uint2*>(a.shadow)[q * 32 + lane] = pk;
  }
}

// NG groups (4 NG probes) per pass.  MULTI: runtime number of passes, each
// pass's fp32 tree sum added into an fp64 accumulator (n_pert > 64).
template <int NG, bool MULTI>
__global__ void __launch_bounds__(kUpdWarps * 32, 4) update_kernel(const UpdateArgs a) {
  constexpr int S = NG >= 4 ? 32 / NG : 8;   // blocks per span
  constexpr int PAIRS = NG * S;              // (group, block) pairs of a pass, <= 32
  extern __shared__ __align__(16) unsigned char dyn[];
  float* tab = reinterpret_cast<float*>(dyn);                       // [ngroups][16]
  uint2* idx_all = reinterpret_cast<uint2*>(dyn + a.ngroups * 64);  // [warps][32][kPairStride]
  float4* stage_all = reinterpret_cast<float4*>(idx_all + kUpdWarps * 32 * kPairStride);
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (int e = threadIdx.x; e < a.ngroups * 16; e += blockDim.x) {
    const int g = e >> 4, s = e & 15;
    double t = 0.0;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = 4 * g + r;
      const float c = i < a.n ? a.coeffs[i] : 0.f;
      if (!isfinite(c)) bad = 1;
      t += ((s >> r) & 1) ? (double)c : -(double)c;
    }
    tab[e] = (float)t;
  }
  __syncthreads();
  if (bad) {
    if (blockIdx.x == 0 && threadIdx.x == 0) latch(a.err, kErrNonfinite);
    return;
  }
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  uint2* idxw = idx_all + warp * 32 * kPairStride;
  float4* stage = stage_all + warp * 2 * S * 32;
  const int64_t nspan = (a.nblk + S - 1) / S;
  const int64_t gw = blockIdx.x * (int64_t)kUpdWarps + warp;
  const int64_t nw = (int64_t)gridDim.x * kUpdWarps;
  const float4* th4 = reinterpret_cast<const float4*>(a.theta);
  // apply role: word lane>>3, elements 4m..4m+3 (m = lane & 7) at positions
  // 2m, 2m+16, 2m+1, 2m+17 = bytes (m>>2, m>>2 + 2) of index words 2(m&3), +1
  const int unit = (lane >> 3) * 4 + (lane & 3);
  const uint32_t sel_lo = 0x4440u | (uint32_t)((lane & 7) >> 2);
  const uint32_t sel_hi = sel_lo + 2;
  // sign role: this lane's (group, block) pair
  const int pg = lane / S, pb = lane % S;

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
  auto write_out = [&](int64_t q, int& sg, bool clean, float4 th, float4 o) {
    store_block(a, q, lane, sg, clean, th, o);
  };
  int buf = 0;
  if (gw < nspan) issue(gw, stage);

  for (int64_t span = gw; span < nspan; span += nw, buf ^= 1) {
    const int64_t q0 = span * S;
    const int nq = (int)min((int64_t)S, a.nblk - q0);
    float4* cur = stage + buf * S * 32;
    if (span + nw < nspan) issue(span + nw, stage + (buf ^ 1) * S * 32);
    else asm volatile("cp.async.commit_group;" ::: "memory");
    // segment of the span's first block; segments start on block boundaries
    int sg = 0;
    while (sg + 1 < a.nseg && q0 * 128 >= a.seg_off[sg + 1]) ++sg;
    const bool clean = (q0 + nq) * 128 <= a.seg_end[sg];
    double acc[MULTI ? S : 1][4];
    for (int ch = 0; ch < (MULTI ? a.chunks : 1); ++ch) {
      // sign phase
      if (lane < PAIRS && pb < nq) {
        const int pbase = (ch * NG + pg) * 4;
        // all four blocks unconditionally (independent chains interleave);
        // probes past n_pert are zeroed afterwards
        uint4 w[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) w[r] = sign_block(a.seed, (uint32_t)(pbase + r), (uint64_t)(q0 + pb));
#pragma unroll
        for (int r = 0; r < 4; ++r)
          if (pbase + r >= a.n) w[r] = make_uint4(0u, 0u, 0u, 0u);
        uint2* dst = idxw + lane * kPairStride;
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
          uint32_t W[8];
          index_bytes(word_of(w[0], wi), word_of(w[1], wi), word_of(w[2], wi), word_of(w[3], wi), W);
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) dst[wi * 4 + cc] = make_uint2(W[2 * cc], W[2 * cc + 1]);
        }
      }
      if (ch == 0) asm volatile("cp.async.wait_group 1;" ::: "memory");
      __syncwarp();
      // apply phase
      const float* tabc = tab + ch * NG * 16;
#pragma unroll
      for (int it = 0; it < S; ++it) {
        if (it < nq) {
          float2 v01[NG], v23[NG];
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            const uint2 wv = idxw[(g * S + it) * kPairStride + unit];
            const float* tg = tabc + g * 16;
            v01[g] = make_float2(table_at(tg, __byte_perm(wv.x, 0u, sel_lo)),
                                 table_at(tg, __byte_perm(wv.x, 0u, sel_hi)));
            v23[g] = make_float2(table_at(tg, __byte_perm(wv.y, 0u, sel_lo)),
                                 table_at(tg, __byte_perm(wv.y, 0u, sel_hi)));
          }
#pragma unroll
          for (int w = 1; w < NG; w *= 2) {
#pragma unroll
            for (int g = 0; g + w < NG; g += 2 * w) {
              v01[g] = add_f32x2(v01[g], v01[g + w]);
              v23[g] = add_f32x2(v23[g], v23[g + w]);
            }
          }
          const float4 th = cur[it * 32 + lane];
          if constexpr (MULTI) {
            if (ch == 0) {
              acc[it][0] = th.x;
              acc[it][1] = th.y;
              acc[it][2] = th.z;
              acc[it][3] = th.w;
            }
            acc[it][0] += v01[0].x;
            acc[it][1] += v01[0].y;
            acc[it][2] += v23[0].x;
            acc[it][3] += v23[0].y;
          } else {
            const float2 o01 = add_f32x2(make_float2(th.x, th.y), v01[0]);
            const float2 o23 = add_f32x2(make_float2(th.z, th.w), v23[0]);
            write_out(q0 + it, sg, clean, th, make_float4(o01.x, o01.y, o23.x, o23.y));
          }
        }
      }
      __syncwarp();   // the next pass's sign phase reuses the index words
    }
    if constexpr (MULTI) {
#pragma unroll
      for (int it = 0; it < S; ++it) {
        if (it < nq)
          write_out(q0 + it, sg, clean, cur[it * 32 + lane],
                    make_float4((float)acc[it][0], (float)acc[it][1], (float)acc[it][2],
                                (float)acc[it][3]));
      }
    }
    __syncwarp();
  }
}

template <int NG, bool MULTI>
static cudaError_t launch_update_ng(const UpdateArgs& a, int sm_count, cudaStream_t st) {
  constexpr int S = NG >= 4 ? 32 / NG : 8;
  const size_t smem = (size_t)a.ngroups * 64 + (size_t)kUpdWarps * 32 * kPairStride * 8 +
                      (size_t)kUpdWarps * 2 * S * 32 * 16;
  cudaFuncSetAttribute(update_kernel<NG, MULTI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)smem);
  cudaFuncSetAttribute(update_kernel<NG, MULTI>, cudaFuncAttributePreferredSharedMemoryCarveout,
                       100);
  const int64_t nspan = (a.nblk + S - 1) / S;
  int64_t grid = (nspan + kUpdWarps - 1) / kUpdWarps;
  // one resident wave: blocks per SM as registers and shared memory allow
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, update_kernel<NG, MULTI>,
                                                    kUpdWarps * 32, smem) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const int64_t cap = (int64_t)sm_count * per_sm;
  if (grid > cap) grid = cap;
  update_kernel<NG, MULTI><<<(int)grid, kUpdWarps * 32, smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Update with eight-probe tables (9..64 probes).  For the probes 8g..8g+7,
//   T_g[s] = sum_{r<8} (-c_{8g+r}) (1 - 2 s_r),   s = 8-bit sign pattern,
// so one lookup stands for eight sign applications, half the lookups and
// tree adds of the four-probe tables.  256 entries read at random would
// collide in the 32 banks, so every entry is stored 16 times: a 64 KB table
// block B holds rows of 256 bytes (row e: entry e), and in each row the
// groups 4B + t (t = 0..3) take bytes 64t..64t+63, one copy per 4 bytes.  In
// one lookup, lanes 0..15 read group 4B + t from copy (lane & 15) and lanes
// 16..31 read group 4B + ((t + 1) & 3), which sits in the other half of the
// banks, so every lane hits its own bank.  The byte offset e * 256 is the
// pattern byte itself moved to byte 1 of the address by one byte permute that
// takes bytes 0, 2 and 3 from the lane's column word (the block base is 64 KB
// aligned), so each lookup is one PRMT and one LDS.
//
// Sign phase: lane t owns one (group, block) pair, computes its eight probes'
// Philox blocks, and per word position transposes the 8 x 32 bit matrix with
// three rounds of delta swaps: byte q of word m then holds the eight probes'
// bits at bit position 8q + m, the byte placement of the four-probe kernel,
// so the apply phase picks a lane's bytes the same way.  Each warp owns a
// slot (index rows and a theta staging buffer) in the shared memory
// around the table blocks.
// ---------------------------------------------------------------------------
constexpr int kIdx8Row = 36;        // 32-bit words per (group, block) row: 32 + 4 pad
constexpr int kUpd8MaxWarps = 16;   // 128 registers a thread

// After the three rounds, bit r of byte q of x[m] is bit 8q + m of the input
// x[r].  Round d exchanges, between x[i] and x[i + d] (i & d == 0), the bits
// of x[i] at positions p with p & d set and those of x[i + d] at p - d: each
// new word is one shift and one three-input select.
__device__ __forceinline__ void transpose8x32(uint32_t (&x)[8]) {
#pragma unroll
  for (int d = 1; d < 8; d <<= 1) {
    const uint32_t m = d == 1 ? 0x55555555u : d == 2 ? 0x33333333u : 0x0F0F0F0Fu;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i & d) continue;
      const uint32_t lo = bit_select(m, x[i], x[i + d] << d);
      const uint32_t hi = bit_select(m, x[i] >> d, x[i + d]);
      x[i] = lo;
      x[i + d] = hi;
    }
  }
}

// Shared-memory load at addr + OFF (OFF: the table block's offset).
template <int OFF>
__device__ __forceinline__ float lds_table(uint32_t addr) {
  float v;
  asm("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(addr), "n"(OFF));
  return v;
}

// The four table values of a lane's four elements for one eight-probe group:
// idx points at the lane's two index words in the group's row for the block.
template <int OFF>
__device__ __forceinline__ void lookup8(const uint32_t* idx, uint32_t col, uint32_t sel_lo,
                                        uint32_t sel_hi, float2& v01, float2& v23) {
  const uint2 wv = *reinterpret_cast<const uint2*>(idx);
  v01.x = lds_table<OFF>(__byte_perm(wv.x, col, sel_lo));
  v01.y = lds_table<OFF>(__byte_perm(wv.x, col, sel_hi));
  v23.x = lds_table<OFF>(__byte_perm(wv.y, col, sel_lo));
  v23.y = lds_table<OFF>(__byte_perm(wv.y, col, sel_hi));
}

// A span's theta copies are issued when the span starts and fly during its
// sign phase; one staging buffer keeps the slot small, so 16 warps fit (with
// two buffers, the next span's copies in flight during this span, only 12 fit
// at 32 probes and 6 at 16, and the kernel ran 8-24% slower).
template <int G8>
__global__ void __launch_bounds__(kUpd8MaxWarps * 32, 1)
    update8_kernel(const UpdateArgs a, uint32_t dyn_bytes) {
  constexpr int S = 32 / G8;            // blocks per span: G8 x S (group, block) pairs = 32 lanes
  constexpr int NB = (G8 + 3) / 4;      // 64 KB table blocks
  constexpr int KG = G8 < 4 ? G8 : 4;   // groups per table block
  constexpr uint32_t kIdxBytes = 32 * kIdx8Row * 4;
  constexpr uint32_t kSlot = kIdxBytes + S * 512;
  static_assert(G8 == 2 || G8 == 4 || G8 == 8, "eight-probe tables: 2, 4 or 8 groups");
  extern __shared__ __align__(16) unsigned char dyn[];
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(dyn);
  const uint32_t t0 = (base + 0xFFFFu) & ~0xFFFFu;
  const uint32_t tend = t0 + NB * 65536u;
  if (tend > base + dyn_bytes) {   // the launcher sizes the allocation so this cannot happen
    if (threadIdx.x == 0) latch(a.err, kErrBounds);
    return;
  }
  bool badc = false;
  for (int e = threadIdx.x; e < G8 * 256; e += blockDim.x) {
    const int g = e >> 8, s = e & 255;
    double t = 0.0;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int i = 8 * g + r;
      const float c = i < a.n ? a.coeffs[i] : 0.f;
      badc |= !isfinite(c);
      t += ((s >> r) & 1) ? (double)c : -(double)c;
    }
    const float v = (float)t;
    float4* row = reinterpret_cast<float4*>(dyn + (t0 - base) + (g / KG) * 65536 + s * 256 +
                                            (g % KG) * 64);
#pragma unroll
    for (int k = 0; k < 4; ++k) row[k] = make_float4(v, v, v, v);
  }
  if (__syncthreads_or(badc)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) latch(a.err, kErrNonfinite);
    return;
  }
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const uint32_t nfront = (t0 - base) / kSlot;
  const uint32_t slot = (uint32_t)warp < nfront ? base + warp * kSlot
                                                : tend + ((uint32_t)warp - nfront) * kSlot;
  if (slot + kSlot > base + dyn_bytes) {   // likewise excluded by the launcher
    if (lane == 0) latch(a.err, kErrBounds);
    return;
  }
  uint32_t* idxw = reinterpret_cast<uint32_t*>(dyn + (slot - base));
  const float4* stage = reinterpret_cast<const float4*>(dyn + (slot - base) + kIdxBytes);
  const uint32_t stage_s = slot + kIdxBytes;
  const int64_t nspan = (a.nblk + S - 1) / S;
  const int64_t gw = blockIdx.x * (int64_t)nwarps + warp;
  const int64_t nw = (int64_t)gridDim.x * nwarps;
  const float4* th4 = reinterpret_cast<const float4*>(a.theta);
  // apply role: as in the four-probe kernel, elements 4m..4m+3 of word
  // lane>>3 (m = lane & 7) take bytes (m>>2, m>>2 + 2) of words 2(m&3), +1;
  // the permute puts the byte at bits 8..15 over the column word
  const int unit = (lane >> 3) * 4 + (lane & 3);
  const uint32_t sel_lo = 0x7604u | ((uint32_t)((lane & 7) >> 2) << 4);
  const uint32_t sel_hi = sel_lo + 0x20u;
  uint32_t col[KG];
  int rowoff[KG];
#pragma unroll
  for (int k = 0; k < KG; ++k) {
    const int t = (k + (lane >> 4)) & (KG - 1);
    col[k] = t0 + 4u * (uint32_t)((lane & 15) + 16 * t);
    rowoff[k] = t * S * kIdx8Row + 2 * unit;
  }
  const int pg = lane / S, pb = lane % S;   // sign role: this lane's (group, block) pair

  // theta copies of a span: lane's float4 of each block (full spans unrolled)
  auto issue = [&](int64_t q0, int nq) {
    const float4* src = th4 + q0 * 32 + lane;
    const uint32_t dst = stage_s + (uint32_t)lane * 16u;
    if (nq == S) {
#pragma unroll
      for (int it = 0; it < S; ++it)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + it * 512),
                     "l"(src + it * 32)
                     : "memory");
    } else {
      for (int it = 0; it < nq; ++it)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + it * 512),
                     "l"(src + it * 32)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  // sum over the probes of block it's table values for this lane's four
  // elements, plus theta
  auto block_out = [&](int it, float4& th) -> float4 {
    float2 v01[G8], v23[G8];
#pragma unroll
    for (int k = 0; k < KG; ++k) {
      lookup8<0>(idxw + it * kIdx8Row + rowoff[k], col[k], sel_lo, sel_hi, v01[k], v23[k]);
      if constexpr (NB == 2)
        lookup8<65536>(idxw + (4 * S + it) * kIdx8Row + rowoff[k], col[k], sel_lo, sel_hi,
                       v01[4 + k], v23[4 + k]);
    }
#pragma unroll
    for (int w = 1; w < G8; w *= 2) {
#pragma unroll
      for (int g = 0; g + w < G8; g += 2 * w) {
        v01[g] = add_f32x2(v01[g], v01[g + w]);
        v23[g] = add_f32x2(v23[g], v23[g + w]);
      }
    }
    th = stage[it * 32 + lane];
    const float2 o01 = add_f32x2(make_float2(th.x, th.y), v01[0]);
    const float2 o23 = add_f32x2(make_float2(th.z, th.w), v23[0]);
    return make_float4(o01.x, o01.y, o23.x, o23.y);
  };
  for (int64_t span = gw; span < nspan; span += nw) {
    const int64_t q0 = span * S;
    const int nq = (int)min((int64_t)S, a.nblk - q0);
    issue(q0, nq);
    int sg = 0;
    while (sg + 1 < a.nseg && q0 * 128 >= a.seg_off[sg + 1]) ++sg;
    const bool clean = (q0 + nq) * 128 <= a.seg_end[sg];
    // sign phase (probes past n_pert have zero coefficients, so their bits
    // select equal table entries and need no masking)
    if (pb < nq) {
      uint4 w[8];
#pragma unroll
      for (int r = 0; r < 8; ++r)
        w[r] = sign_block(a.seed, (uint32_t)(8 * pg + r), (uint64_t)(q0 + pb));
      uint32_t* row = idxw + lane * kIdx8Row;
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {
        uint32_t x[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) x[r] = word_of(w[r], wi);
        transpose8x32(x);
        reinterpret_cast<uint4*>(row + wi * 8)[0] = make_uint4(x[0], x[1], x[2], x[3]);
        reinterpret_cast<uint4*>(row + wi * 8)[1] = make_uint4(x[4], x[5], x[6], x[7]);
      }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncwarp();
    // apply phase: a full span inside one segment's real entries with the
    // shadow present (all but a few spans) stores without per-block checks
    if (nq == S && clean && a.shadow) {
      float4* tdst = reinterpret_cast<float4*>(a.theta) + q0 * 32 + lane;
      uint2* sdst = reinterpret_cast<uint2*>(a.shadow) + q0 * 32 + lane;
#pragma unroll
      for (int it = 0; it < S; ++it) {
        float4 th;
        const float4 o = block_out(it, th);
        tdst[it * 32] = o;
        __nv_bfloat162 lo = __floats2bfloat162_rn(o.x, o.y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(o.z, o.w);
        sdst[it * 32] = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
      }
    } else {
#pragma unroll
      for (int it = 0; it < S; ++it) {
        if (it < nq) {
          float4 th;
          const float4 o = block_out(it, th);
          store_block(a, q0 + it, lane, sg, clean, th, o);
        }
      }
    }
    __syncwarp();   // the next span's sign phase and copies reuse the slot
  }
}

template <int G8>
static cudaError_t launch_update8(const UpdateArgs& a, int sm_count, cudaStream_t st) {
  constexpr int S = 32 / G8;
  constexpr uint32_t kSlot = 32 * kIdx8Row * 4 + S * 512;
  constexpr uint32_t kTables = ((G8 + 3) / 4) * 65536u;
  int dev = 0, optin = 0;
  cudaGetDevice(&dev);
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return cudaErrorInvalidValue;
  // the table blocks start at the first 64 KB boundary at or after the
  // allocation's base: the slots fit in the two pieces around them, each
  // piece losing less than one slot to the cut
  const uint32_t dyn = (uint32_t)optin;
  if (dyn < kTables + 65536u) return cudaErrorInvalidValue;
  int warps = (int)((dyn - kTables) / kSlot) - 1;
  if (warps > kUpd8MaxWarps) warps = kUpd8MaxWarps;
  if (warps < 1) return cudaErrorInvalidValue;
  cudaFuncSetAttribute(update8_kernel<G8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
  const int64_t nspan = (a.nblk + S - 1) / S;
  int64_t grid = (nspan + warps - 1) / warps;
  if (grid > sm_count) grid = sm_count;
  update8_kernel<G8><<<(int)grid, warps * 32, dyn, st>>>(a, dyn);
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
  if (n > 8 && n <= 64) {
    a.chunks = 1;
    a.ngroups = 0;
    if (n <= 16) return launch_update8<2>(a, ctx->sm_count, st);
    if (n <= 32) return launch_update8<4>(a, ctx->sm_count, st);
    return launch_update8<8>(a, ctx->sm_count, st);
  }
  // up to 8 probes (one or two four-probe groups), and above 64 in passes
  // of 16 four-probe groups
  const int ng = (n + 3) / 4;
  if (ng <= 2) {
    a.ngroups = ng;
    a.chunks = 1;
    return ng == 1 ? launch_update_ng<1, false>(a, ctx->sm_count, st)
                   : launch_update_ng<2, false>(a, ctx->sm_count, st);
  }
  a.chunks = (ng + 15) / 16;
  a.ngroups = a.chunks * 16;
  return launch_update_ng<16, true>(a, ctx->sm_count, st);
}

}  // namespace zo
