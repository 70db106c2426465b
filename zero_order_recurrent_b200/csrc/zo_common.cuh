// Shared device helpers for the CD-RGE kernels: the probe-sign generator,
// error latching and small numeric helpers.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/zo.h"

namespace zo {

// Device error word bits (latched with atomicOr, read by zo_sync_status).
enum : unsigned {
  kErrTimeout = 1u,
  kErrBounds = 2u,
  kErrNonfinite = 4u,
};

// Upper bound on parameter segments: E, (W_l, b_l) x 8 layers, W_out, b_out.
constexpr int kMaxLayers = 8;
constexpr int kMaxSeg = 2 + 2 * kMaxLayers;

// Philox4x32-10 (Salmon, Moraes, Dror & Shaw, SC'11).  One round maps
// (c0, c1, c2, c3) with key (k0, k1) to
//   (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0));
// the key advances by the Weyl constants between rounds.
constexpr uint32_t kPhiloxM0 = 0xD2511F53u;
constexpr uint32_t kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u;
constexpr uint32_t kPhiloxW1 = 0xBB67AE85u;

__device__ __forceinline__ uint4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                               uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += kPhiloxW0;
      k1 += kPhiloxW1;
    }
    const uint32_t hi0 = __umulhi(kPhiloxM0, c0), lo0 = kPhiloxM0 * c0;
    const uint32_t hi1 = __umulhi(kPhiloxM1, c2), lo1 = kPhiloxM1 * c2;
    const uint32_t n0 = hi1 ^ c1 ^ k0;
    const uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return make_uint4(c0, c1, c2, c3);
}

// The four sign words of 128-element block q of probe i: counter
// (q lo, q hi, i, 0), key (seed lo, seed hi).
__device__ __forceinline__ uint4 sign_block(uint64_t seed, uint32_t probe, uint64_t q) {
  return philox4x32_10((uint32_t)q, (uint32_t)(q >> 32), probe, 0u, (uint32_t)seed,
                       (uint32_t)(seed >> 32));
}

__device__ __forceinline__ uint32_t word_of(const uint4& w, int idx) {
  return idx == 0 ? w.x : idx == 1 ? w.y : idx == 2 ? w.z : w.w;
}

// Bit position of element e (0..31) inside its word: elements 2m and 2m+1
// sit at bits m and m + 16, so one shift lines a bf16 pair up with the sign
// bits (15, 31) of a packed bf16x2.
__device__ __forceinline__ int bit_pos(int e) { return (e >> 1) + ((e & 1) << 4); }

// Sign bit (1 means p = -1) of element j given its block's words.
__device__ __forceinline__ uint32_t sign_bit(const uint4& w, int64_t j) {
  const int e = (int)(j & 31);
  return (word_of(w, (int)((j >> 5) & 3)) >> bit_pos(e)) & 1u;
}

// p_ij as +-1.0f, computing the block on the spot (for scattered elements).
__device__ __forceinline__ float sign_at(uint64_t seed, uint32_t probe, int64_t j) {
  const uint4 w = sign_block(seed, probe, (uint64_t)(j >> 7));
  return sign_bit(w, j) ? -1.f : 1.f;
}

// x with its sign flipped when bit 31 of m is set.
__device__ __forceinline__ float flip_sign(float x, uint32_t m) {
  return __uint_as_float(__float_as_uint(x) ^ (m & 0x80000000u));
}

__device__ __forceinline__ void latch(unsigned* err, unsigned bit) {
  if (err) atomicOr(err, bit);
}

__device__ __forceinline__ float sigmoid_acc(float x) { return 1.f / (1.f + expf(-x)); }

}  // namespace zo
