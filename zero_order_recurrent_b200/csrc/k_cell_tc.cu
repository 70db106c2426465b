// Perturbed LSTM cell on the 5th-generation tensor cores (sm_100a).
//
// For every probe-sign ps = 2*ci + s of a chunk, layer l and step t:
//   G[ps] = [x_t | h_{t-1}][ps] (W_l + (s ? -eps : eps) P_{probe})^T + (b_l +- eps p),
//   c_t = sigma(f) c_{t-1} + sigma(i) tanh(g),  h_t = sigma(o) tanh(c_t),
// i.e. one complete forward step at Theta +- eps p_i (pith.science review,
// "What carries the argument"; alex-wiki "Method").  The perturbed operand is
// never stored in HBM: the bf16 shadow tile of W_l arrives by TMA, eight
// generator warps add +-eps in place from the probe's Philox words, and
// tcgen05.mma consumes it with fp32 accumulation in tensor memory.
//
// Tile: 256 batch rows x BN gate rows (BN/4 hidden units, the four gate blocks
// side by side so the epilogue sees i, f, g, o of a unit together) x 64-deep K
// stages.  Two forms:
//   CG = 2 (cell steps and the vocabulary table): a cluster of two CTAs runs
//     one tcgen05.mma.cta_group::2 (M = 256, N = 256) per K step.  Each CTA
//     holds 128 of the rows of A and half of B (CTA 0 the gate rows of i and
//     f, CTA 1 those of g and o), loads and perturbs only that half, and
//     receives the 128 x 256 accumulator of its own rows in its tensor memory
//     (all four gates).  An accumulator takes 256 columns, so two fit: the
//     epilogue of one tile runs while the MMAs of the next fill the other.
//     The MMA is issued by one thread of CTA 0; the other CTA's generator and
//     epilogue warps arrive on CTA 0's barriers through the cluster, and MMA
//     completion is signalled to both CTAs' barriers.
//   CG = 1 (output layer + cross-entropy): one CTA, MT = 2 sub-tiles of 128
//     rows, each a tcgen05.mma.cta_group::1 (M = 128).
// Warp roles (448 threads):
//   warp 0       TMA producer (this CTA's A rows, its gate boxes of W_l)
//   warp 1       TMEM allocator; MMA issuer (CTA 0 of a pair)
//   warps 2..9   perturbation: W tile += +-eps p in shared memory, two warps
//                per SM sub-partition to hide latency
//   warps 10..13 epilogue: TMEM -> gates -> c, h (TMEM lane quadrant = warp % 4)
// Every mbarrier wait is bounded: past ~2 s the CTA raises an abort flag, the
// error word gets ZO_ERR_TIMEOUT, all roles leave their loops, and tensor
// memory is freed before exit.  No TMA copy uses a multicast form; only the
// MMA-completion commit is multicast to the two CTAs of a pair.
#include <cudaTypedefs.h>

#include "zo_common.cuh"
#include "zo_internal.h"

namespace zo {

// generator warps: eight (one W row a thread on single-CTA tiles, half a row
// on pair tiles)
// (ew = 8 on single-CTA tiles: four generator warps, two rows a thread, and
// eight epilogue warps, two per TMEM lane quadrant, each taking half the units)
__host__ __device__ constexpr int gen_warps(int cg, int ew = 4) {
  return ew == 8 ? 4 : 8;
}
__host__ __device__ constexpr int tc_threads(int cg, int ew = 4) {
  return (2 + gen_warps(cg, ew) + ew) * 32;
}
constexpr uint64_t kWaitLimitNs = kDefaultWaitNs;   // default bound of a wait

struct CellArgs {
  int K0;          // input width of the layer
  int H;
  int Ktot;        // K0 + H: row length of W_l
  int nk;          // K stages to run (K0/64 at t == 0 where h_{-1} = 0)
  int B, Bmax;
  int m_tiles, n_tiles;
  int64_t tiles;
  int group;       // probe-sign x M tiles walked together (L2 locality)
  uint64_t seed;
  int probe0;
  float eps;
  int64_t offW;    // theta offset of W_l (Philox element index base)
  const float* small_p;   // perturbed small segments
  int64_t sstride, soffb; // per probe-sign stride, offset of b_l
  float* cst;      // fp32; [P][cst_rows(Bmax)/128][H/4][128][4], MODE 2: [P][Bmax][H]
  __nv_bfloat16* hout;    // [P][Bmax][H]
  int first;       // t == 0: c_{-1} = 0
  float* raw;      // optional [P][Bmax][4H] pre-activations (then c, h are not written)
  unsigned* err;
  int gstride;     // rows between the four B boxes (H for the cell, BN/4 for the loss)
  int kbeg;        // first K stage (the input stages are skipped when a vocabulary
                   // table supplies the input term)
  const float* vt; // vocabulary table [P][vtrows][4H] fp32 (layer 0), or null
  int vtrows;
  const int32_t* tokens;   // [B][T] (with vt)
  // cross-entropy epilogue (MODE 1)
  int V, T, t;
  const int32_t* targets;  // [B][T]
  float* rowloss;          // [P][Bmax], accumulated
  const __nv_bfloat16* wsh;  // bf16 shadow of W_l (row stride Ktot), read directly with GB
  uint64_t wait_ns;        // bound of every mbarrier wait
  int stall;               // test hook: the producer issues nothing (all waits run out)
};

// Cell state of units u.. (u a multiple of 4) in the 128-row block that starts
// at batch row b0 of probe-sign ps: the state is stored
// [ps][row/128][unit/4][row%128][4] floats, so a warp's 32 consecutive rows
// of one four-unit group are 512 contiguous bytes.
__device__ __forceinline__ float* cst_quad(const CellArgs& a, int ps, int b0, int u) {
  const uint32_t nb = (uint32_t)(a.Bmax + 127) >> 7;
  const uint32_t q = ((uint32_t)ps * nb + ((uint32_t)b0 >> 7)) * ((uint32_t)a.H >> 2) + ((uint32_t)u >> 2);
  return a.cst + ((uint64_t)q << 9);
}

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits on a barrier that the other CTA of a pair arrives on: acquire at
// cluster scope, pairing with the release of mbar_arrive_cluster.
__device__ __forceinline__ bool mbar_try_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait.  Returns false (and raises the CTA abort flag) if the phase
// did not complete within limit_ns, or if another role already aborted.
// CLUSTER: the barrier also receives arrivals from the other CTA of a pair
// (acquire at cluster scope).
template <bool CLUSTER = false>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned* err, uint64_t limit_ns) {
  auto try_once = [&] { return CLUSTER ? mbar_try_cluster(bar, parity) : mbar_try(bar, parity); };
  if (try_once()) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (try_once()) return true;
    if ((i & 255) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit_ns) {
        *abort_flag = 1;
        latch(err, kErrTimeout);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Bulk prefetch of [p, p + bytes) into L2 (16-byte aligned, multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void* p, int bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// K-major operand tile in the 128-byte swizzled canonical layout: rows of
// 64 bf16 (128 B), 8-row atoms of 1024 B; SBO = 1024 B, LBO unused (1),
// descriptor version 1, layout type 2 (SWIZZLE_128B).
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// kind::f16 instruction descriptor: D fp32, A and B bf16, both K-major, M x N.
__host__ __device__ constexpr uint32_t umma_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// ---- CTA-pair (cluster of two) forms -------------------------------------
// cp.async.bulk of `bytes` (a multiple of 16, 16-byte aligned) from this CTA's
// shared memory to `dst` in another CTA of the cluster, completing `bytes`
// transactions on the barrier `bar` of that CTA (dst and bar: shared::cluster)
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst, uint32_t src, uint32_t bytes,
                                                  uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, "
      "[%3];" ::"r"(dst),
      "r"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}

// shared::cluster address of the same shared-memory offset in CTA `rank`
__device__ __forceinline__ uint32_t peer_addr(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}


// arrive on a barrier of the cluster (here: CTA 0's), releasing at cluster scope
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// M = 256 MMA over the pair: A rows 0..127 and B rows 0..N/2-1 from CTA 0's
// shared memory, the rest from CTA 1's at the same offsets; each CTA's tensor
// memory receives its own 128 rows.
__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// completion of this thread's earlier pair MMAs -> one arrival on the barrier
// at offset `bar` in both CTAs of the pair
__device__ __forceinline__ void umma_commit_pair_both(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

// ... or on this CTA's barrier only
__device__ __forceinline__ void umma_commit_pair_local(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// After tmem_wait_ld: ties each register a tcgen05.ld wrote to a point after
// the wait (the load defines them only asynchronously), so no read of them
// can be scheduled before it.  Emits no instruction.
template <int N>
__device__ __forceinline__ void tmem_regs_ready(uint32_t* r) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

__device__ __forceinline__ float tanh_fast(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float sigmoid_fast(float x) { return fmaf(0.5f, tanh_fast(0.5f * x), 0.5f); }

__device__ __forceinline__ uint32_t bf16x2_add(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hadd2(*reinterpret_cast<__nv_bfloat162*>(&a),
                             *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// ---------------------------------------------------------------------------
// Tile order: GA (probe-sign, M-tile) pairs walked together across all N tiles,
// so a wave of CTAs shares a few A panels and a few W panels.
// ---------------------------------------------------------------------------
struct TileCoord {
  int ps, m, n;
};

__device__ __forceinline__ TileCoord decode_tile(const CellArgs& a, int64_t tile, int P) {
  const int64_t pm_count = (int64_t)P * a.m_tiles;
  const int64_t per_group = (int64_t)a.group * a.n_tiles;
  const int64_t g = tile / per_group;
  const int64_t r = tile - g * per_group;
  const int64_t first = g * a.group;
  const int64_t ga = min((int64_t)a.group, pm_count - first);
  const int64_t pm = first + r % ga;
  TileCoord c;
  c.n = (int)(r / ga);
  c.ps = (int)(pm / a.m_tiles);
  c.m = (int)(pm % a.m_tiles);
  return c;
}

template <int MT, int BN, int STAGES, int ACC, int CG, int EW = 4>
struct TcCfg {
  static constexpr int U = BN / 4;                  // hidden units per tile
  static constexpr int BL = BN / CG;                // gate rows of B held by this CTA
  static constexpr int GPC = 4 / CG;                // gate blocks held by this CTA
  static constexpr int A_SUB = 128 * 128;           // one 128-row sub-tile, bytes
  static constexpr int A_BYTES = MT * A_SUB;
  static constexpr int B_BYTES = BL * 128;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int ROWS = 128 * MT * CG;        // batch rows per tile
  static constexpr int COLS = MT * BN;              // TMEM columns per accumulator
  static constexpr int TMEM_COLS = COLS * ACC;
  static constexpr int EPI = EW * 4 * U * 4;         // per epilogue warp: bias slice [4][U]
  static constexpr int SMEM = STAGES * STAGE + 1024 + 512 + EPI;
  static_assert(BN % 64 == 0 && BN <= 256, "BN");
  static_assert(CG == 1 || (CG == 2 && MT == 1 && BN == 256), "pair tiles are 256 x 256");
  static_assert(TMEM_COLS == 128 || TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM columns");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

// MODE 0: cell step.  1: output projection + cross-entropy.  2: cell step of
// layer 0 whose input term comes from the vocabulary table (added in the
// epilogue).  3: the vocabulary table itself (raw accumulators, no bias).
// XP = 1 (MODE 0, 2, 3): the perturbation as a product of its own,
// G = A W^T + A (+-eps P)^T - the K stages run twice, first over the bf16
// shadow tiles of W untouched, then over tiles the generator warps fill with
// +-bf16(eps) p (only A is loaded for those), both into one accumulator - so
// the +- pair differs by exactly the eps term instead of by the rounding of
// bf16(theta) +- eps.  Twice the MMA work of XP = 0.
//
// GB = 1 (pair tiles, XP = 0): the generator warps read their rows of the W
// tile straight from global memory into registers, three stages ahead, add
// +-eps p there and store the perturbed tile into shared memory (swizzled);
// only A arrives by TMA.  The W tile then crosses shared memory once (the
// store) instead of three times (TMA write, load, store).
template <int MT, int BN, int STAGES, int ACC, int MODE, int CG, int XP = 0, int GB = 0, int EW = 4>
__global__ void __launch_bounds__(tc_threads(CG, EW), 1)
    cell_tc_kernel(const __grid_constant__ CUtensorMap mapA0, const __grid_constant__ CUtensorMap mapA1,
                   const __grid_constant__ CUtensorMap mapW, const CellArgs a, int P) {
  using C = TcCfg<MT, BN, STAGES, ACC, CG, EW>;
  static_assert(EW == 4 || (EW == 8 && CG == 1 && MODE != 1), "eight epilogue warps: cell tiles");
  constexpr bool PAIR = CG == 2;
  constexpr int kGenWarps = gen_warps(CG, EW);
  constexpr int kGenThreads = kGenWarps * 32;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE);
  // full[s], ready[s], empty[s], acc_full[ACC], acc_empty[ACC], drain
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto ready_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto empty_bar = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
  auto accf_bar = [&](int b) { return bar0 + 8u * (3 * STAGES + b); };
  auto acce_bar = [&](int b) { return bar0 + 8u * (3 * STAGES + ACC + b); };
  const uint32_t drain_bar = bar0 + 8u * (3 * STAGES + 2 * ACC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * STAGES + 2 * ACC + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // 16-byte handshake words, one per stage, at [bar0 + 256, bar0 + 256 + 16 STAGES)
  auto hs_word = [&](int s) { return bar0 + 256u + 16u * s; };
  static_assert(8 * (3 * STAGES + 2 * ACC + 1) + 8 <= 256 && 256 + 16 * STAGES <= 512,
                "barrier area");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // position in the pair (0 issues the MMAs) and the tile walk of the pair
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const int64_t walker = PAIR ? (int64_t)cluster_id_x() : (int64_t)blockIdx.x;
  const int64_t walkers = PAIR ? (int64_t)cluster_count_x() : (int64_t)gridDim.x;
  // K stages of a tile (twice over with XP: W, then +-eps P)
  const int kend = XP ? 2 * a.nk - a.kbeg : a.nk;
  // where generator and epilogue warps report: CTA 0's barrier (through the
  // cluster from CTA 1)
  auto report = [&](uint32_t bar) {
    if (!PAIR || rank == 0)
      mbar_arrive(bar);
    else
      mbar_arrive_cluster(peer_addr(bar, 0));
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      // CTA 1's generator warps arrive on their own barrier; CTA 0's counts
      // its own generator warps and its producer, which also expects the 16
      // bytes that CTA 1 copies in once its half of the stage is ready
      mbar_init(ready_bar(s), kGenWarps + (PAIR && rank == 0 ? 1 : 0));
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < ACC; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), EW * CG);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_async_smem();
  }
  if (warp == 0 && lane == 0) {
    prefetch_map(&mapA0);
    prefetch_map(&mapA1);
    prefetch_map(&mapW);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(C::TMEM_COLS)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(C::TMEM_COLS)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  // the other CTA's barriers are initialised before anyone arrives on them
  if constexpr (PAIR) cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !a.stall) {
      uint32_t it = 0;
      bool ok = true;
      for (int64_t tile = walker; tile < a.tiles && ok; tile += walkers) {
        const TileCoord tc = decode_tile(a, tile, P);
        const int row0 = tc.m * C::ROWS + (int)rank * 128 * MT;
        for (int kb = a.kbeg; kb < kend; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait<PAIR>(empty_bar(s), ph ^ 1, abort_flag, a.err, a.wait_ns)) {
            ok = false;
            break;
          }
          const bool pstage = XP && kb >= a.nk;   // a +-eps P stage: A only
          mbar_expect_tx(full_bar(s), (pstage || GB) ? C::A_BYTES : C::STAGE);
          const uint32_t sa = sbase + s * C::STAGE;
          const uint32_t sb = sa + C::A_BYTES;
          const int kk = (pstage ? kb - a.nk + a.kbeg : kb) * 64;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            if (kk < a.K0)
              tma_load_3d(sa + mt * C::A_SUB, &mapA0, full_bar(s), kk, row0 + mt * 128, tc.ps);
            else
              tma_load_3d(sa + mt * C::A_SUB, &mapA1, full_bar(s), kk - a.K0, row0 + mt * 128,
                          tc.ps);
          }
          if (!pstage && !GB) {
#pragma unroll
            for (int gi = 0; gi < C::GPC; ++gi) {
              const int g = (int)rank * C::GPC + gi;
              tma_load_2d(sb + gi * C::U * 128, &mapW, full_bar(s), kk,
                          g * a.gstride + tc.n * C::U);
            }
          }
          // CTA 0: one arrival and the 16 bytes CTA 1's handshake copy brings
          if (PAIR && rank == 0) mbar_expect_tx(ready_bar(s), 16);
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA can exit
        const uint32_t issued = it;
        for (int s = 0; s < STAGES && (uint32_t)s < issued; ++s) {
          const uint32_t n_iss = (issued - 1 - s) / STAGES + 1;
          const uint64_t t0 = globaltimer();
          while (!mbar_try(full_bar(s), (n_iss - 1) & 1) && globaltimer() - t0 < 100000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (PAIR && lane == 0 && rank == 1) {
      // handshake: once this CTA's generator warps have perturbed their half
      // of a stage (each fenced its writes for the async proxy and arrived on
      // this CTA's barrier), copy 16 bytes into CTA 0 with cp.async.bulk; the
      // copy's completion on CTA 0's barrier is what CTA 0's MMA thread waits
      // for, the same async-proxy completion that a TMA load into one CTA
      // signalling the other CTA's barrier uses - no cluster-wide fence
      uint32_t it = 0;
      bool ok = true;
      for (int64_t tile = walker; tile < a.tiles && ok; tile += walkers) {
        for (int kb = a.kbeg; kb < kend; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(ready_bar(s), (it / STAGES) & 1, abort_flag, a.err, a.wait_ns)) {
            ok = false;
            break;
          }
          bulk_copy_to_peer(peer_addr(hs_word(s), 0), hs_word(s), 16, peer_addr(ready_bar(s), 0));
        }
      }
      // after an abort a copy may still be on its way into CTA 0: give it
      // time to land before the cluster can exit
      if (!ok) {
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 50000ull) {
        }
      }
    }
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = umma_idesc(128 * CG, BN);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int64_t tile = walker; tile < a.tiles && ok; tile += walkers, ++tcount) {
        const int ab = tcount % ACC;
        const uint32_t aph = (tcount / ACC) & 1;
        if (!mbar_wait<PAIR>(acce_bar(ab), aph ^ 1, abort_flag, a.err, a.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dcol = tmem_base + ab * C::COLS;
        for (int kb = a.kbeg; kb < kend; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait<PAIR>(ready_bar(s), ph, abort_flag, a.err, a.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = sbase + s * C::STAGE;
          const uint64_t bdesc = umma_desc(sa + C::A_BYTES);
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16) {
            const uint32_t acc = (kb != a.kbeg || k16 != 0) ? 1u : 0u;
            if constexpr (PAIR) {
              umma_bf16_pair(dcol, umma_desc(sa) + 2 * k16, bdesc + 2 * k16, idesc, acc);
            } else {
#pragma unroll
              for (int mt = 0; mt < MT; ++mt)
                umma_bf16(dcol + mt * BN, umma_desc(sa + mt * C::A_SUB) + 2 * k16, bdesc + 2 * k16,
                          idesc, acc);
            }
          }
          if constexpr (PAIR)
            umma_commit_pair_both(empty_bar(s));
          else
            umma_commit(empty_bar(s));
        }
        if (!ok) break;
        if constexpr (PAIR)
          umma_commit_pair_both(accf_bar(ab));
        else
          umma_commit(accf_bar(ab));
      }
      // all MMAs issued by this thread complete before tensor memory is freed
      if constexpr (PAIR)
        umma_commit_pair_local(drain_bar);
      else
        umma_commit(drain_bar);
      const uint64_t t0 = globaltimer();
      while (!mbar_try(drain_bar, 0) && globaltimer() - t0 < 100000000ull) {
      }
    }
  } else if (warp < 2 + kGenWarps) {
    // ------------------------------------------------------------ perturbation
    // BL >= kGenThreads: RPT rows per thread, all 8 chunks of each row;
    // BL <  kGenThreads: TPR threads share a row, CPT chunks each
    constexpr int BL = C::BL;
    constexpr int RPT = (BL + kGenThreads - 1) / kGenThreads;
    constexpr int TPR = BL >= kGenThreads ? 1 : kGenThreads / BL;
    constexpr int CPT = 8 / TPR;
    const int gt = (threadIdx.x - 64) % (BL < kGenThreads ? BL : kGenThreads);
    const int c0 = ((threadIdx.x - 64) / (BL < kGenThreads ? BL : kGenThreads)) * CPT;
    const float epsf = a.eps;
    const __nv_bfloat16 eb = __float2bfloat16_rn(epsf);
    const uint32_t eps_bits = (uint32_t)(*reinterpret_cast<const uint16_t*>(&eb));
    const uint32_t epsp2 = eps_bits | (eps_bits << 16);
    const uint32_t epsn2 = epsp2 ^ 0x80008000u;
    uint32_t it = 0;
    bool ok = true;
    if constexpr (GB) {
      // Coalesced rows: warp w owns rows w*WR .. w*WR + WR - 1 of the CTA's B
      // half; lane l reads the 16-byte chunk c = l & 7 of rows
      // w*WR + 4 i + (l >> 3), i < WR/4, so eight lanes cover a row's 128 bytes.
      // Lane l (l < WR) derives the Philox block of row w*WR + l and hands
      // the two words a row's 64 elements need to the lanes that use them.
      static_assert(PAIR && XP == 0, "direct W loads: pair tiles");
      constexpr int D = 3;                           // stages of loads in flight
      constexpr int WR = BL / kGenWarps;             // rows per warp
      constexpr int NI = WR / 4;                     // rows per lane
      const int gw = (threadIdx.x - 64) >> 5;        // generator warp 0..7
      const int c = lane & 7, rs = lane >> 3;
      const int rp = gw * WR + (lane % WR);          // the row whose Philox block this lane derives
      const int gp = (int)rank * C::GPC + rp / C::U, up = rp % C::U;
      int64_t rbase[NI];
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        const int r = gw * WR + 4 * i + rs;
        const int g = (int)rank * C::GPC + r / C::U, u = r % C::U;
        rbase[i] = (int64_t)g * a.gstride + u;
      }
      uint4 buf[D][NI];
      int64_t ltile = walker;
      int lkb = a.kbeg;
      auto issue = [&](uint4 (&dst)[NI]) {
        if (ltile < a.tiles) {
          const TileCoord lt = decode_tile(a, ltile, P);
#pragma unroll
          for (int i = 0; i < NI; ++i)
            dst[i] = __ldg(reinterpret_cast<const uint4*>(
                a.wsh + (rbase[i] + (int64_t)lt.n * C::U) * a.Ktot + (int64_t)lkb * 64 + c * 8));
          if (++lkb == a.nk) {
            lkb = a.kbeg;
            ltile += walkers;
          }
        }
      };
#pragma unroll
      for (int d = 0; d < D; ++d) issue(buf[d]);
      int64_t ctile = walker;
      int ckb = a.kbeg;
      TileCoord ct = decode_tile(a, ctile < a.tiles ? ctile : 0, P);
      int64_t cq = -1;
      uint4 cw = make_uint4(0u, 0u, 0u, 0u);
      while (ok && ctile < a.tiles) {
#pragma unroll
        for (int d = 0; d < D; ++d) {
          if (ok && ctile < a.tiles) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if (!mbar_wait(full_bar(s), ph, abort_flag, a.err, a.wait_ns)) {
              ok = false;
            } else {
              const uint32_t probe = (uint32_t)(a.probe0 + (ct.ps >> 1));
              const uint32_t e2 = (ct.ps & 1) ? epsn2 : epsp2;
              // this lane's Philox row: words of the stage's half-block
              const int64_t jp = a.offW + ((int64_t)gp * a.gstride + (int64_t)ct.n * C::U + up) *
                                              a.Ktot + (int64_t)ckb * 64;
              const int64_t q = jp >> 7;
              if (q != cq) {
                cw = sign_block(a.seed, probe, (uint64_t)q);
                cq = q;
              }
              const bool upper = (jp >> 6) & 1;
              const uint32_t wlo = upper ? cw.z : cw.x, whi = upper ? cw.w : cw.y;
              uint8_t* tileB = smem + s * C::STAGE + C::A_BYTES;
#pragma unroll
              for (int i = 0; i < NI; ++i) {
                const int r = gw * WR + 4 * i + rs;
                const uint32_t lo = __shfl_sync(0xffffffffu, wlo, 4 * i + rs);
                const uint32_t hi = __shfl_sync(0xffffffffu, whi, 4 * i + rs);
                const uint32_t w = (c < 4 ? lo : hi) >> (4 * (c & 3));
                uint4 v = buf[d][i];
                v.x = bf16x2_add(v.x, ((w << 15) & 0x80008000u) ^ e2);
                v.y = bf16x2_add(v.y, ((w << 14) & 0x80008000u) ^ e2);
                v.z = bf16x2_add(v.z, ((w << 13) & 0x80008000u) ^ e2);
                v.w = bf16x2_add(v.w, ((w << 12) & 0x80008000u) ^ e2);
                *reinterpret_cast<uint4*>(tileB + r * 128 + ((c ^ (r & 7)) << 4)) = v;
              }
              fence_async_smem();
              __syncwarp();
              if (lane == 0) mbar_arrive(ready_bar(s));
              issue(buf[d]);
              ++it;
              if (++ckb == a.nk) {
                ckb = a.kbeg;
                ctile += walkers;
                cq = -1;
                if (ctile < a.tiles) ct = decode_tile(a, ctile, P);
              }
            }
          }
        }
      }
    }
    for (int64_t tile = walker; tile < a.tiles && ok && !GB; tile += walkers) {
      const TileCoord tc = decode_tile(a, tile, P);
      const uint32_t probe = (uint32_t)(a.probe0 + (tc.ps >> 1));
      const uint32_t e2 = (tc.ps & 1) ? epsn2 : epsp2;
      int64_t cq[RPT];
      uint4 cw[RPT];
#pragma unroll
      for (int rr = 0; rr < RPT; ++rr) cq[rr] = -1;
      for (int kb = a.kbeg; kb < kend; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!mbar_wait(full_bar(s), ph, abort_flag, a.err, a.wait_ns)) {
          ok = false;
          break;
        }
        uint8_t* tileB = smem + s * C::STAGE + C::A_BYTES;
        // XP: W stages go to the MMA as loaded; +-eps P stages are written here
        const bool wstage = XP && kb < a.nk;
        const int kbk = XP && kb >= a.nk ? kb - a.nk + a.kbeg : kb;
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr) {
          const int r = gt + rr * kGenThreads;
          if (r < BL && !wstage) {
            const int g = (int)rank * C::GPC + r / C::U, u = r % C::U;
            const int64_t R = (int64_t)g * a.gstride + (int64_t)tc.n * C::U + u;
            const int64_t j0 = a.offW + R * a.Ktot + (int64_t)kbk * 64;
            const int64_t q = j0 >> 7;
            if (q != cq[rr]) {
              cw[rr] = sign_block(a.seed, probe, (uint64_t)q);
              cq[rr] = q;
            }
            const bool upper = (j0 >> 6) & 1;
            const uint32_t wlo = upper ? cw[rr].z : cw[rr].x;
            const uint32_t whi = upper ? cw[rr].w : cw[rr].y;
            uint8_t* row = tileB + r * 128;
#pragma unroll
            for (int cc = 0; cc < CPT; ++cc) {
              const int c16 = c0 + cc;
              uint4* p = reinterpret_cast<uint4*>(row + ((c16 ^ (r & 7)) << 4));
              const uint32_t w = (c16 < 4 ? wlo : whi) >> (4 * (c16 & 3));
              if (XP) {
                // the +-eps p tile itself
                *p = make_uint4(((w << 15) & 0x80008000u) ^ e2, ((w << 14) & 0x80008000u) ^ e2,
                                ((w << 13) & 0x80008000u) ^ e2, ((w << 12) & 0x80008000u) ^ e2);
              } else {
                uint4 v = *p;
                v.x = bf16x2_add(v.x, ((w << 15) & 0x80008000u) ^ e2);
                v.y = bf16x2_add(v.y, ((w << 14) & 0x80008000u) ^ e2);
                v.z = bf16x2_add(v.z, ((w << 13) & 0x80008000u) ^ e2);
                v.w = bf16x2_add(v.w, ((w << 12) & 0x80008000u) ^ e2);
                *p = v;
              }
            }
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(ready_bar(s));
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;                      // TMEM lane quadrant
    const int ew = warp - 2 - kGenWarps;               // epilogue warp 0 .. EW-1
    // units of the tile this warp finishes: all of them, or (EW = 8) one half
    constexpr int UW = C::U * 4 / EW;
    const int ubeg = EW == 8 ? (ew >> 2) * UW : 0;
    const int uend = ubeg + UW;
    const int rloc = quad * 32 + lane;
    // this warp's copy of the tile's bias slice [4 gates][U units]
    float* bias_s = reinterpret_cast<float*>(smem + STAGES * C::STAGE + 512) + ew * 4 * C::U;
    uint32_t tcount = 0;
    bool ok = true;
    for (int64_t tile = walker; tile < a.tiles && ok; tile += walkers, ++tcount) {
      const TileCoord tc = decode_tile(a, tile, P);
      const int ab = tcount % ACC;
      const uint32_t aph = (tcount / ACC) & 1;
      const int brow0 = tc.m * C::ROWS + (int)rank * 128 * MT;   // this CTA's first batch row
      if constexpr (MODE == 0 || MODE == 2) {
        // staged while the tile's MMAs run, so the epilogue's bias reads are
        // shared-memory broadcasts instead of one L2 round trip per chunk
        const float* bsrc = a.small_p + tc.ps * a.sstride + a.soffb + tc.n * C::U;
        __syncwarp();
        for (int i = lane; i < 4 * C::U; i += 32) {
          const int g = i / C::U;
          bias_s[i] = __ldg(bsrc + g * a.H + (i - g * C::U));
        }
        __syncwarp();
      }
      if ((MODE == 0 || MODE == 2) && !a.first && !a.raw) {
        // while this tile's MMAs run, pull its c_{t-1} rows (and the token's
        // vocabulary-table rows) into L2 so the epilogue's loads hit L2
        for (int mt = 0; mt < MT; ++mt) {
          const int b = brow0 + mt * 128 + rloc;
          if (b < a.B) {
            // the block's units [ubeg, ubeg + UW) are one contiguous run of
            // UW x 128 floats; each of the 128 rows' threads pulls 1/128 of it
            if constexpr (MODE == 2)
              prefetch_l2(a.cst + ((int64_t)tc.ps * a.Bmax + b) * a.H + tc.n * C::U + ubeg,
                          UW * (int)sizeof(float));
            else
              prefetch_l2(cst_quad(a, tc.ps, b - rloc, tc.n * C::U + ubeg) + rloc * UW,
                          UW * (int)sizeof(float));
            if constexpr (MODE == 2) {
              const int tok = a.tokens[(int64_t)b * a.T + a.t];
              if (tok >= 0 && tok < a.V) {
                const float* tr =
                    a.vt + ((int64_t)tc.ps * a.vtrows + tok) * 4 * a.H + tc.n * C::U + ubeg;
#pragma unroll
                for (int g = 0; g < 4; ++g) prefetch_l2(tr + g * a.H, UW * (int)sizeof(float));
              }
            }
          }
        }
      }
      if (!mbar_wait<PAIR>(accf_bar(ab), aph, abort_flag, a.err, a.wait_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* bias = a.small_p + tc.ps * a.sstride + a.soffb;
      if constexpr (MODE == 1) {
        // logits of one row live in one TMEM lane: softmax cross-entropy per row
        for (int mt = 0; mt < MT; ++mt) {
          const int b = brow0 + mt * 128 + rloc;
          uint32_t z[BN];
#pragma unroll
          for (int q = 0; q < BN / 16; ++q) {
            uint32_t (&zq)[16] = *reinterpret_cast<uint32_t(*)[16]>(z + 16 * q);
            tmem_ld16(tmem_base + ((uint32_t)(quad * 32) << 16) + ab * C::COLS + mt * BN + 16 * q,
                      zq);
          }
          tmem_wait_ld();
          tmem_regs_ready<BN>(z);
          if (b < a.B) {
            int tg = a.targets[(int64_t)b * a.T + a.t];
            if (tg >= a.V || tg < -1) {
              latch(a.err, kErrBounds);
              tg = -1;
            }
            if (tg >= 0) {
              float m = -INFINITY, zt = 0.f;
#pragma unroll
              for (int v = 0; v < BN; ++v)
                if (v < a.V) {
                  const float zv = __uint_as_float(z[v]) + __ldg(bias + v);
                  z[v] = __float_as_uint(zv);
                  m = fmaxf(m, zv);
                  if (v == tg) zt = zv;
                }
              float sum = 0.f;
#pragma unroll
              for (int v = 0; v < BN; ++v)
                if (v < a.V) sum += expf(__uint_as_float(z[v]) - m);
              a.rowloss[(int64_t)tc.ps * a.Bmax + b] += m + logf(sum) - zt;
            }
          }
        }
      } else
      for (int mt = 0; mt < MT; ++mt) {
        const int b = brow0 + mt * 128 + rloc;
        const int64_t rowoff = ((int64_t)tc.ps * a.Bmax + b) * a.H;
        const bool live = b < a.B;
        const bool need_c = live && !a.first && !a.raw;
        // this row's c: units 4q..4q+3 of the tile at crow[q * QS].  Layer 0
        // from the vocabulary table (MODE 2, whose table values fill the
        // registers the four-unit layout's address arithmetic would need)
        // keeps c row-major, [ps][row][unit]
        constexpr int QS = MODE == 2 ? 1 : 128;
        float4* crow =
            MODE == 2
                ? reinterpret_cast<float4*>(a.cst + rowoff + tc.n * C::U)
                : reinterpret_cast<float4*>(cst_quad(a, tc.ps, b - rloc, tc.n * C::U)) + rloc;
        // input term from the vocabulary table: the row of this batch row's token
        const float* trow = nullptr;
        if constexpr (MODE == 2) {
          if (live) {
            int tok = a.tokens[(int64_t)b * a.T + a.t];
            if (tok < 0 || tok >= a.V) {
              latch(a.err, kErrBounds);
              tok = 0;
            }
            trow = a.vt + ((int64_t)tc.ps * a.vtrows + tok) * 4 * a.H + tc.n * C::U;
          }
        }
        // c_{t-1} is loaded two 8-unit chunks ahead (one with the table, whose
        // loads need the registers), so its latency overlaps the TMEM loads
        // and gate arithmetic of the chunks before
        constexpr bool kTwoAhead = MODE != 2;
        float4 cn0 = make_float4(0.f, 0.f, 0.f, 0.f), cn1 = cn0, cm0 = cn0, cm1 = cn0;
        if (need_c) {
          cn0 = crow[(ubeg >> 2) * QS];
          cn1 = crow[((ubeg >> 2) + 1) * QS];
          if (kTwoAhead && ubeg + 8 < uend) {
            cm0 = crow[((ubeg >> 2) + 2) * QS];
            cm1 = crow[((ubeg >> 2) + 3) * QS];
          }
        }
#pragma unroll 1
        for (int u0 = ubeg; u0 < uend; u0 += 8) {
          // table loads issued before the TMEM loads: their latency overlaps the wait
          float4 tv[4][2];
          if constexpr (MODE == 2) {
            if (live) {
#pragma unroll
              for (int g = 0; g < 4; ++g)
#pragma unroll
                for (int q4 = 0; q4 < 2; ++q4)
                  tv[g][q4] = __ldg(reinterpret_cast<const float4*>(trow + g * a.H + u0) + q4);
            }
          }
          uint32_t acc[4][8];
#pragma unroll
          for (int g = 0; g < 4; ++g)
            tmem_ld8(tmem_base + ((uint32_t)(quad * 32) << 16) + ab * C::COLS + mt * BN +
                         g * C::U + u0,
                     acc[g]);
          const float4 cc0 = cn0, cc1 = cn1;
          if constexpr (kTwoAhead) {
            cn0 = cm0;
            cn1 = cm1;
            if (need_c && u0 + 16 < uend) {
              cm0 = crow[((u0 >> 2) + 4) * QS];
              cm1 = crow[((u0 >> 2) + 5) * QS];
            }
          } else if (need_c && u0 + 8 < uend) {
            cn0 = crow[((u0 >> 2) + 2) * QS];
            cn1 = crow[((u0 >> 2) + 3) * QS];
          }
          tmem_wait_ld();
          tmem_regs_ready<32>(&acc[0][0]);
          if (live) {
            const int unit0 = tc.n * C::U + u0;
            float pre[4][8];
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const float4* bp = reinterpret_cast<const float4*>(bias_s + g * C::U + u0);
#pragma unroll
              for (int q4 = 0; q4 < 2; ++q4) {
                float4 bv = MODE == 3 ? make_float4(0.f, 0.f, 0.f, 0.f) : bp[q4];
                if constexpr (MODE == 2) {
                  bv.x += tv[g][q4].x;
                  bv.y += tv[g][q4].y;
                  bv.z += tv[g][q4].z;
                  bv.w += tv[g][q4].w;
                }
                pre[g][4 * q4 + 0] = __uint_as_float(acc[g][4 * q4 + 0]) + bv.x;
                pre[g][4 * q4 + 1] = __uint_as_float(acc[g][4 * q4 + 1]) + bv.y;
                pre[g][4 * q4 + 2] = __uint_as_float(acc[g][4 * q4 + 2]) + bv.z;
                pre[g][4 * q4 + 3] = __uint_as_float(acc[g][4 * q4 + 3]) + bv.w;
              }
            }
            if (a.raw) {
              float* rp = a.raw + ((int64_t)tc.ps * a.Bmax + b) * 4 * a.H;
#pragma unroll
              for (int g = 0; g < 4; ++g)
#pragma unroll
                for (int q4 = 0; q4 < 2; ++q4)
                  reinterpret_cast<float4*>(rp + g * a.H + unit0)[q4] =
                      make_float4(pre[g][4 * q4], pre[g][4 * q4 + 1], pre[g][4 * q4 + 2],
                                  pre[g][4 * q4 + 3]);
            } else {
              const float cprev[8] = {cc0.x, cc0.y, cc0.z, cc0.w, cc1.x, cc1.y, cc1.z, cc1.w};
              float cn[8];
              uint32_t hp[4];
#pragma unroll
              for (int i = 0; i < 8; i += 2) {
                float hv[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const float ig = sigmoid_fast(pre[0][i + e]);
                  const float fg = sigmoid_fast(pre[1][i + e]);
                  const float gg = tanh_fast(pre[2][i + e]);
                  const float og = sigmoid_fast(pre[3][i + e]);
                  cn[i + e] = fmaf(fg, cprev[i + e], ig * gg);
                  hv[e] = og * tanh_fast(cn[i + e]);
                }
                __nv_bfloat162 pr = __floats2bfloat162_rn(hv[0], hv[1]);
                hp[i >> 1] = *reinterpret_cast<uint32_t*>(&pr);
              }
              crow[(u0 >> 2) * QS] = make_float4(cn[0], cn[1], cn[2], cn[3]);
              crow[((u0 >> 2) + 1) * QS] = make_float4(cn[4], cn[5], cn[6], cn[7]);
              *reinterpret_cast<uint4*>(a.hout + rowoff + unit0) = make_uint4(hp[0], hp[1], hp[2], hp[3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) report(acce_bar(ab));
    }
  }

  tc_fence_before();
  __syncthreads();
  // after an abort, CTA 1's handshake copies may still be landing in CTA 0
  if (PAIR && rank == 0 && threadIdx.x == 0 && *abort_flag) {
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < 50000ull) {
    }
  }
  // neither CTA of a pair leaves while the other may still read its shared
  // memory (MMA operands) or arrive on its barriers
  if constexpr (PAIR) {
    __syncthreads();
    cluster_sync_all();
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (PAIR)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(C::TMEM_COLS)
                   : "memory");
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(C::TMEM_COLS)
                   : "memory");
  }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [P][B][K] bf16 activations, box 64 (K) x 128 (rows) x 1, 128-byte swizzle.
bool map_act(CUtensorMap* m, void* base, int64_t K, int64_t B, int64_t P) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)B, (cuuint64_t)P};
  cuuint64_t strides[2] = {(cuuint64_t)(K * 2), (cuuint64_t)(K * 2 * B)};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// W_l shadow [4H][Ktot] bf16, box 64 (K) x rows.
bool map_w(CUtensorMap* m, void* base, int64_t Ktot, int64_t rows, int box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)Ktot, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(Ktot * 2)};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool make_cell_maps(zo_ctx* c) {
  const zo_model_spec& s = c->spec;
  c->maps = new (std::nothrow) CellMaps();
  if (!c->maps) return false;
  const int64_t P = 2 * (int64_t)c->chunk, B = s.max_batch, E = s.embed, H = s.hidden;
  const int L = s.layers;
  bool ok = map_act(&c->maps->x, c->x, E, B, P);
  for (int l = 0; l < L; ++l)
    for (int par = 0; par < 2; ++par)
      ok = ok && map_act(&c->maps->h[l][par], c->h + ((int64_t)l * 2 + par) * P * B * H, H, B, P);
  for (int l = 0; l < L; ++l) {
    const int64_t Ktot = (l == 0 ? E : H) + H;
    ok = ok && map_w(&c->maps->w[l], c->shadow + c->seg.off[c->seg.W[l]], Ktot, 4 * H, 64);
  }
  ok = ok && map_w(&c->maps->wout, c->shadow + c->seg.off[c->seg.Wout], H, s.vocab, 16);
  return ok;
}

template <int MT, int BN, int STAGES, int ACC, int MODE, int CG, int XP = 0, int GB = 0,
          int EW = 4>
static cudaError_t launch_cfg(const CUtensorMap& A0, const CUtensorMap& A1, const CUtensorMap& Wm,
                              CellArgs a, int P, int sms, cudaStream_t st) {
  using C = TcCfg<MT, BN, STAGES, ACC, CG, EW>;
  auto kern = cell_tc_kernel<MT, BN, STAGES, ACC, MODE, CG, XP, GB, EW>;
  a.m_tiles = (a.B + C::ROWS - 1) / C::ROWS;
  a.n_tiles = MODE != 1 ? a.H / C::U : 1;
  a.tiles = (int64_t)P * a.m_tiles * a.n_tiles;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  if constexpr (CG == 1) {
    const int64_t grid = a.tiles < sms ? a.tiles : sms;
    kern<<<(int)grid, tc_threads(CG, EW), C::SMEM, st>>>(A0, A1, Wm, a, P);
    count_launch();
    return cudaGetLastError();
  } else {
    // one cluster of two CTAs per pair of SMs, as many as can be resident
    static int max_clusters = 0;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(tc_threads(CG, EW), 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (max_clusters == 0) {
      cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = sms / 2;
      }
      max_clusters = n;
    }
    const int64_t clusters = a.tiles < max_clusters ? a.tiles : max_clusters;
    cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
    e = cudaLaunchKernelEx(&cfg, kern, A0, A1, Wm, a, P);
    count_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
}

cudaError_t launch_cell_tc(const zo_ctx* ctx, int layer, int t, int B, int nprobe, int probe0,
                           uint64_t seed, float eps, float* raw_out, const int32_t* tokens, int T,
                           bool vocab, cudaStream_t st, uint64_t wait_ns, int stall) {
  const zo_model_spec& s = ctx->spec;
  const int H = s.hidden, E = s.embed;
  const int P = 2 * nprobe;
  const int K0 = layer == 0 ? E : H;
  // with the vocabulary table, layer 0 runs only its recurrent K stages (none
  // at t = 0: that step is launch_vocab_first)
  const bool tab = vocab && layer == 0;
  if (tab && (t == 0 || !ctx->vt)) return cudaErrorInvalidValue;
  CellArgs a;
  a.wait_ns = wait_ns;
  a.stall = stall;
  a.K0 = K0;
  a.H = H;
  a.Ktot = K0 + H;
  a.nk = (t == 0 ? K0 : K0 + H) / 64;
  a.kbeg = tab ? K0 / 64 : 0;
  a.vt = tab ? ctx->vt : nullptr;
  a.vtrows = kVocabRows;
  a.tokens = tokens;
  a.B = B;
  a.Bmax = s.max_batch;
  // (probe-sign, M-tile) panels walked together, each W panel crossing HBM
  // once per group: 12 where an A panel (256 rows x the launch's K, bf16) is
  // 4 MB or more (K >= 8192: the 270M layer-1 and 1.1B launches, measured
  // ~1% faster than 8), else 8 (smaller panels measured ~1% slower with more)
  a.group = (a.nk - a.kbeg) * 64 >= 8192 ? 12 : 8;
  a.seed = seed;
  a.probe0 = probe0;
  a.eps = eps;
  a.offW = ctx->seg.off[ctx->seg.W[layer]];
  a.small_p = ctx->small_p;
  a.sstride = ctx->small.stride;
  a.soffb = ctx->small.b[layer];
  const int64_t PB = 2 * (int64_t)ctx->chunk * s.max_batch;
  a.cst = ctx->cst + (int64_t)layer * 2 * ctx->chunk * cst_rows(s.max_batch) * H;
  a.hout = ctx->h + ((int64_t)layer * 2 + (t & 1)) * PB * H;
  a.first = t == 0;
  a.raw = raw_out;
  a.err = ctx->err;
  a.V = s.vocab;
  a.T = T;
  a.t = t;
  a.targets = nullptr;
  a.rowloss = nullptr;
  const CellMaps& m = *ctx->maps;
  const CUtensorMap& A0 = layer == 0 ? m.x : m.h[layer - 1][t & 1];
  const CUtensorMap& A1 = m.h[layer][(t + 1) & 1];
  a.gstride = H;
  // 256 batch rows x 256 gate rows per tile on a CTA pair, two accumulators
  // of 256 TMEM columns per CTA, six 32 KB stages
  a.wsh = ctx->shadow + ctx->seg.off[ctx->seg.W[layer]];
  const int sms = ctx->sm_count;
  const CUtensorMap& Wm = m.w[layer];
  switch (ctx->cell_variant) {
    case ZO_CELL_SINGLE_EXACT_EPS:
      if (tab) return launch_cfg<2, 256, 3, 1, 2, 1, 1>(A0, A1, Wm, a, P, sms, st);
      return launch_cfg<2, 256, 3, 1, 0, 1, 1>(A0, A1, Wm, a, P, sms, st);
    case ZO_CELL_PAIR:
      if (tab) return launch_cfg<1, 256, 6, 2, 2, 2>(A0, A1, Wm, a, P, sms, st);
      return launch_cfg<1, 256, 6, 2, 0, 2>(A0, A1, Wm, a, P, sms, st);
    case ZO_CELL_PAIR_EXACT_EPS:
      if (tab) return launch_cfg<1, 256, 6, 2, 2, 2, 1>(A0, A1, Wm, a, P, sms, st);
      return launch_cfg<1, 256, 6, 2, 0, 2, 1>(A0, A1, Wm, a, P, sms, st);
    case ZO_CELL_PAIR_DIRECT_W:
      if (tab) return launch_cfg<1, 256, 6, 2, 2, 2, 0, 1>(A0, A1, Wm, a, P, sms, st);
      return launch_cfg<1, 256, 6, 2, 0, 2, 0, 1>(A0, A1, Wm, a, P, sms, st);
    case ZO_CELL_SINGLE_EPI8:
      if (tab) return launch_cfg<2, 256, 3, 1, 2, 1, 0, 0, 8>(A0, A1, Wm, a, P, sms, st);
      return launch_cfg<2, 256, 3, 1, 0, 1, 0, 0, 8>(A0, A1, Wm, a, P, sms, st);
    default:
      // one CTA per 256 x 256 tile: two M = 128 MMAs per K slice on one B,
      // one accumulator, three 64 KB stages
      if (tab) return launch_cfg<2, 256, 3, 1, 2, 1>(A0, A1, Wm, a, P, sms, st);
      return launch_cfg<2, 256, 3, 1, 0, 1>(A0, A1, Wm, a, P, sms, st);
  }
}

// Output projection + softmax cross-entropy for step t on the same
// tensor-core mainloop: A = h_top[t] (bf16), B = bf16(W_out) +- eps P formed
// in shared memory (V <= 64 rows, the rest zero), logits of a row in one TMEM
// lane; rowloss[ps][b] += logsumexp(z_b) - z_b[target].
cudaError_t launch_loss_tc(const zo_ctx* ctx, const int32_t* targets, int t, int B, int T,
                           int nprobe, int probe0, uint64_t seed, float eps, cudaStream_t st,
                           uint64_t wait_ns, int stall) {
  const zo_model_spec& s = ctx->spec;
  const int H = s.hidden, L = s.layers;
  const int P = 2 * nprobe;
  CellArgs a;
  a.wait_ns = wait_ns;
  a.stall = stall;
  a.K0 = H;
  a.H = H;
  a.Ktot = H;
  a.nk = H / 64;
  a.B = B;
  a.Bmax = s.max_batch;
  // (probe-sign, M-tile) panels walked together, each W panel crossing HBM
  // once per group: 12 where an A panel (256 rows x the launch's K, bf16) is
  // 4 MB or more (K >= 8192: the 270M layer-1 and 1.1B launches, measured
  // ~1% faster than 8), else 8 (smaller panels measured ~1% slower with more)
  a.group = (a.nk - a.kbeg) * 64 >= 8192 ? 12 : 8;
  a.seed = seed;
  a.probe0 = probe0;
  a.eps = eps;
  a.offW = ctx->seg.off[ctx->seg.Wout];
  a.small_p = ctx->small_p;
  a.sstride = ctx->small.stride;
  a.soffb = ctx->small.bout;
  a.cst = nullptr;
  a.hout = nullptr;
  a.first = 0;
  a.raw = nullptr;
  a.err = ctx->err;
  a.gstride = 16;
  a.kbeg = 0;
  a.vt = nullptr;
  a.vtrows = 0;
  a.tokens = nullptr;
  a.V = s.vocab;
  a.T = T;
  a.t = t;
  a.targets = targets;
  a.rowloss = ctx->rowloss;
  const CellMaps& m = *ctx->maps;
  const CUtensorMap& A0 = m.h[L - 1][t & 1];
  return launch_cfg<2, 64, 4, 2, 1, 1>(A0, A0, m.wout, a, P, ctx->sm_count, st);
}

// Vocabulary table of layer 0's input term for the chunk's probe-signs:
// vt[ps][v][:] = E'_ps[v] (W_0x +- eps P)^T, E'_ps the perturbed embedding in
// bf16, W_0x the first E columns of W_0 perturbed in shared memory as in every
// cell launch; the same mainloop with the vocabulary rows as the batch, the
// input K stages only, and the raw fp32 accumulators (no bias) as output.
cudaError_t launch_vocab_table(const zo_ctx* ctx, int nprobe, int probe0, uint64_t seed, float eps,
                               cudaStream_t st) {
  const zo_model_spec& s = ctx->spec;
  if (!ctx->vt) return cudaErrorInvalidValue;
  const int H = s.hidden, E = s.embed;
  const int P = 2 * nprobe;
  CellArgs a;
  a.wait_ns = kWaitLimitNs;
  a.stall = 0;
  a.K0 = E;
  a.H = H;
  a.Ktot = E + H;
  a.nk = E / 64;
  a.kbeg = 0;
  a.vt = nullptr;
  a.vtrows = kVocabRows;
  a.tokens = nullptr;
  a.B = s.vocab;             // live rows: the vocabulary
  a.Bmax = kVocabRows;       // row stride of the raw output
  a.group = 8;
  a.seed = seed;
  a.probe0 = probe0;
  a.eps = eps;
  a.offW = ctx->seg.off[ctx->seg.W[0]];
  a.small_p = ctx->small_p;
  a.sstride = ctx->small.stride;
  a.soffb = ctx->small.b[0];
  a.cst = nullptr;
  a.hout = nullptr;
  a.first = 1;
  a.raw = ctx->vt;
  a.err = ctx->err;
  a.V = s.vocab;
  a.T = 0;
  a.t = 0;
  a.targets = nullptr;
  a.rowloss = nullptr;
  a.gstride = H;
  const CellMaps& m = *ctx->maps;
  a.wsh = ctx->shadow + ctx->seg.off[ctx->seg.W[0]];
  const int sms = ctx->sm_count;
  switch (ctx->cell_variant) {
    case ZO_CELL_SINGLE_EXACT_EPS:
      return launch_cfg<2, 256, 3, 1, 3, 1, 1>(m.x, m.x, m.w[0], a, P, sms, st);
    case ZO_CELL_PAIR:
      return launch_cfg<1, 256, 6, 2, 3, 2>(m.x, m.x, m.w[0], a, P, sms, st);
    case ZO_CELL_PAIR_EXACT_EPS:
      return launch_cfg<1, 256, 6, 2, 3, 2, 1>(m.x, m.x, m.w[0], a, P, sms, st);
    case ZO_CELL_PAIR_DIRECT_W:
      return launch_cfg<1, 256, 6, 2, 3, 2, 0, 1>(m.x, m.x, m.w[0], a, P, sms, st);
    case ZO_CELL_SINGLE_EPI8:
      return launch_cfg<2, 256, 3, 1, 3, 1, 0, 0, 8>(m.x, m.x, m.w[0], a, P, sms, st);
    default:
      return launch_cfg<2, 256, 3, 1, 3, 1>(m.x, m.x, m.w[0], a, P, sms, st);
  }
}

}  // namespace zo
