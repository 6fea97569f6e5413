// nm_gemm2.cuh -- persistent 2-CTA sparse GEMM (tcgen05 cta_group::2) for
// the large (prefill) shapes.
//
// A cluster of two CTAs (on two SMs) computes 256 x BN output tiles:
//   CTA rank r holds A rows [256 tm + 128 r, +128) and B rows
//   [BN tn + (BN/2) r, +BN/2); the leader (rank 0) issues one
//   tcgen05.mma.sp.cta_group::2 per K = 32 slice and both CTAs receive their
//   128 x BN half of the product in their own tensor memory.
// Per SM this reads A 4 KB + B 8 KB (BN = 256) of shared memory per 128-cycle
// MMA, below the shared-memory port; a one-SM 128 x 128 tile needs about
// 1.5x the port for 2:4 operands, which is why this kernel exists.
//
// Pipelines (bounded waits everywhere):
//   smem ring  : full[s] lives in the leader and counts both CTAs' TMA bytes
//                (TMA .cta_group::2 signals the leader's barrier, no multicast);
//                empty[s] in both CTAs is arrived by the leader's commit,
//                multicast to the pair.
//   accumulator: NACC buffers; tmem_full[b] in both CTAs (leader commit,
//                multicast); tmem_empty[b] in the leader, arrived remotely by
//                the 4 epilogue warps of both CTAs.
// Tiles are visited A-block fastest so that concurrently running clusters
// share the B tile (the larger, streamed operand) through L2.
//
// FP8 = true runs the 8-bit product (tcgen05.mma.sp kind::f8f6f4, E4M3 x
// E4M3): a k-block is then 256 lifted K -- the same bytes per stage as a
// 128-K bf16 block -- with four K = 64 MMAs, two 16-byte-per-row metadata
// blocks per 128 rows (tensor-memory columns +2 per MMA), and the epilogue
// multiplies the accumulator by the row scale of A and the column scale of B.
//
// LIFT = true is the in-GEMM lift of the weight-side (2n-2):2n product: B,
// the lifted activations, is not read from a lifted copy in global memory.
// Eight more warps ("lift warps", 256 threads per CTA) fill each stage's B
// half themselves, from the raw activations X [rows_b][K] (row stride
// lift_ldx), in the layout the TMA would have left: lifted column j of a
// k-block is raw column g M + 2w + (j % 4) with (g, w) the group and window of
// lifted window j / 4, rows and columns past the operand zero.  A lane takes
// one window (8 bytes) of a 128-lifted-column row, so that one instruction of
// a warp reads about 170 consecutive bytes of X; the copies are asynchronous
// global -> shared copies (cp.async, one of 8 bytes or two of 4 by the
// source's alignment, zero-filled past the operand) written straight into
// the swizzled stage, so no register holds the data and several stages are
// in flight at once.  Each lift thread then arrives on its CTA's lift
// barrier when its copies have landed; one more warp per CTA (the forwarder)
// waits on it, fences the async proxy and arrives on the leader's full
// barrier (two arrivals per stage besides the producer's).  The summation
// order is that of the TMA-fed product, so results are equal bit for bit.
//
// MSUB = 2 makes the tile 512 x BN: each k-slice issues two M = 256 MMAs that
// share the B stage (CTA r holds A rows 512 tm + 256 u + 128 r for u = 0, 1).
// That cuts the shared-memory fill per MMA cycle from 64 + 8192/BN to
// 32 + 8192/BN bytes per SM, which is what the L2 -> SM path can sustain;
// tensor memory then holds one accumulator set (NACC = 1).
#pragma once
#include <type_traits>

#include "nm_device.cuh"

namespace nm {

__device__ __forceinline__ uint32_t cluster_rank_2() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t leader_addr(uint32_t local) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(r) : "r"(local));
  return r;
}
// TMA 2D load into this CTA's smem, completion bytes counted on the barrier
// at shared::cluster address `bar_cluster` (the leader's).
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap* m, uint32_t bar_cluster, void* dst,
                                                 int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" :: "r"(bar_cluster) : "memory");
}
__device__ __forceinline__ void tmem_alloc2(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
               :: "r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
      :: "r"(smem_u32(bar)), "h"(static_cast<uint16_t>(3)) : "memory");
}
__device__ __forceinline__ void tc_cp_pair_128x128b(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;" :: "r"(taddr), "l"(desc) : "memory");
}
__device__ __forceinline__ void tc_mma_sp_pair_e4m3(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                    uint32_t e_tmem, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.sp.cta_group::2.kind::f8f6f4 [%0], %1, %2, [%5], %3, p;\n\t}"
      :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(e_tmem)
      : "memory");
}
__device__ __forceinline__ void tc_mma_sp_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t e_tmem,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.sp.cta_group::2.kind::f16 [%0], %1, %2, [%5], %3, p;\n\t}"
      :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(e_tmem)
      : "memory");
}

// TMA 2D store smem -> global (bulk-group completion; the group waits are in
// nm_device.cuh).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, const void* src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
               :: "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(src)), "r"(x), "r"(y) : "memory");
}

__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct Gemm2Args {
  int64_t rows_a, rows_b;
  int kb;                 // sparse k-blocks (128 lifted K each), then kb_dense dense ones (64 K each)
  int kb_dense;
  int64_t k_dense_x0;     // B column where the dense part starts
  int64_t meta_kb;        // metadata blocks per 128-row block
  int tiles_m, tiles_n;
  void* Y;
  int64_t ldy;
  int out_fp32;
  int transpose_out;
  int tma_store;          // 1: bf16 row-major Y written by TMA from a staging tile;
                          // 2: the same for Y stored transposed (Y[b][a])
  const float* scale_a;   // 8-bit product: per-row scale of A (nullptr: none); bf16 product:
                          // the row scale of the affine epilogue (nullptr: none)
  const float* scale_b;   // 8-bit product: per-row scale of B, i.e. per output column
  const float* shift_a;   // bf16 affine epilogue: y = acc * scale_a[a] + shift_a[a] * sum_b[b]
  const float* sum_b;
  int last_half;          // 8-bit product: the last k-block holds only 128 lifted K
  int out_split_tiles;    // output-split (-1: none): output m-tiles below it are 2:4 rows
                          // (sparse k-blocks only), the rest dense rows (dense k-blocks
                          // only, A rows counted from the dense matrix's first row, B from
                          // column 0)
  // Split last round (stream-K tail; sk_parts < 2: none).  Tiles [0, sk_full)
  // run whole in persistent rounds (sk_full is a multiple of the cluster
  // count); in the round after them, cluster u takes k-part u % sk_parts of
  // tile sk_full + u / sk_parts and leaves its fp32 accumulator in sk_ws
  // (unit ((tile - sk_full) * sk_parts + part), [256 MSUB rows][BN], no epilogue
  // scaling); k_sk_fixup sums the parts and writes those tiles of Y.
  int sk_full;
  int sk_parts;
  float* sk_ws;
};

// In-GEMM lift parameters (LIFT = true only; the other instantiations keep
// the plain parameter type).
struct Gemm2LiftArgs : Gemm2Args {
  const uint16_t* lift_x;   // raw activations [rows_b][lift_k], bf16
  int64_t lift_ldx;         // row stride of lift_x, elements
  int64_t lift_k;           // raw K
  int lift_m;               // group size M of the (2n-2):2n pattern
};
constexpr int kLiftWarps2 = 8;
constexpr int kLiftThreads2 = 192 + 32 * kLiftWarps2 + 32;   // + the forwarder warp
enum : unsigned { kWhereLift2 = 4 };

// Asynchronous global -> shared copies of 4 or 8 bytes (zero-filled when
// `valid` is false: no byte is read), and the arrival on an mbarrier once the
// calling thread's earlier copies have landed (counted in the barrier's
// arrival count).
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" :: "r"(dst), "l"(src), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_8(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" :: "r"(dst), "l"(src), "r"(valid ? 8 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" :: "r"(smem_u32(bar)) : "memory");
}

// The tile a cluster takes in its round j of the persistent loop: round j
// covers tiles [j P, j P + P) for P clusters.  Output-split products, whose
// tiles differ in length (dense tiles first, then 2:4 ones), run the odd
// rounds in reverse cluster order, so that the clusters that took the longest
// tiles in one round take the shortest in the next (the sequence increases,
// so the first index past the end closes the loop).
__device__ __forceinline__ int tile2_at(int round, int cluster, int clusters, int out_split_tiles) {
  const bool rev = out_split_tiles >= 0 && (round & 1);
  return round * clusters + (rev ? clusters - 1 - cluster : cluster);
}

// One m-tile's place: the output tile index, the tile index inside its A
// matrix, and its k-blocks [kb_lo, kb_hi).  Output-split products schedule
// their dense tiles (twice the bytes of a 2:4 tile) first.
struct Tile2 {
  int out, a, kb_lo, kb_hi;
};
__device__ __forceinline__ Tile2 tile2_of(const Gemm2Args& g, int tm) {
  const int tsp = g.out_split_tiles;
  if (tsp < 0) return {tm, tm, 0, g.kb + g.kb_dense};
  const int nd = g.tiles_m - tsp;
  if (tm < nd) return {tsp + tm, tm, g.kb, g.kb + g.kb_dense};
  return {tm - nd, tm - nd, 0, g.kb};
}

// The j-th piece of work of a cluster: an output tile (t < 0: no more work),
// its k-block range, and its stream-K part (-1: the whole tile).
struct Work2 {
  int t, part;
  Tile2 tl;
};
__device__ __forceinline__ Work2 work2_at(const Gemm2Args& g, int j, int cluster, int clusters) {
  const int tiles = g.tiles_m * g.tiles_n;
  Work2 w{-1, -1, {0, 0, 0, 0}};
  if (g.sk_parts > 1 && j >= g.sk_full / clusters) {
    if (j > g.sk_full / clusters) return w;
    const int t = g.sk_full + cluster / g.sk_parts;
    if (t >= tiles) return w;
    w.t = t;
    w.part = cluster % g.sk_parts;
    w.tl = tile2_of(g, t % g.tiles_m);
    const int lo = w.tl.kb_lo, n = w.tl.kb_hi - w.tl.kb_lo;
    w.tl.kb_lo = lo + n * w.part / g.sk_parts;
    w.tl.kb_hi = lo + n * (w.part + 1) / g.sk_parts;
    return w;
  }
  const int t = tile2_at(j, cluster, clusters, g.out_split_tiles);
  if (t >= tiles) return w;
  w.t = t;
  w.tl = tile2_of(g, t % g.tiles_m);
  return w;
}

template <int BN, int NACC, int MSUB, bool FP8 = false>
struct Gemm2Cfg {
  static constexpr int kHalfN = BN / 2;
  static constexpr int kA1 = 128 * 128;                // one subtile: 128 rows x 128 stored bytes
  static constexpr int kA = MSUB * kA1;
  static constexpr int kB = 2 * kHalfN * 128;          // two 128-byte-wide column halves
  static constexpr int kEBlocks = FP8 ? 2 : 1;         // 128-K metadata blocks per k-block
  static constexpr int kE = MSUB * 2048 * kEBlocks;
  static constexpr int kStage = kA + kB + kE;
  static constexpr int kStaging = 4 * 2 * 32 * 32 * 2;  // 4 epilogue warps x 2 buffers x 32x32 bf16
  static constexpr int kStagesRaw = (232448 - kStaging - 2048) / kStage;
  static constexpr int kStages = kStagesRaw > 6 ? 6 : kStagesRaw;
  static constexpr int kTmemCols = 512;
  static constexpr int kAccStride = 256;               // accumulator (b, u) at column 256 (b MSUB + u)
  static constexpr int kMetaCol = (NACC * MSUB - 1) * kAccStride + BN;
  static constexpr int kMetaCols = 4 * kEBlocks * MSUB;   // metadata columns per stage
  static constexpr int kSmem = kStages * kStage + kStaging + 1024 + 512;
  static_assert(NACC * MSUB <= 2, "two accumulators of up to 256 columns");
  static_assert(kMetaCol + kMetaCols * kStages <= kTmemCols, "tensor memory budget");
  static_assert(kHalfN % 8 == 0 && BN % 16 == 0 && BN <= 256, "MMA N");
  static_assert(kStages >= 3, "ring too shallow");
};

// Issues the copies of one stage's B half for the in-GEMM lift (lift warps,
// 256 threads): rows [y0, y0 + BN/2) of the lifted activations, lifted
// columns [128 kb, 128 kb + 128), into the two 128-byte-swizzled column
// halves at sB_stage.  Lane l copies window 32 kb + l of rows w, w + 8, ...
// (w the lift warp).
template <int BN>
__device__ __forceinline__ void lift_stage_b(const Gemm2LiftArgs& args, int kb, int64_t y0, uint8_t* sB_stage) {
  constexpr int HN = BN / 2;
  const int t = static_cast<int>(threadIdx.x) - 192;     // 0 .. 255
  const int lw = t / 32, lane = t % 32;
  // 32-bit index arithmetic: K' / 4 < 2^31 (host check)
  const uint32_t M = static_cast<uint32_t>(args.lift_m);
  const uint32_t nw = M / 2 - 1;
  const uint32_t nwin = static_cast<uint32_t>(args.lift_k / args.lift_m) * nw;   // lifted windows per row
  const uint32_t q = static_cast<uint32_t>(kb) * 32u + static_cast<uint32_t>(lane);
  const uint32_t g = q / nw, w = q - g * nw;
  const bool q_ok = q < nwin;
  const int64_t e0 = q_ok ? static_cast<int64_t>(g) * M + 2 * w : 0;    // raw element of the window
  const bool wide = (e0 % 4) == 0;                        // the window's 8 source bytes are 8-byte aligned
  // destination: chunk lane / 2 of the 128-column row (half lane / 16), its
  // lower or upper 8 bytes
  const int c = lane / 2, h = c / 8, c8 = c % 8;
  const uint32_t sb = smem_u32(sB_stage) + h * (HN * 128) + 8 * (lane % 2);
  const uint16_t* x = args.lift_x;
  for (int rr = lw; rr < HN; rr += kLiftWarps2) {
    const int64_t row = y0 + rr;
    const bool ok = q_ok && row < args.rows_b;
    const uint16_t* src = x + (ok ? row * args.lift_ldx + e0 : 0);
    const uint32_t dst = sb + rr * 128 + 16 * (c8 ^ (rr % 8));
    if (wide) {
      cp_async_8(dst, src, ok);
    } else {
      cp_async_4(dst, src, ok);
      cp_async_4(dst + 4, src + 2, ok);
    }
  }
}

template <int BN, int NACC, int MSUB, bool FP8 = false, bool LIFT = false>
__global__ void __launch_bounds__(LIFT ? kLiftThreads2 : 192, 1)
k_nm_gemm_2cta(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmY,
               const __grid_constant__ CUtensorMap tmAd,
               const std::conditional_t<LIFT, Gemm2LiftArgs, Gemm2Args> args) {
  static_assert(!LIFT || (!FP8 && MSUB == 1), "in-GEMM lift: bf16, 256-row tiles");
  using Cfg = Gemm2Cfg<BN, NACC, MSUB, FP8>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw2[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw2) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + S * Cfg::kA;
  uint8_t* sE = sB + S * Cfg::kB;
  uint8_t* sY = sE + S * Cfg::kE;                    // epilogue staging (1024-aligned)
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(sY + Cfg::kStaging);
  uint64_t* empty_bar = full_bar + S;
  uint64_t* tfull_bar = empty_bar + S;
  uint64_t* tempty_bar = tfull_bar + NACC;
  uint64_t* lift_bar = tempty_bar + NACC;            // in-GEMM lift: the stage's copies have landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lift_bar + (LIFT ? S : 0));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_rank_2();
  const bool leader = rank == 0;
  const int cluster_id = blockIdx.x / 2;
  const int num_clusters = gridDim.x / 2;
  const int tiles = args.tiles_m * args.tiles_n;

  if (threadIdx.x == 0) {
    // full: the producer's expect_tx arrival, plus (in-GEMM lift) the
    // forwarder's of both CTAs; lift: one arrival per lift thread, made when
    // its copies of the stage have landed
    for (int s = 0; s < S; ++s) { mbar_init(&full_bar[s], LIFT ? 3 : 1); mbar_init(&empty_bar[s], 1); }
    if (LIFT)
      for (int s = 0; s < S; ++s) mbar_init(&lift_bar[s], 32 * kLiftWarps2);
    for (int b = 0; b < NACC; ++b) { mbar_init(&tfull_bar[b], 1); mbar_init(&tempty_bar[b], 8); }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA); prefetch_tmap(&tmB); prefetch_tmap(&tmE);
    if (args.tma_store) prefetch_tmap(&tmY);
    if (args.kb_dense > 0) prefetch_tmap(&tmAd);
  }
  if (warp == 1) { tmem_alloc2(tmem_slot, Cfg::kTmemCols); tmem_relinquish2(); }
  tc_fence_before();
  cluster_barrier();          // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tmem_meta = tmem_base + Cfg::kMetaCol;
  griddep_launch_dependents();
  griddep_wait();                                    // operands and Y belong to the preceding kernel until it ends

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      const uint32_t stage_tx = static_cast<uint32_t>(2 * (Cfg::kA + Cfg::kB + Cfg::kE));
      const uint32_t dense_tx = static_cast<uint32_t>(2 * (MSUB * Cfg::kA1 + Cfg::kHalfN * 128));
      int it = 0;
      bool ok = true;
      for (int j = 0; ok; ++j) {
        const Work2 wk = work2_at(args, j, cluster_id, num_clusters);
        if (wk.t < 0) break;
        const Tile2 tl = wk.tl;
        const int tm = tl.a, tn = wk.t / args.tiles_m;
        const int32_t yb = tn * BN + static_cast<int32_t>(rank) * Cfg::kHalfN;
        for (int kb = tl.kb_lo; kb < tl.kb_hi; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
          if (!mbar_wait(&empty_bar[s], ph ^ 1u, abort_flag, kWhereProducer)) { ok = false; break; }
          const uint32_t fb = leader_addr(smem_u32(&full_bar[s]));
          if (kb >= args.kb) {
            // dense k-block: 64 K of A (per subtile) and of the B half
            const int kd = kb - args.kb;
            if (leader) mbar_arrive_expect_tx(&full_bar[s], dense_tx);
#pragma unroll
            for (int u = 0; u < MSUB; ++u) {
              const int64_t rb = (static_cast<int64_t>(tm) * MSUB + u) * 2 + rank;
              tma_load_2d_pair(&tmAd, fb, sA + s * Cfg::kA + u * Cfg::kA1, kd * 64, static_cast<int32_t>(rb * 128));
            }
            tma_load_2d_pair(&tmB, fb, sB + s * Cfg::kB, static_cast<int32_t>(args.k_dense_x0) + kd * 64, yb);
            continue;
          }
          if constexpr (FP8) {
            // 256 lifted K: A 128 stored bytes, B two 128-byte halves, two
            // metadata blocks (one when the last block holds only 128 K)
            const int eb = (args.last_half && kb == args.kb - 1) ? 1 : 2;
            if (leader)
              mbar_arrive_expect_tx(&full_bar[s],
                                    static_cast<uint32_t>(2 * (Cfg::kA + Cfg::kB / 2 * eb + MSUB * 2048 * eb)));
#pragma unroll
            for (int u = 0; u < MSUB; ++u) {
              const int64_t rb = (static_cast<int64_t>(tm) * MSUB + u) * 2 + rank;
              tma_load_2d_pair(&tmA, fb, sA + s * Cfg::kA + u * Cfg::kA1, kb * 128, static_cast<int32_t>(rb * 128));
              for (int e = 0; e < eb; ++e)
                tma_load_2d_pair(&tmE, fb, sE + s * Cfg::kE + (u * 2 + e) * 2048, 0,
                                 static_cast<int32_t>((rb * args.meta_kb + 2 * kb + e) * 16));
            }
            tma_load_2d_pair(&tmB, fb, sB + s * Cfg::kB, kb * 256, yb);
            if (eb == 2) tma_load_2d_pair(&tmB, fb, sB + s * Cfg::kB + Cfg::kHalfN * 128, kb * 256 + 128, yb);
          } else {
            // in-GEMM lift: B comes from the lift warps, the TMA brings A and metadata
            if (leader) mbar_arrive_expect_tx(&full_bar[s], LIFT ? stage_tx - 2 * Cfg::kB : stage_tx);
#pragma unroll
            for (int u = 0; u < MSUB; ++u) {
              const int64_t rb = (static_cast<int64_t>(tm) * MSUB + u) * 2 + rank;     // 128-row block
              tma_load_2d_pair(&tmA, fb, sA + s * Cfg::kA + u * Cfg::kA1, kb * 64, static_cast<int32_t>(rb * 128));
              tma_load_2d_pair(&tmE, fb, sE + s * Cfg::kE + u * 2048, 0,
                               static_cast<int32_t>((rb * args.meta_kb + kb) * 16));
            }
            if constexpr (!LIFT) {
              tma_load_2d_pair(&tmB, fb, sB + s * Cfg::kB, kb * 128, yb);
              tma_load_2d_pair(&tmB, fb, sB + s * Cfg::kB + Cfg::kHalfN * 128, kb * 128 + 64, yb);
            }
          }
        }
      }
      // Every stage this CTA filled was released by the leader's commit
      // (multicast to both CTAs) before the CTA may exit: wait for the last
      // S releases so no arrival is still in flight.
      for (int j = (it > S ? it - S : 0); j < it; ++j)
        mbar_wait(&empty_bar[j % S], static_cast<uint32_t>(j / S) & 1u, nullptr, kWhereProducer, 200000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA (leader)
    if (leader && elect_one()) {
      const uint32_t idesc = idesc_bf16(256, BN, true);
      const uint32_t idesc_dn = idesc_bf16(256, BN, false);
      int it = 0, lt = 0;
      bool ok = true;
      for (int j = 0; ok; ++j, ++lt) {
        const Work2 wk = work2_at(args, j, cluster_id, num_clusters);
        if (wk.t < 0) break;
        const Tile2 tl = wk.tl;
        const int b = lt % NACC;
        const uint32_t use = static_cast<uint32_t>(lt / NACC);
        if (!mbar_wait(&tempty_bar[b], (use & 1u) ^ 1u, abort_flag, kWhereMma)) break;
        tc_fence_after();
        const uint32_t acc = tmem_base + b * MSUB * Cfg::kAccStride;
        for (int kb = tl.kb_lo; kb < tl.kb_hi; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
          const uint32_t accum0 = kb > tl.kb_lo ? 1u : 0u;     // the tile's first k-block overwrites
          if (!mbar_wait<LIFT>(&full_bar[s], ph, abort_flag, kWhereMma)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * Cfg::kA);
          const uint32_t b0 = smem_u32(sB + s * Cfg::kB);
          if (kb >= args.kb) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t bd = desc_sw128_kmajor(b0 + 32u * kk);
#pragma unroll
              for (int u = 0; u < MSUB; ++u) {
                const uint64_t ad = desc_sw128_kmajor(a0 + u * Cfg::kA1 + 32u * kk);
                tc_mma_pair(acc + u * Cfg::kAccStride, ad, bd, idesc_dn, (accum0 | static_cast<uint32_t>(kk > 0)));
              }
            }
            tc_commit_pair(&empty_bar[s]);
            continue;
          }
          const uint32_t e_col = tmem_meta + static_cast<uint32_t>(Cfg::kMetaCols) * s;
          if constexpr (FP8) {
            // metadata block e of subtile u -> columns e_col + 8u + 4e; MMA kk
            // (64 lifted K) reads its two columns at e_col + 8u + 2kk
            const int nkk = (args.last_half && kb == args.kb - 1) ? 2 : 4;
#pragma unroll
            for (int u = 0; u < MSUB; ++u)
              for (int e = 0; e < nkk / 2; ++e)
                tc_cp_pair_128x128b(e_col + 8u * u + 4u * e,
                                    desc_plain_128x16(smem_u32(sE + s * Cfg::kE + (u * 2 + e) * 2048)));
            const uint32_t idesc8 = idesc_e4m3(256, BN, true);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              if (kk < nkk) {
                const uint64_t bd = desc_sw128_kmajor(b0 + (kk / 2) * (Cfg::kHalfN * 128) + (kk % 2) * 64);
#pragma unroll
                for (int u = 0; u < MSUB; ++u) {
                  const uint64_t ad = desc_sw128_kmajor(a0 + u * Cfg::kA1 + 32u * kk);
                  tc_mma_sp_pair_e4m3(acc + u * Cfg::kAccStride, ad, bd, e_col + 8u * u + 2u * kk, idesc8,
                                      (accum0 | static_cast<uint32_t>(kk > 0)));
                }
              }
            }
          } else {
#pragma unroll
            for (int u = 0; u < MSUB; ++u)
              tc_cp_pair_128x128b(e_col + 4u * u, desc_plain_128x16(smem_u32(sE + s * Cfg::kE + u * 2048)));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t bd = desc_sw128_kmajor(b0 + (kk / 2) * (Cfg::kHalfN * 128) + (kk % 2) * 64);
#pragma unroll
              for (int u = 0; u < MSUB; ++u) {
                const uint64_t ad = desc_sw128_kmajor(a0 + u * Cfg::kA1 + 32u * kk);
                tc_mma_sp_pair(acc + u * Cfg::kAccStride, ad, bd, e_col + 4u * u + (kk & ~1),
                               idesc | static_cast<uint32_t>(kk & 1), (accum0 | static_cast<uint32_t>(kk > 0)));
              }
            }
          }
          tc_commit_pair(&empty_bar[s]);
        }
        if (ok) tc_commit_pair(&tfull_bar[b]);
      }
    }
  } else if (LIFT && warp >= 6) {
    // ------------------------------------- lift warps and their forwarder
    if constexpr (LIFT) {
      const bool forwarder = warp == 6 + kLiftWarps2;
      if (!forwarder || lane == 0) {
        int it = 0;
        bool ok = true;
        for (int j = 0; ok; ++j) {
          const Work2 wk = work2_at(args, j, cluster_id, num_clusters);
          if (wk.t < 0) break;
          const int tn = wk.t / args.tiles_m;
          const int64_t y0 = static_cast<int64_t>(tn) * BN + static_cast<int64_t>(rank) * Cfg::kHalfN;
          for (int kb = wk.tl.kb_lo; kb < wk.tl.kb_hi; ++kb, ++it) {
            const int s = it % S;
            const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
            if (forwarder) {
              // the lift threads' copies of this stage have landed: publish
              // them to the tensor cores of the pair
              if (!mbar_wait(&lift_bar[s], ph, abort_flag, kWhereLift2)) { ok = false; break; }
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
              mbar_arrive_cluster(leader_addr(smem_u32(&full_bar[s])));
            } else {
              if (!mbar_wait(&empty_bar[s], ph ^ 1u, abort_flag, kWhereLift2)) { ok = false; break; }
              lift_stage_b<BN>(args, kb, y0, sB + s * Cfg::kB);
              cp_async_arrive_noinc(&lift_bar[s]);
            }
          }
        }
        // copies still in flight land before the CTA may exit
        if (!forwarder) asm volatile("cp.async.wait_all;" ::: "memory");
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp % 4;
    const uint32_t tempty_leader0 = leader_addr(smem_u32(&tempty_bar[0]));
    const uint32_t tempty_leader1 = leader_addr(smem_u32(&tempty_bar[NACC > 1 ? 1 : 0]));
    int lt = 0;
    uint32_t ebuf = 0;                                // staging tiles issued by this warp
    GemmArgs st{};
    st.rows_a = args.rows_a;
    st.rows_b = args.rows_b;
    st.Y = args.Y;
    st.ldy = args.ldy;
    st.out_fp32 = args.out_fp32;
    st.transpose_out = args.transpose_out;
    for (int j = 0;; ++j, ++lt) {
      const Work2 wk = work2_at(args, j, cluster_id, num_clusters);
      if (wk.t < 0) break;
      const int tm = wk.tl.out, tn = wk.t / args.tiles_m;
      const int b = lt % NACC;
      const uint32_t use = static_cast<uint32_t>(lt / NACC);
      if (!mbar_wait_warp(&tfull_bar[b], use & 1u, abort_flag, kWhereEpilogue)) break;
      tc_fence_after();
      if constexpr (NACC == 1 && MSUB == 1 && !FP8 && !LIFT) {
        // One accumulator: the next tile's MMAs wait for it.  A plain bf16
        // tile is read out whole into registers (BN / 2 bf16 pairs per
        // thread) and the accumulator released before the stores, so the
        // stores overlap the next tile's MMAs.
        if (wk.part < 0 && args.tma_store != 0 && args.scale_a == nullptr) {
          const int64_t row0 = static_cast<int64_t>(tm) * 256 + rank * 128 + q * 32;
          const uint32_t acc = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
          uint32_t pk[BN / 2];
#pragma unroll
          for (int c0 = 0; c0 < BN; c0 += 32) {
            uint32_t v[32];
            tc_ld_32x32b_x32(acc + c0, v);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
              pk[c0 / 2 + i] = *reinterpret_cast<uint32_t*>(&h);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(tempty_leader0);
#pragma unroll
          for (int c0 = 0; c0 < BN; c0 += 32) {
            uint8_t* buf = sY + (q * 2 + (ebuf & 1)) * 2048;
            if (lane == 0 && ebuf >= 2) bulk_wait_read1();
            __syncwarp();
            if (args.tma_store == 2) {
              // transposed: [32 columns of this tile][32 rows] staging tile
              uint16_t* t = reinterpret_cast<uint16_t*>(buf);
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                t[(2 * i) * 32 + lane] = static_cast<uint16_t>(pk[c0 / 2 + i] & 0xFFFFu);
                t[(2 * i + 1) * 32 + lane] = static_cast<uint16_t>(pk[c0 / 2 + i] >> 16);
              }
            } else {
              // 32 rows x 32 bf16, 64-byte swizzle (as below)
#pragma unroll
              for (int j = 0; j < 4; ++j)
                *reinterpret_cast<uint4*>(buf + lane * 64 + 16 * (j ^ ((lane >> 1) & 3))) =
                    make_uint4(pk[c0 / 2 + 4 * j], pk[c0 / 2 + 4 * j + 1], pk[c0 / 2 + 4 * j + 2],
                               pk[c0 / 2 + 4 * j + 3]);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
              if (args.tma_store == 2)
                tma_store_2d(&tmY, buf, static_cast<int32_t>(row0),
                             static_cast<int32_t>(static_cast<int64_t>(tn) * BN + c0));
              else
                tma_store_2d(&tmY, buf, static_cast<int32_t>(static_cast<int64_t>(tn) * BN + c0),
                             static_cast<int32_t>(row0));
              bulk_commit();
            }
            ++ebuf;
          }
          continue;
        }
      }
#pragma unroll 1
      for (int u = 0; u < MSUB; ++u) {
        const int64_t row0 = (static_cast<int64_t>(tm) * MSUB + u) * 256 + rank * 128 + q * 32;
        const int64_t ra = row0 + lane;
        const uint32_t acc = tmem_base + (b * MSUB + u) * Cfg::kAccStride + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t v[32];
          tc_ld_32x32b_x32(acc + c0, v);
          tc_wait_ld();
          if (wk.part >= 0) {
            // stream-K part: the raw fp32 accumulator goes to its workspace unit
            float4* dst = reinterpret_cast<float4*>(
                args.sk_ws +
                (static_cast<size_t>(wk.t - args.sk_full) * args.sk_parts + wk.part) * (256 * MSUB * BN) +
                static_cast<size_t>(u * 256 + rank * 128 + q * 32 + lane) * BN + c0);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                   __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
            continue;
          }
          if constexpr (FP8) {
            // rescale: acc * scale_a[row] * scale_b[column]
            const float sa = ra < args.rows_a ? __ldg(args.scale_a + ra) : 0.0f;
            const int64_t cb0 = static_cast<int64_t>(tn) * BN + c0;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float sb = cb0 + i < args.rows_b ? __ldg(args.scale_b + cb0 + i) : 0.0f;
              v[i] = __float_as_uint(__uint_as_float(v[i]) * sa * sb);
            }
          } else if (args.scale_a != nullptr) {
            // the per-token corrections of the activation operand
            const float sa = ra < args.rows_a ? __ldg(args.scale_a + ra) : 0.0f;
            const float mu = ra < args.rows_a ? __ldg(args.shift_a + ra) : 0.0f;
            const int64_t cb0 = static_cast<int64_t>(tn) * BN + c0;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float cs = cb0 + i < args.rows_b ? __ldg(args.sum_b + cb0 + i) : 0.0f;
              v[i] = __float_as_uint(__fmaf_rn(mu, cs, __uint_as_float(v[i]) * sa));
            }
          }
          if (args.tma_store == 2) {
            // transposed: the staging tile is [32 columns of this tile][32 rows],
            // so that each of its rows is 64 contiguous bytes of one row of Y
            uint8_t* buf = sY + (q * 2 + (ebuf & 1)) * 2048;
            if (lane == 0 && ebuf >= 2) bulk_wait_read1();
            __syncwarp();
            __nv_bfloat16* t = reinterpret_cast<__nv_bfloat16*>(buf);
#pragma unroll
            for (int i = 0; i < 32; ++i) t[i * 32 + lane] = __float2bfloat16_rn(__uint_as_float(v[i]));
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmY, buf, static_cast<int32_t>(row0),
                           static_cast<int32_t>(static_cast<int64_t>(tn) * BN + c0));
              bulk_commit();
            }
            ++ebuf;
          } else if (args.tma_store) {
            // 32 rows x 32 bf16 staging tile, 64-byte swizzle: row r's 16-byte
            // chunk j sits at r*64 + 16*(j ^ ((r >> 1) & 3)).  Two buffers per
            // warp; a buffer is rewritten only after its previous store read it.
            uint8_t* buf = sY + (q * 2 + (ebuf & 1)) * 2048;
            if (lane == 0 && ebuf >= 2) bulk_wait_read1();
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t p[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(v[8 * j + 2 * k]),
                                                         __uint_as_float(v[8 * j + 2 * k + 1]));
                p[k] = *reinterpret_cast<uint32_t*>(&h);
              }
              *reinterpret_cast<uint4*>(buf + lane * 64 + 16 * (j ^ ((lane >> 1) & 3))) =
                  make_uint4(p[0], p[1], p[2], p[3]);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmY, buf, static_cast<int32_t>(static_cast<int64_t>(tn) * BN + c0),
                           static_cast<int32_t>(row0));
              bulk_commit();
            }
            ++ebuf;
          } else if (c0 + 32 <= BN) {
            store_row_chunk<32>(st, ra, static_cast<int64_t>(tn) * BN + c0, v);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c0 + i < BN) store_out(st, ra, static_cast<int64_t>(tn) * BN + c0 + i, __uint_as_float(v[i]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(b == 0 ? tempty_leader0 : tempty_leader1);
    }
    if (args.tma_store && lane == 0) bulk_wait_all();   // stores done before the CTA exits
    __syncwarp();
  }

  tc_fence_before();
  __syncwarp();
  cluster_barrier();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem_base, Cfg::kTmemCols);
  }
}

// Stream-K fixup: every split tile of Y is the sum, in part order, of its
// parts' fp32 partial tiles (workspace units, [tile_rows][BN]), converted as
// the GEMM epilogue converts (fp32 or bf16 nearest-even; Y[a][b] or, with
// transpose, Y[b][a]).  A thread takes four consecutive columns of one row
// (one 16-byte load per part); consecutive threads take consecutive columns
// (Y[a][b]) or consecutive rows (Y[b][a]), so that the stores coalesce.
__global__ void __launch_bounds__(256)
k_sk_fixup(const float* __restrict__ ws, int sk_full, int sk_parts, int tail_tiles, int tiles_m, int tile_rows,
           int BN, int64_t rows_a, int64_t rows_b, void* __restrict__ Y, int64_t ldy, int out_fp32, int transpose) {
  griddep_launch_dependents();
  griddep_wait();                                      // the partial tiles of the preceding GEMM
  const int64_t unit = static_cast<int64_t>(tile_rows) * BN;
  const int64_t quads = unit / 4;
  const int64_t total = static_cast<int64_t>(tail_tiles) * quads;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int tl = static_cast<int>(idx / quads);
    const int e = static_cast<int>(idx - tl * quads);
    const int t = sk_full + tl;
    const int64_t a0 = static_cast<int64_t>(t % tiles_m) * tile_rows, b0 = static_cast<int64_t>(t / tiles_m) * BN;
    const int ra = transpose ? e % tile_rows : e / (BN / 4);
    const int cb = 4 * (transpose ? e / tile_rows : e % (BN / 4));
    // all of a group of up to eight parts' loads in flight before the adds
    // (still added in part order)
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float* u0 = ws + static_cast<int64_t>(tl) * sk_parts * unit + static_cast<int64_t>(ra) * BN + cb;
    for (int p0 = 0; p0 < sk_parts; p0 += 8) {
      float4 x[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (p0 + i < sk_parts) x[i] = __ldcg(reinterpret_cast<const float4*>(u0 + (p0 + i) * unit));
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (p0 + i < sk_parts) { acc.x += x[i].x; acc.y += x[i].y; acc.z += x[i].z; acc.w += x[i].w; }
    }
    const float v[4] = {acc.x, acc.y, acc.z, acc.w};
    const int64_t a = a0 + ra;
    if (a >= rows_a) continue;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t b = b0 + cb + i;
      if (b >= rows_b) continue;
      const int64_t off = transpose ? b * ldy + a : a * ldy + b;
      if (out_fp32) static_cast<float*>(Y)[off] = v[i];
      else static_cast<__nv_bfloat16*>(Y)[off] = __float2bfloat16_rn(v[i]);
    }
  }
}

}  // namespace nm
