// nm_gemm.cuh -- tcgen05 GEMM for 2:4-compressed (sparse) and dense k-blocks.
//
//   D[128 x BN] (TMEM, fp32) = sum over k-blocks of A_kb . B_kb^T
//
// A k-block is either
//   sparse: A = 128 rows x 64 stored bf16 (128 lifted K, 2:4 compressed),
//           B = BN rows x 128 bf16, metadata 2048 B; 4 x tcgen05.mma.sp (K=32)
//   dense : A = 128 rows x 64 bf16, B = BN rows x 64 bf16; 4 x tcgen05.mma (K=16)
// Sparse k-blocks come first (they cover B columns [0, K's)), then the dense
// ones (B columns K's + 64*kd ...): this one loop serves the plain sparse
// GEMM, the dense comparator and the hybrid input-split product.  In an
// output-split product (out_split_tiles >= 0) A's first out_split_tiles
// row tiles are sparse and run the sparse k-blocks only, the rest are dense
// (rows of the dense A matrix from 0) and run the dense k-blocks only, both
// over B columns [0, K); dense tiles are scheduled first (they are longer).
//
// Warp roles (192 threads): warp 0 = TMA producer, warp 1 = TMEM owner and
// MMA issuer, warps 2..5 = epilogue (warp w reads TMEM lanes 32*(w%4)..).
// Split-K: the `splits` CTAs of one output tile form a thread-block cluster
// and the tile is summed in rank order through distributed shared memory -- no
// global scratch.  Rank r owns rows [r*128/splits, (r+1)*128/splits).  For
// BN <= 32 every CTA pushes its partial rows into the owner's receive buffer
// (st.async, counted on the owner's mbarrier) and the owner sums them as soon
// as they have landed; wider tiles keep the partial in their own ring memory
// and are summed by distributed loads between two cluster barriers.
#pragma once
#include <type_traits>

#include "nm_device.cuh"

namespace nm {

constexpr int kBM = 128;
constexpr int kABytes = kBM * 128;          // one 128 B-wide swizzled tile
constexpr int kEBytes = 2048;               // metadata of one sparse k-block

struct GemmArgs {
  int64_t rows_a, rows_b;
  int kb_sparse, kb_dense;
  int64_t k_dense_x0;                       // B column where the dense part starts
  const uint8_t* meta;                      // metadata image of A's sparse part
  int64_t meta_kb;                          // metadata blocks per 128-row block
  void* Y;
  int64_t ldy;
  int out_fp32;
  int transpose_out;                        // 1: Y[b][a]; 0: Y[a][b]
  int splits;                               // CTAs per output tile (cluster size)
  int a_static;                             // A (and its metadata) may be read before the
                                            // preceding kernel finishes; B only after
  int out_split_tiles;                      // -1, or the number of sparse row tiles of an
                                            // output-split product
  // epilogue scaling: y = (acc * row_scale[a]) * col_scale[b] + row_shift[a] *
  // col_sum[b], each factor or term left out when its pointer is null (the
  // per-token corrections: row_scale, row_shift, col_sum; the 8-bit product:
  // row_scale, col_scale)
  const float* row_scale;
  const float* row_shift;
  const float* col_sum;
  const float* col_scale;
  int fp8_last_half;                        // 8-bit product: the last k-block holds only 128 lifted K
};

// In-GEMM lift (weight-side products, bf16, BN <= 32): B is the lift of a
// raw activation X [rows_b][lift_k] (tensor map tmB, boxes of 256 columns x
// BN rows, no swizzle), formed once per CTA in shared memory.  A separate
// parameter type, so that the other instantiations keep theirs unchanged.
struct LiftArgs : GemmArgs {
  int lift_m;                               // group size M of the (2n-2):2n pattern
  int64_t lift_k;                           // raw K
  int lift_boxes;                           // raw-X boxes a CTA may load (shared-memory budget)
  int lift_kb;                              // k-blocks a CTA may hold in its lifted panel
  int lift_raw_off, lift_panel_off;         // byte offsets of the raw boxes and the panel from the
                                            // (1024-aligned) shared-memory base
};

// FP8: a sparse k-block is 256 lifted K of E4M3 codes (A 128 stored bytes
// per row, B two 128-byte halves, two metadata blocks into 8 TMEM columns).
template <int BN, bool FP8 = false>
struct GemmCfg {
  static constexpr bool kPush = BN <= 32;                        // push split-K reduction
  static constexpr int kRecvBytes = kPush ? kBM * BN * 4 : 0;    // [splits][128/splits][BN] fp32
  static constexpr int kBBytes = 2 * BN * 128;
  static constexpr int kEStage = FP8 ? 2 * kEBytes : kEBytes;    // metadata bytes per stage
  static constexpr int kMetaCols = FP8 ? 8 : 4;                  // TMEM columns of metadata per stage
  static constexpr int kStageBytes = kABytes + kBBytes + kEStage;
  static constexpr int kStagesRaw = (200 * 1024) / kStageBytes;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static constexpr int kTmemNeed = BN + kMetaCols * kStages;
  static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128
                                 : kTmemNeed <= 256 ? 256 : 512;
  static constexpr int kSmemBytes = kStages * kStageBytes + kRecvBytes + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(kStages >= 2, "tile too large for the shared memory ring");
  static_assert(kBM * BN * 4 <= kStages * (kABytes + kBBytes), "split-K tile must fit the ring");
};

enum : unsigned { kWhereProducer = 1, kWhereMma = 2, kWhereEpilogue = 3 };

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Split cluster barrier: arrive (release) and wait (acquire), every thread once.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t mapa_shared_bar(const uint64_t* bar, uint32_t rank) {
  return mapa_shared(smem_u32(bar), rank);
}
// Asynchronous 16-byte store into a cluster peer's shared memory; its bytes
// complete on the peer's mbarrier.
__device__ __forceinline__ void st_async_f32x4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                               uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];"
               :: "r"(addr), "r"(a), "r"(b), "r"(c), "r"(d), "r"(bar) : "memory");
}
__device__ __forceinline__ float4 ld_dsmem_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ void store_out_raw(const GemmArgs& a, int64_t ra, int64_t cb, float v) {
  if (ra >= a.rows_a || cb >= a.rows_b) return;
  const int64_t off = a.transpose_out ? cb * a.ldy + ra : ra * a.ldy + cb;
  if (a.out_fp32) static_cast<float*>(a.Y)[off] = v;
  else static_cast<__nv_bfloat16*>(a.Y)[off] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float scale_out(const GemmArgs& a, int64_t ra, int64_t cb, float v) {
  if (a.row_scale != nullptr) v = v * a.row_scale[ra];
  if (a.col_scale != nullptr) v = v * a.col_scale[cb];
  if (a.row_shift != nullptr) v = __fmaf_rn(a.row_shift[ra], a.col_sum[cb], v);
  return v;
}

__device__ __forceinline__ void store_out(const GemmArgs& a, int64_t ra, int64_t cb, float v) {
  if (ra >= a.rows_a || cb >= a.rows_b) return;
  store_out_raw(a, ra, cb, scale_out(a, ra, cb, v));
}

// Stores CW (16 or 32) consecutive accumulator columns of row `ra`
// (columns cb0 .. cb0+CW-1).
template <int CW>
__device__ __forceinline__ void store_row_chunk(const GemmArgs& a, int64_t ra, int64_t cb0,
                                                const uint32_t (&v_in)[CW]) {
  if (ra >= a.rows_a) return;
  uint32_t v[CW];
#pragma unroll
  for (int i = 0; i < CW; ++i) v[i] = v_in[i];
  if (a.row_scale != nullptr || a.col_scale != nullptr || a.row_shift != nullptr) {
#pragma unroll
    for (int i = 0; i < CW; ++i)
      if (cb0 + i < a.rows_b) v[i] = __float_as_uint(scale_out(a, ra, cb0 + i, __uint_as_float(v[i])));
  }
  if (a.transpose_out && cb0 + CW <= a.rows_b) {
    // Y[b][a]: lane = a, so each store instruction of the warp writes 32
    // consecutive outputs of one row of Y
    if (a.out_fp32) {
      float* p = static_cast<float*>(a.Y) + cb0 * a.ldy + ra;
#pragma unroll
      for (int i = 0; i < CW; ++i) p[i * a.ldy] = __uint_as_float(v[i]);
    } else {
      __nv_bfloat16* p = static_cast<__nv_bfloat16*>(a.Y) + cb0 * a.ldy + ra;
#pragma unroll
      for (int i = 0; i < CW; ++i) p[i * a.ldy] = __float2bfloat16_rn(__uint_as_float(v[i]));
    }
    return;
  }
  if (!a.transpose_out && cb0 + CW <= a.rows_b && (a.ldy % 8) == 0) {
    if (a.out_fp32) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.Y) + ra * a.ldy + cb0);
#pragma unroll
      for (int i = 0; i < CW / 4; ++i)
        dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                             __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
    } else {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.Y) + ra * a.ldy + cb0);
#pragma unroll
      for (int i = 0; i < CW / 8; ++i) {
        uint32_t p[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(v[8 * i + 2 * j]),
                                                   __uint_as_float(v[8 * i + 2 * j + 1]));
          p[j] = *reinterpret_cast<uint32_t*>(&h);
        }
        dst[i] = make_uint4(p[0], p[1], p[2], p[3]);
      }
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < CW; ++i) store_out_raw(a, ra, cb0 + i, __uint_as_float(v[i]));
}

// In-GEMM lift, run by the four epilogue warps (128 threads) of one CTA
// before its epilogue.  The CTA's k-blocks [kb_begin, kb_end) cover lifted
// columns [128 kb_begin, 128 kb_end); lifted column j of a (2n-2):2n pattern
// (M = 2n, n-1 windows of width 4 at stride 2 per group) is raw column
// g M + 2w + (j % 4) with g = j / (4(n-1)), w = (j % (4(n-1))) / 4.  The raw
// columns [c_base, (g_hi + 1) M) come in by TMA (boxes of 256 columns x BN
// rows, zero-filled past the matrix); then every window (4 lifted columns, 8
// bytes per row) is copied from shared memory into the 128-byte-swizzled
// K-major image the MMA descriptors expect (k-block i, half h, row r, 16-byte
// chunk c at i*2*BN*128 + h*BN*128 + r*128 + 16*(c ^ (r % 8)); a window is
// either half of a chunk).  Lifted columns past K' are zero, as a TMA load of
// the lifted matrix would leave them.  The async proxy is fenced before the
// arrival on panel_bar.
template <int BN>
__device__ __forceinline__ void lift_panel(const LiftArgs& args, const CUtensorMap& tmX, int kb_begin, int kb_end,
                                           uint8_t* sXr, uint8_t* sP, uint64_t* xraw_bar, uint64_t* panel_bar,
                                           volatile int* abort_flag) {
  const int t = static_cast<int>(threadIdx.x) - 64;              // 0 .. 127
  // 32-bit index arithmetic throughout: K and K' are below 2^24 (host check)
  const int M = args.lift_m;
  const int nw = M / 2 - 1;                                       // windows per group
  const uint32_t L = 4u * static_cast<uint32_t>(nw);              // lifted columns per group
  const uint32_t k_lift = (static_cast<uint32_t>(args.lift_k) / static_cast<uint32_t>(M)) * L;
  const uint32_t j_lo = static_cast<uint32_t>(kb_begin) * 128u;
  const uint32_t j_hi = max(min(static_cast<uint32_t>(kb_end) * 128u, k_lift), j_lo);   // empty range: no windows
  const uint32_t c_base = ((j_lo / L) * static_cast<uint32_t>(M)) & ~7u;   // 16-byte aligned TMA x coordinate
  const uint32_t c_end = (j_hi > j_lo) ? ((j_hi - 1u) / L + 1u) * static_cast<uint32_t>(M) : c_base;
  const int nbox = static_cast<int>((c_end - c_base + 255u) / 256u);
  bool ok = nbox <= args.lift_boxes && (kb_end - kb_begin) <= args.lift_kb;
  if (!ok) {
    if (t == 0) record_status(kStatusUnsupported, kWhereEpilogue);
  } else {
    if (t == 0) {
      griddep_wait();                                             // X may come from the preceding kernel
      mbar_arrive_expect_tx(xraw_bar, static_cast<uint32_t>(nbox * BN * 512));
      for (int b = 0; b < nbox; ++b)
        tma_load_2d(&tmX, xraw_bar, sXr + b * (BN * 512), static_cast<int32_t>(c_base + 256u * b), 0);
    }
    ok = mbar_wait(xraw_bar, 0u, abort_flag, kWhereEpilogue);
    // copies still in flight land before the CTA may exit
    if (!ok && t == 0) mbar_wait(xraw_bar, 0u, nullptr, kWhereEpilogue, 100000000ull);
  }
  if (ok) {
    // Window-major: a thread takes windows t, t+128, ... of the CTA's range;
    // the index arithmetic is done once per window (g = q / nw as a
    // multiply-high by ceil(2^32 / nw), exact for q < 2^22 and nw <= 15), then
    // the window is copied down all BN rows: two 4-byte loads and one 8-byte
    // store per row at compile-time row offsets, all independent.  A warp's
    // 32 windows are one k-block: its stores fill two 128-byte panel rows.
    const uint32_t magic = nw > 1 ? 0xFFFFFFFFu / static_cast<uint32_t>(nw) + 1u : 0u;
    // the raw base address passes through a volatile asm placed after the
    // wait on xraw_bar, so the (non-volatile, freely scheduled) loads below
    // cannot be hoisted above it
    uint32_t raw_s;
    asm volatile("mov.b32 %0, %1;" : "=r"(raw_s) : "r"(smem_u32(sXr)) : "memory");
    const uint32_t pan_s = smem_u32(sP);
    const uint32_t q_lo = j_lo / 4u, nwin = (j_hi - j_lo) / 4u;
    for (uint32_t qi = static_cast<uint32_t>(t); qi < nwin; qi += 128u) {
      const uint32_t q = q_lo + qi;
      const uint32_t g = nw > 1 ? __umulhi(q, magic) : q;
      const uint32_t w = q - g * static_cast<uint32_t>(nw);
      const uint32_t col = g * static_cast<uint32_t>(M) + 2u * w - c_base;   // 4 columns, never across a box edge
      const uint32_t src = raw_s + (col / 256u) * (BN * 512) + (col % 256u) * 2u;
      const uint32_t p = 4u * qi;
      const uint32_t c = (p % 64u) / 8u;
      const uint32_t dst = pan_s + (p / 128u) * (2 * BN * 128) + ((p % 128u) / 64u) * (BN * 128) + 8u * ((p % 8u) / 4u);
      uint32_t a[BN], b[BN];
#pragma unroll
      for (int r = 0; r < BN; ++r) {
        asm("ld.shared.b32 %0, [%1];" : "=r"(a[r]) : "r"(src + r * 512));
        asm("ld.shared.b32 %0, [%1];" : "=r"(b[r]) : "r"(src + r * 512 + 4));
      }
#pragma unroll
      for (int r = 0; r < BN; ++r)
        asm volatile("st.shared.v2.b32 [%0], {%1, %2};"
                     :: "r"(dst + r * 128 + 16u * (c ^ static_cast<uint32_t>(r % 8))), "r"(a[r]), "r"(b[r]) : "memory");
    }
    // lifted columns [j_hi, 128 kb_end) past K' are zero, as a TMA load of
    // the lifted matrix would leave them
    const uint32_t p_end = static_cast<uint32_t>(kb_end - kb_begin) * 128u;
    for (uint32_t e = static_cast<uint32_t>(t); e < (p_end - (j_hi - j_lo)) / 4u * BN; e += 128u) {
      const uint32_t r = e % BN, p = (j_hi - j_lo) + 4u * (e / BN);
      const uint32_t c = (p % 64u) / 8u;
      const uint32_t dst = pan_s + (p / 128u) * (2 * BN * 128) + ((p % 128u) / 64u) * (BN * 128) + r * 128 +
                           16u * (c ^ (r % 8u)) + 8u * ((p % 8u) / 4u);
      asm volatile("st.shared.v2.b32 [%0], {%1, %2};" :: "r"(dst), "r"(0u), "r"(0u) : "memory");
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");    // generic writes -> tensor-core reads
  // Arrive even on failure: the MMA issuer then sees the abort flag or a
  // zero panel, never waits forever.
  if (!ok) *abort_flag = 1;
  mbar_arrive(panel_bar);
}

// LIFT_RING > 0 is the in-GEMM lift instantiation (bf16, BN <= 32): B comes
// from the lifted panel and the ring holds LIFT_RING stages of A and
// metadata; otherwise the ring holds Cfg::kStages full stages.
template <int BN, bool FP8 = false, int LIFT_RING = 0>
__global__ void __launch_bounds__(192, 1)
k_nm_gemm(const __grid_constant__ CUtensorMap tmA_s, const __grid_constant__ CUtensorMap tmA_d,
          const __grid_constant__ CUtensorMap tmB,
          const std::conditional_t<(LIFT_RING > 0), LiftArgs, GemmArgs> args) {
  using Cfg = GemmCfg<BN, FP8>;
  constexpr bool lift = LIFT_RING > 0;
  static_assert(!lift || (!FP8 && BN <= 32), "in-GEMM lift: bf16, at most 32 activation rows");
  constexpr int S = lift ? LIFT_RING : Cfg::kStages;
  constexpr int b_stage = lift ? 0 : Cfg::kBBytes;   // in-GEMM lift: B lives in the panel, not the ring
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + S * kABytes;
  uint8_t* sE = sB + S * b_stage;
  float* sRecv = reinterpret_cast<float*>(sE + S * Cfg::kEStage);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(sE + S * Cfg::kEStage + Cfg::kRecvBytes);
  uint64_t* empty_bar = full_bar + S;
  uint64_t* accum_bar = empty_bar + S;
  uint64_t* red_bar = accum_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint64_t* xraw_bar = red_bar + 2;                  // in-GEMM lift: raw X landed
  uint64_t* panel_bar = red_bar + 3;                 // in-GEMM lift: lifted panel written
  uint8_t* sP = nullptr;                             // in-GEMM lift: the lifted panel
  if constexpr (lift) sP = smem + args.lift_panel_off;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t tiles_m = gridDim.x;
  const int tsp = args.out_split_tiles;
  // output-split: dense tiles (the longer ones) take the first blocks
  const int64_t m_tile = tsp < 0 ? blockIdx.x
                                 : (blockIdx.x < tiles_m - tsp ? tsp + blockIdx.x : blockIdx.x - (tiles_m - tsp));
  const int64_t n_tile = blockIdx.y;
  const bool dense_tile = tsp >= 0 && m_tile >= tsp;
  const int split = static_cast<int>(blockIdx.z);
  const int kb_lo = dense_tile ? args.kb_sparse : 0;
  const int kb_hi = tsp < 0 ? args.kb_sparse + args.kb_dense : (dense_tile ? args.kb_sparse + args.kb_dense : args.kb_sparse);
  const int kb_total = kb_hi - kb_lo;
  const int kb_begin = kb_lo + static_cast<int>(static_cast<int64_t>(kb_total) * split / args.splits);
  const int kb_end = kb_lo + static_cast<int>(static_cast<int64_t>(kb_total) * (split + 1) / args.splits);

  const bool push = Cfg::kPush && args.splits > 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    mbar_init(accum_bar, 1);
    mbar_init(red_bar, 1);
    if constexpr (lift) {
      mbar_init(xraw_bar, 1);
      mbar_init(panel_bar, 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
    // the owner's share of every rank's partial tile: 128 rows x BN fp32 in all
    if (push) mbar_arrive_expect_tx(red_bar, static_cast<uint32_t>(Cfg::kRecvBytes));
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA_s); prefetch_tmap(&tmA_d); prefetch_tmap(&tmB);
  }
  if (warp == 1) { tmem_alloc(tmem_slot, Cfg::kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_slot;
  const uint32_t tmem_meta = tmem_acc + BN;
  griddep_launch_dependents();                       // the next kernel may begin its set-up
  // Push split-K: the cluster's receive barriers exist before any partial is
  // pushed (epilogue warps wait on this; the other warps before they exit).
  if (push) cluster_arrive();

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (elect_one()) {
      const int32_t y_a = static_cast<int32_t>((dense_tile ? m_tile - tsp : m_tile) * kBM);
      const int32_t y_b = static_cast<int32_t>(n_tile * BN);
      // 8-bit: metadata blocks (and B halves) in this k-block, 1 for a last
      // block of 128 lifted K
      auto halves = [&](int kb) { return (FP8 && args.fp8_last_half && kb == args.kb_sparse - 1) ? 1 : 2; };
      auto load_a = [&](int kb, int s) {
        uint8_t* a_dst = sA + s * kABytes;
        if constexpr (FP8) {
          const int eb = halves(kb);
          mbar_arrive_expect_tx(&full_bar[s], kABytes + BN * 128 * eb + kEBytes * eb);
          tma_load_2d(&tmA_s, &full_bar[s], a_dst, kb * 128, y_a);
          for (int e = 0; e < eb; ++e)
            bulk_load(sE + s * Cfg::kEStage + e * kEBytes, args.meta + (m_tile * args.meta_kb + 2 * kb + e) * kEBytes,
                      kEBytes, &full_bar[s]);
        } else if (kb < args.kb_sparse) {
          mbar_arrive_expect_tx(&full_bar[s], kABytes + b_stage + kEBytes);
          tma_load_2d(&tmA_s, &full_bar[s], a_dst, kb * 64, y_a);
          bulk_load(sE + s * Cfg::kEStage, args.meta + (m_tile * args.meta_kb + kb) * kEBytes, kEBytes,
                    &full_bar[s]);
        } else {
          mbar_arrive_expect_tx(&full_bar[s], kABytes + BN * 128);
          tma_load_2d(&tmA_d, &full_bar[s], a_dst, (kb - args.kb_sparse) * 64, y_a);
        }
      };
      auto load_b = [&](int kb, int s) {
        if constexpr (lift) return;                      // B is formed in the panel
        uint8_t* b_dst = sB + s * Cfg::kBBytes;
        if constexpr (FP8) {
          tma_load_2d(&tmB, &full_bar[s], b_dst, kb * 256, y_b);
          if (halves(kb) == 2) tma_load_2d(&tmB, &full_bar[s], b_dst + BN * 128, kb * 256 + 128, y_b);
        } else if (kb < args.kb_sparse) {
          tma_load_2d(&tmB, &full_bar[s], b_dst, kb * 128, y_b);
          tma_load_2d(&tmB, &full_bar[s], b_dst + BN * 128, kb * 128 + 64, y_b);
        } else {
          tma_load_2d(&tmB, &full_bar[s], b_dst,
                      static_cast<int32_t>(args.k_dense_x0) + (kb - args.kb_sparse) * 64, y_b);
        }
      };
      // The static operand of the first ring's worth of stages is requested
      // while the preceding kernel may still run; everything else waits for it.
      int it = 0;
      int pre = 0;
      if (args.a_static) {
        pre = kb_end - kb_begin < S ? kb_end - kb_begin : S;
        for (int j = 0; j < pre; ++j) load_a(kb_begin + j, j);
      }
      griddep_wait();
      for (int j = 0; j < pre; ++j) load_b(kb_begin + j, j);
      it = pre;
      for (int kb = kb_begin + pre; kb < kb_end; ++kb, ++it) {
        const int s = it % S;
        const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
        if (!mbar_wait(&empty_bar[s], ph ^ 1u, abort_flag, kWhereProducer)) break;
        load_a(kb, s);
        load_b(kb, s);
      }
      // Only the last S loads can still be in flight (a stage is reissued only
      // after the MMA released it); wait for them before the CTA may exit.
      for (int j = (it > S ? it - S : 0); j < it; ++j)
        mbar_wait(&full_bar[j % S], static_cast<uint32_t>(j / S) & 1u, nullptr, kWhereProducer,
                  100000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    if (elect_one()) {
      const uint32_t idesc_sp = idesc_bf16(kBM, BN, true);
      const uint32_t idesc_dn = idesc_bf16(kBM, BN, false);
      int it = 0;
      bool ok = true;
      if constexpr (lift) ok = mbar_wait(panel_bar, 0u, abort_flag, kWhereMma);
      const int kb_stop = ok ? kb_end : kb_begin;
      for (int kb = kb_begin; kb < kb_stop; ++kb, ++it) {
        const int s = it % S;
        const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
        if (!mbar_wait(&full_bar[s], ph, abort_flag, kWhereMma)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + s * kABytes);
        const uint32_t b0 = lift ? smem_u32(sP + (kb - kb_begin) * Cfg::kBBytes) : smem_u32(sB + s * Cfg::kBBytes);
        if constexpr (FP8) {
          // two metadata blocks -> columns e_col, e_col + 4; MMA kk (64
          // lifted K) reads the column pair at e_col + 2 kk
          const uint32_t e_col = tmem_meta + static_cast<uint32_t>(Cfg::kMetaCols) * s;
          const int nkk = (args.fp8_last_half && kb == args.kb_sparse - 1) ? 2 : 4;
          for (int e = 0; e < nkk / 2; ++e)
            tc_cp_128x128b(e_col + 4u * e, desc_plain_128x16(smem_u32(sE + s * Cfg::kEStage + e * kEBytes)));
          const uint32_t idesc8 = idesc_e4m3(kBM, BN, true);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            if (kk < nkk) {
              const uint64_t ad = desc_sw128_kmajor(a0 + 32u * kk);
              const uint64_t bd = desc_sw128_kmajor(b0 + (kk / 2) * (BN * 128) + (kk % 2) * 64);
              tc_mma_sp_e4m3(tmem_acc, ad, bd, e_col + 2u * kk, idesc8, (it > 0 || kk > 0) ? 1u : 0u);
            }
          }
        } else if (kb < args.kb_sparse) {
          const uint32_t e_col = tmem_meta + 4u * s;
          tc_cp_128x128b(e_col, desc_plain_128x16(smem_u32(sE + s * Cfg::kEStage)));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = desc_sw128_kmajor(a0 + 32u * kk);
            const uint64_t bd = desc_sw128_kmajor(b0 + (kk / 2) * (BN * 128) + (kk % 2) * 64);
            // The metadata operand is addressed in pairs of columns: the even
            // column goes in the address, the odd/even choice in the
            // instruction descriptor's sparse-id2 field (bits 0-1).
            tc_mma_sp_f16(tmem_acc, ad, bd, e_col + (kk & ~1), idesc_sp | static_cast<uint32_t>(kk & 1),
                          (it > 0 || kk > 0) ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = desc_sw128_kmajor(a0 + 32u * kk);
            const uint64_t bd = desc_sw128_kmajor(b0 + 32u * kk);
            tc_mma_f16(tmem_acc, ad, bd, idesc_dn, (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc_commit(&empty_bar[s]);
      }
      if (ok) tc_commit(accum_bar);
    }
  } else {
    // -------------------------------------------------------- epilogue
    const int q = warp % 4;
    if constexpr (lift) {
      lift_panel<BN>(args, tmB, kb_begin, kb_end, smem + args.lift_raw_off, sP, xraw_bar, panel_bar, abort_flag);
    }
    const bool ok = mbar_wait_warp(accum_bar, 0u, abort_flag, kWhereEpilogue);
    griddep_wait();                                  // Y may still be in use upstream
    tc_fence_after();
    if (push) {
      __syncwarp();
      cluster_wait();                                // every receive barrier of the cluster is set up
    }
    if (ok) {
      const int64_t row_local = q * 32 + lane;
      const int64_t ra = m_tile * kBM + row_local;
      float* red = reinterpret_cast<float*>(smem);        // split-K partial tile
      if (args.splits > 1 && !push) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      constexpr int CW = BN < 32 ? BN : 32;              // columns per TMEM load
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += CW) {
        uint32_t v[CW];
        tc_ld_32x32b<CW>(tmem_acc + (static_cast<uint32_t>(q * 32) << 16) + c0, v);
        tc_wait_ld();
        if (push) {
          // this row goes to its owner's slot for this rank
          const int rows_per = kBM / args.splits;
          const uint32_t owner = static_cast<uint32_t>(row_local / rows_per);
          const uint32_t slot = cluster_ctarank() * rows_per + static_cast<uint32_t>(row_local % rows_per);
          const uint32_t dst = mapa_shared(smem_u32(sRecv + slot * BN + c0), owner);
          const uint32_t bar = mapa_shared_bar(red_bar, owner);
#pragma unroll
          for (int i = 0; i < CW / 4; ++i)
            st_async_f32x4(dst + 16u * i, v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3], bar);
        } else if (args.splits == 1) {
          store_row_chunk<CW>(args, ra, n_tile * BN + c0, v);
        } else {
          float4* dst = reinterpret_cast<float4*>(red + row_local * BN + c0);
#pragma unroll
          for (int i = 0; i < CW / 4; ++i)
            dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                 __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
        }
      }
    }
    if (push) {
      // Sum the pushed partials of this CTA's rows in rank order, once they
      // have all landed.
      if (mbar_wait(red_bar, 0u, nullptr, kWhereEpilogue)) {
        const int rows_per = kBM / args.splits;
        const uint32_t rank = cluster_ctarank();
        const int quads = rows_per * (BN / 4);
        const int t = threadIdx.x - 64;
        for (int e = t; e < quads; e += 128) {
          const int rl = args.transpose_out ? e % rows_per : e / (BN / 4);
          const int c = 4 * (args.transpose_out ? e / rows_per : e % (BN / 4));
          float4 acc = *reinterpret_cast<const float4*>(sRecv + rl * BN + c);
#pragma unroll
          for (int p = 1; p < 8; ++p)
            if (p < args.splits) {
              const float4 x = *reinterpret_cast<const float4*>(sRecv + (p * rows_per + rl) * BN + c);
              acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
            }
          const int64_t ra = m_tile * kBM + static_cast<int64_t>(rank) * rows_per + rl, cb = n_tile * BN + c;
          store_out(args, ra, cb, acc.x);
          store_out(args, ra, cb + 1, acc.y);
          store_out(args, ra, cb + 2, acc.z);
          store_out(args, ra, cb + 3, acc.w);
        }
      }
    }
  }
  if (push && warp < 2) {
    __syncwarp();
    cluster_wait();                                    // matches the set-up arrival
  }

  if (args.splits > 1 && !push) {
    // Sum the cluster's partial tiles in rank order; rank r owns rows
    // [r*128/splits, (r+1)*128/splits) of the tile.
    __syncwarp();
    cluster_sync_all();
    if (!*abort_flag) {
      // Four consecutive columns per thread; all partial loads are issued
      // before the (rank-ordered, hence deterministic) sum.
      const uint32_t rank = cluster_ctarank();
      const int rows_per = kBM / args.splits;
      const int quads = rows_per * (BN / 4);
      const uint32_t red_base = smem_u32(smem);
      griddep_wait();
      for (int e = threadIdx.x; e < quads; e += blockDim.x) {
        const int rl = args.transpose_out ? e % rows_per : e / (BN / 4);
        const int c = 4 * (args.transpose_out ? e / rows_per : e % (BN / 4));
        const int row_local = static_cast<int>(rank) * rows_per + rl;
        const uint32_t off = red_base + static_cast<uint32_t>((row_local * BN + c) * 4);
        float4 part[8];
#pragma unroll
        for (int p = 0; p < 8; ++p)
          if (p < args.splits) part[p] = ld_dsmem_f32x4(mapa_shared(off, static_cast<uint32_t>(p)));
        float4 acc = part[0];
#pragma unroll
        for (int p = 1; p < 8; ++p)
          if (p < args.splits) {
            acc.x += part[p].x; acc.y += part[p].y; acc.z += part[p].z; acc.w += part[p].w;
          }
        const int64_t ra = m_tile * kBM + row_local, cb = n_tile * BN + c;
        store_out(args, ra, cb, acc.x);
        store_out(args, ra, cb + 1, acc.y);
        store_out(args, ra, cb + 2, acc.z);
        store_out(args, ra, cb + 3, acc.w);
      }
    }
    cluster_sync_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_acc, Cfg::kTmemCols);
  }
}

}  // namespace nm
