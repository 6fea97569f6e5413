// nm_prune.cuh -- prune + window-compress, lift, and the offline hybrid
// selection kernels.  HBM-bound SIMT code: 128-bit coalesced loads, integer
// magnitude keys, results written in the layouts the GEMM consumes.
#pragma once
#include "nm_device.cuh"

namespace nm {

// Splits a 32-bit word into its elements (two 16-bit or one 32-bit).
__device__ __forceinline__ void split_word(uint32_t w, uint16_t* out) {
  out[0] = static_cast<uint16_t>(w & 0xFFFFu);
  out[1] = static_cast<uint16_t>(w >> 16);
}
__device__ __forceinline__ void split_word(uint32_t w, uint32_t* out) { out[0] = w; }

__device__ __forceinline__ uint16_t to_bf16_bits(uint16_t b) { return b; }
__device__ __forceinline__ uint16_t to_bf16_bits(uint32_t f) {
  __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(f));
  return *reinterpret_cast<uint16_t*>(&h);
}

// Unique ordering key: magnitude bits first, then the lower index wins.
__device__ __forceinline__ uint32_t order_key(uint16_t b, int i) {
  return (static_cast<uint32_t>(b & 0x7FFFu) << 5) | static_cast<uint32_t>(31 - i);
}
__device__ __forceinline__ uint64_t order_key(uint32_t b, int i) {
  return (static_cast<uint64_t>(b & 0x7FFFFFFFu) << 5) | static_cast<uint64_t>(31 - i);
}
template <typename K> __device__ __forceinline__ K kmax(K a, K b) { return a > b ? a : b; }
template <typename K> __device__ __forceinline__ K kmin(K a, K b) { return a < b ? a : b; }

// Bitonic network, descending, on M (power of two) distinct keys in registers.
template <int M> struct Log2 { static constexpr int value = 1 + Log2<M / 2>::value; };
template <> struct Log2<1> { static constexpr int value = 0; };

template <int M, typename K>
__device__ __forceinline__ void bitonic_desc(K (&a)[M]) {
  constexpr int L = Log2<M>::value;
#pragma unroll
  for (int lk = 1; lk <= L; ++lk) {
    const int k = 1 << lk;
#pragma unroll
    for (int lj = lk - 1; lj >= 0; --lj) {
      const int j = 1 << lj;
#pragma unroll
      for (int i = 0; i < M; ++i) {
        const int l = i ^ j;
        if (l > i) {
          const K x = a[i], y = a[l];
          if ((i & k) == 0) { a[i] = kmax(x, y); a[l] = kmin(x, y); }
          else { a[i] = kmin(x, y); a[l] = kmax(x, y); }
        }
      }
    }
  }
}

// Batcher's odd-even merge network on N (power of two) inputs, as a
// compile-time list of comparators: N(log N)(log N - 1)/4 + N - 1 of them
// (19 for 8, 63 for 16, 191 for 32), fewer than the bitonic network's.
template <int N>
struct OddEvenNet {
  int n = 0;
  unsigned char lo[256] = {}, hi[256] = {};
  constexpr OddEvenNet() {
    for (int p = 1; p < N; p <<= 1)
      for (int k = p; k >= 1; k >>= 1)
        for (int j = k % p; j + k < N; j += 2 * k)
          for (int i = 0; i < k; ++i)
            if (i + j + k < N && (i + j) / (2 * p) == (i + j + k) / (2 * p)) {
              lo[n] = static_cast<unsigned char>(i + j);
              hi[n] = static_cast<unsigned char>(i + j + k);
              ++n;
            }
  }
};

// Sorts N keys in registers in descending order.
template <int N, typename K>
__device__ __forceinline__ void oddeven_desc(K (&a)[N]) {
  constexpr OddEvenNet<N> net{};
#pragma unroll
  for (int c = 0; c < net.n; ++c) {
    const K x = a[net.lo[c]], y = a[net.hi[c]];
    a[net.lo[c]] = kmax(x, y);
    a[net.hi[c]] = kmin(x, y);
  }
}

// Raw bytes of one group, as loaded (16-byte words, or one 8-byte word).
template <int M, typename T>
struct GroupRaw {
  static constexpr int BYTES = M * static_cast<int>(sizeof(T));
  static constexpr int NV = BYTES >= 16 ? BYTES / 16 : 1;
  uint4 v[NV];
};

template <int M, typename T>
__device__ __forceinline__ void load_raw(const T* __restrict__ p, GroupRaw<M, T>& g) {
  if constexpr (GroupRaw<M, T>::BYTES >= 16) {
#pragma unroll
    for (int i = 0; i < GroupRaw<M, T>::NV; ++i) g.v[i] = __ldg(reinterpret_cast<const uint4*>(p) + i);
  } else {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    g.v[0] = make_uint4(u.x, u.y, 0u, 0u);
  }
}

template <int M, typename T>
__device__ __forceinline__ void unpack_raw(const GroupRaw<M, T>& g, T (&x)[M]) {
  constexpr int PW = 4 / static_cast<int>(sizeof(T));
  constexpr int WORDS = M / PW;                                   // 32-bit words in the group
#pragma unroll
  for (int wi = 0; wi < WORDS; ++wi) {
    const uint4& q = g.v[wi / 4];
    const uint32_t w = (wi % 4 == 0) ? q.x : (wi % 4 == 1) ? q.y : (wi % 4 == 2) ? q.z : q.w;
    split_word(w, &x[wi * PW]);
  }
}

// The N-th largest of M distinct keys.  For N = M/2 the two halves are sorted
// and merged: the N largest of the union are max(a_i, b_{N-1-i}).
template <int M, typename Key>
__device__ __forceinline__ Key nth_largest(const Key (&key)[M], int N) {
  if constexpr (M >= 4) {
    if (2 * N == M) {
      constexpr int H = M / 2;
      Key a[H], b[H];
#pragma unroll
      for (int i = 0; i < H; ++i) { a[i] = key[i]; b[i] = key[H + i]; }
      bitonic_desc<H, Key>(a);
      bitonic_desc<H, Key>(b);
      Key thr = kmax(a[0], b[H - 1]);
#pragma unroll
      for (int i = 1; i < H; ++i) thr = kmin(thr, kmax(a[i], b[H - 1 - i]));
      return thr;
    }
  }
  Key srt[M];
#pragma unroll
  for (int i = 0; i < M; ++i) srt[i] = key[i];
  bitonic_desc<M, Key>(srt);
  Key thr = srt[0];                          // srt[N-1]: the minimum of the first N, others masked to ~0
#pragma unroll
  for (int k = 1; k < M; ++k) thr = kmin(thr, srt[k] | static_cast<Key>(static_cast<int64_t>(N - 1 - k) >> 63));
  return thr;
}

// Prune + window-compress one group held in registers: returns the keep bits,
// writes the NW value words and index pairs.
template <int M, typename T>
__device__ __forceinline__ uint32_t compress_group(const GroupRaw<M, T>& raw, int N, uint32_t* val_out,
                                                   uint8_t* nib_out) {
  constexpr int NW = M / 2 - 1;
  T x[M];
  unpack_raw<M, T>(raw, x);
  uint32_t P[M / 2];                          // bf16 pairs (2p, 2p+1)
#pragma unroll
  for (int p = 0; p < M / 2; ++p)
    P[p] = static_cast<uint32_t>(to_bf16_bits(x[2 * p])) | (static_cast<uint32_t>(to_bf16_bits(x[2 * p + 1])) << 16);
  using Key = decltype(order_key(x[0], 0));
  Key key[M];
#pragma unroll
  for (int i = 0; i < M; ++i) key[i] = order_key(x[i], i);
  uint32_t keep = 0u;
  if (N > 0) {
    const Key thr = nth_largest<M, Key>(key, N);
#pragma unroll
    for (int i = 0; i < M; ++i) keep |= (key[i] >= thr ? 1u : 0u) << i;
  }
  uint32_t placed = 0u;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const uint32_t c = (keep >> (2 * w)) & ~(placed >> (2 * w)) & 0xFu;
    const uint32_t f = c & (0u - c);
    const uint32_t rest = c ^ f;
    const uint32_t sb = rest & (0u - rest);
    placed |= (f | sb) << (2 * w);
    int i0 = 0, i1 = 1;
    uint32_t zmask = 0u;
    if (sb) { i0 = __ffs(f) - 1; i1 = __ffs(sb) - 1; zmask = 0xFFFFFFFFu; }
    else if (f) {
      const int a = __ffs(f) - 1;
      if (a == 0) { zmask = 0x0000FFFFu; } else { i1 = a; zmask = 0xFFFF0000u; }
    }
    const uint32_t sel = static_cast<uint32_t>((0x10 + 0x22 * i0) | ((0x10 + 0x22 * i1) << 8));
    val_out[w] = __byte_perm(P[w], P[w + 1], sel) & zmask;
    nib_out[w] = static_cast<uint8_t>(i0 | (i1 << 2));
  }
  return keep;
}

// Window tables, indexed by the 4-bit set c of still-unplaced kept positions
// of a window (local positions 0..3).  The window takes the lowest two
// positions of c; one entry at a is paired with the lowest other index (its
// slot holds +0.0), none gives (0, 1) with both slots +0.0.
//   wt[c]      = {byte-permute selector picking the two values out of the
//                 window's four (bits 0-15), AND mask zeroing padded slots}
//   wt[16 + c] = {allowed mask of the next window, scaled by 8 (bits 3-6:
//                 its positions 0,1 unless this window placed them as its
//                 positions 2,3; positions 2,3 always), index pair i0 | i1 << 2}
// A table row is 8 bytes, so that c * 8 is the row's byte offset.
__device__ __forceinline__ void window_rows(uint32_t c, uint2* row_val, uint2* row_next) {
  const uint32_t f = c & (0u - c);
  const uint32_t rest = c ^ f;
  const uint32_t sb = rest & (0u - rest);
  const uint32_t taken = f | sb;
  int i0 = 0, i1 = 1;
  bool z0 = true, z1 = true;                      // slot holds padding
  if (sb) { i0 = __ffs(f) - 1; i1 = __ffs(sb) - 1; z0 = z1 = false; }
  else if (f) {
    const int a = __ffs(f) - 1;
    if (a == 0) { z0 = false; } else { i1 = a; z1 = false; }
  }
  const uint32_t sel = static_cast<uint32_t>((0x10 + 0x22 * i0) | ((0x10 + 0x22 * i1) << 8));
  const uint32_t zmask = (z0 ? 0u : 0x0000FFFFu) | (z1 ? 0u : 0xFFFF0000u);
  const uint32_t allowed = ((~(taken >> 2)) & 0x3u) | 0xCu;
  *row_val = make_uint2(sel, zmask);
  *row_next = make_uint2(allowed << 3, static_cast<uint32_t>(i0 | (i1 << 2)));
}

// Two 16-bit lanes per 32-bit word: one instruction does two comparators.
__device__ __forceinline__ uint32_t vmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t vmin2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t swap16(uint32_t a) { return __byte_perm(a, 0u, 0x1032); }

// Sorts the low lanes and the high lanes of H words, each descending, with
// one odd-even merge network.
template <int H>
__device__ __forceinline__ void oddeven_desc_x2(uint32_t (&a)[H]) {
  constexpr OddEvenNet<H> net{};
#pragma unroll
  for (int c = 0; c < net.n; ++c) {
    const uint32_t x = a[net.lo[c]], y = a[net.hi[c]];
    a[net.lo[c]] = vmax2(x, y);
    a[net.hi[c]] = vmin2(x, y);
  }
}

// Bit i (element i of the group) set iff lane value >= t, from words
// Q[p] = (|x[2p]|, |x[2p+1]|) of 15-bit magnitudes and C = (0x8000 - t) in
// both lanes: a lane of Q[p] + C never carries out, and its bit 15 is set iff
// the magnitude is at least t.
template <int H>
__device__ __forceinline__ uint32_t lane_ge_bits(const uint32_t (&Q)[H], uint32_t C) {
  uint32_t acc0 = 0u, acc1 = 0u;
#pragma unroll
  for (int p = 0; p < H; ++p) {
    const uint32_t e = Q[p] + C;
    const int q = p % 8;
    const uint32_t b = (e >> (15 - 2 * q)) & (0x00010001u << (2 * q));
    if (p < 8) acc0 |= b; else acc1 |= b;
  }
  uint32_t m = (acc0 & 0x5555u) | (acc0 >> 15);
  if constexpr (H > 8) m |= ((acc1 & 0x5555u) | (acc1 >> 15)) << 16;
  return m;
}

// Keep bits for N = M/2: the M/2 largest magnitudes, ties to the lower index.
// The even entries (low lanes) and the odd entries (high lanes) are sorted
// together; the M/2 largest of their union are max(a_i, b_{M/2-1-i}), whose
// minimum is the threshold t.  Entries above t are kept; entries equal to t
// fill the remaining places in index order.
template <int M>
__device__ __forceinline__ uint32_t half_keep_bf16(const uint32_t (&P)[M / 2]) {
  constexpr int H = M / 2;
  uint32_t Q[H], S[H];
#pragma unroll
  for (int p = 0; p < H; ++p) { Q[p] = P[p] & 0x7FFF7FFFu; S[p] = Q[p]; }
  oddeven_desc_x2<H>(S);
  uint32_t z = vmax2(S[0], swap16(S[H - 1]));
#pragma unroll
  for (int i = 1; i < H / 2; ++i) z = vmin2(z, vmax2(S[i], swap16(S[H - 1 - i])));
  const uint32_t t2 = vmin2(z, swap16(z));                // t in both lanes
  uint32_t keep = lane_ge_bits<H>(Q, 0x80008000u - t2);
  if (__popc(keep) != H) {                                // ties at t
    const uint32_t gt = lane_ge_bits<H>(Q, 0x80008000u - t2 - 0x00010001u);
    uint32_t eq = keep & ~gt;
    const int need = H - __popc(gt);
    while (__popc(eq) > need) eq &= ~(0x80000000u >> __clz(eq));
    keep = gt | eq;
  }
  return keep;
}

// bf16 groups held as 32-bit pair words P[p] = (x[2p], x[2p+1]): unique keys
// are formed on the fly, kept entries are those whose key is at least the N-th
// largest (sign of thr - 1 - key), windows come from the table.
template <int M>
__device__ __forceinline__ uint32_t ukey_bf16(const uint32_t (&P)[M / 2], int i) {
  const uint32_t w = P[i >> 1];
  const uint32_t k = (i & 1) ? ((w >> 16) & 0x7FFFu) : (w & 0x7FFFu);
  return (k << 5) | static_cast<uint32_t>(31 - i);
}

template <int M>
__device__ __forceinline__ uint32_t compress_group_bf16(const uint32_t (&P)[M / 2], int N, const uint2* wt,
                                                        uint32_t* val_out, uint8_t* nib_out) {
  constexpr int NW = M / 2 - 1;
  uint32_t keep = 0u;
  if (2 * N == M) {
    keep = half_keep_bf16<M>(P);
  } else if (N > 0) {
    uint32_t srt[M];
#pragma unroll
    for (int i = 0; i < M; ++i) srt[i] = ukey_bf16<M>(P, i);
    oddeven_desc<M, uint32_t>(srt);
    uint32_t thr = srt[0];                      // srt[N-1]: the minimum of the first N, others masked to ~0
#pragma unroll
    for (int k = 1; k < M; ++k) thr = kmin(thr, srt[k] | static_cast<uint32_t>((N - 1 - k) >> 31));
    const uint32_t t1 = thr - 1u;
#pragma unroll
    for (int i = 0; i < M; ++i) keep |= ((t1 - ukey_bf16<M>(P, i)) >> 31) << i;
  }
  // Windows left to right: the row offset of window w is its four keep bits,
  // scaled by 8, masked by what window w - 1 allows (the chain is one AND and
  // one table read per window).
  const char* tv = reinterpret_cast<const char*>(wt);
  uint32_t allowed8 = 0x78u;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const uint32_t k8 = (w == 0) ? (keep << 3) : (w == 1) ? (keep << 1) : (keep >> (2 * w - 3));
    const uint32_t off = k8 & allowed8 & 0x78u;
    const uint2 ev = *reinterpret_cast<const uint2*>(tv + off);
    const uint2 en = *reinterpret_cast<const uint2*>(tv + 128 + off);
    val_out[w] = __byte_perm(P[w], P[w + 1], ev.x) & ev.y;
    nib_out[w] = static_cast<uint8_t>(en.y);
    allowed8 = en.x;
  }
  return keep;
}

// Groups per lane: a bf16 lane takes at least 16 elements (two 16-byte
// loads), so that small groups (M = 4, 8) do not make the CTA task tiny.
__host__ __device__ constexpr int prune_groups_per_lane(int M, int elem_bytes) { return (elem_bytes == 2 && M < 16) ? 16 / M : 1; }

// Loads the G groups of one lane; a lane that runs past the end of the row
// (only the last lane of a row whose group count is not a multiple of G)
// loads its valid groups one by one and zeroes the rest.
template <int M, int G, typename T>
__device__ __forceinline__ void load_lane(const T* __restrict__ p, int64_t nvalid, GroupRaw<M * G, T>& g) {
  if (nvalid >= G) { load_raw<M * G, T>(p, g); return; }
  if constexpr (G > 1) {
#pragma unroll
    for (int i = 0; i < GroupRaw<M * G, T>::NV; ++i) g.v[i] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int j = 0; j < G; ++j) {
      if (j < nvalid) {
        if constexpr (M == 8) {
          g.v[j] = __ldg(reinterpret_cast<const uint4*>(p) + j);
        } else {
          const uint2 u = __ldg(reinterpret_cast<const uint2*>(p) + j);
          if (j % 2 == 0) { g.v[j / 2].x = u.x; g.v[j / 2].y = u.y; }
          else { g.v[j / 2].z = u.x; g.v[j / 2].w = u.y; }
        }
      }
    }
  }
}

// One CTA task = 16 consecutive rows x 32 lanes of G consecutive groups (a
// "chunk" of the row group); warp w takes rows 2w and 2w+1.  A task row holds
// 32*G*NW windows, exactly G*NW metadata blocks of 32 windows, and 16 rows are
// one contiguous 256-byte run inside a block (lanes 16j..16j+15 of the
// tensor-memory image), so the CTA writes its metadata as whole 16-byte lane
// rows.  Per row: pruned (entry kept iff fewer than N entries beat it), split
// over windows (window w takes the lowest two not yet placed kept entries of
// positions 2w..2w+3; one entry is paired with the lowest other local index,
// none gives (0, 1); padded slots hold +0.0), values written through a
// shared-memory staging row that leaves as one bulk copy (two staging rows
// per warp, so a copy reads while the other row is formed).  Rows past `rows`
// (up to the 128-row padding of the image) and windows past K'/4 get the
// index pair (0, 1).
//
// The grid is persistent: CTA b takes tasks b, b + gridDim.x, ... (row-group
// major), stepped without divisions.  Each warp keeps the two rows it works
// on in registers and requests the next task's row k as soon as it has
// consumed row k of the current one, so one row's loads are in flight while
// the other is processed and while the CTA writes the metadata.
constexpr int kPruneWarps = 8;

// Resident CTAs per SM the register budget is sized for: bf16 groups of up to
// 16 run four CTAs per SM, M = 32 three (80 registers; measured faster than
// two CTAs of 123 registers, and than four with spills); fp32 CTAs are larger.
__host__ __device__ constexpr int prune_min_blocks(int M, int elem_bytes) {
  return elem_bytes != 2 ? 1 : (M >= 32 ? 3 : 4);
}

// Task geometry: chunks per row group, ceil(groups / (32 G)), and the task
// count, (rows rounded up to 128) / 16 * cpr.
struct PruneGrid {
  uint32_t cpr;
  uint32_t tasks;
};

// Q8 = true (bf16 input only) writes the kept values as E4M3 codes --
// code = e4m3(v * (1 / row_scale[r])) -- two bytes per window instead of two
// bf16, and the metadata as the 8-bit image (row m, window j of a 128 x 128-K
// block at byte 16 m + j/2, low nibble for even j).
//
// XF = true (bf16 input only) is the transform mode of the per-token
// corrections: with row_shift, every element is first replaced by
// bf16(fl32(x - row_shift[r])) and the prune runs on that (D-PTS); with
// stats, each (row, chunk of 32 G groups) leaves the fp64 sum and sum of
// squares of its kept entries at stats[(r * chunks + chunk) * 2] for the VAR
// factor.
// SPLIT = true (bf16 weights, M = 8, 16, 32) writes the windows of each row
// in the split order: every group's even windows (which tile it, so that the
// matching lifted activations are the raw ones), then every group's odd
// windows.  A task row stages its even windows first; its metadata blocks go
// to the even region (blocks below K/128) and the odd region after it.
template <int M, typename T, bool Q8 = false, bool XF = false, bool SPLIT = false>
__global__ void __launch_bounds__(kPruneWarps * 32, prune_min_blocks(M, sizeof(T)))
k_prune_compress(const T* __restrict__ src, int64_t rows, int64_t K, int64_t ld, int N,
                 uint32_t* __restrict__ mask_out, void* __restrict__ vals_out,
                 uint8_t* __restrict__ meta_out, int64_t Kl, int64_t KB, PruneGrid pg,
                 const float* __restrict__ row_scale, const float* __restrict__ row_shift,
                 double* __restrict__ stats) {
  static_assert(!Q8 || sizeof(T) == 2, "8-bit output from bf16 input");
  static_assert(!XF || (sizeof(T) == 2 && !Q8), "transform mode: bf16 input, bf16 output");
  static_assert(!SPLIT || (sizeof(T) == 2 && !Q8 && !XF && M % 4 == 0 && M >= 8), "split order: bf16 weights");
  constexpr int G = prune_groups_per_lane(M, static_cast<int>(sizeof(T)));
  constexpr int NW = M / 2 - 1;                   // windows per group
  constexpr int NWL = G * NW;                     // windows per lane
  constexpr int WIN = 32 * NWL;                   // windows per task row = NWL blocks
  constexpr int LM = G * M;                       // elements (keep bits) per lane
  constexpr int NE = M / 4, NO = M / 4 - 1;       // split order: even and odd windows per group
  constexpr int WIN_E = 32 * G * NE;              // split order: even windows per task row
  constexpr int NWLE = G * NE;                    // split order: even metadata blocks per task row
  // staged rows of 768 bytes and more leave as bulk copies; shorter ones (2:4)
  // were measured faster as 16-byte stores by the lanes
  constexpr bool kBulkRow = WIN * (Q8 ? 2 : 4) >= 768;
  // index pairs of the task's 16 rows; two buffers (alternate tasks), so one
  // barrier per task separates a task's rows from its metadata pass, and the
  // next barrier separates that pass from the rewrite two tasks later
  __shared__ __align__(16) uint8_t s_nib_buf[2][16][WIN];
  __shared__ __align__(16) uint32_t s_val[kPruneWarps][kBulkRow ? 2 : 1][WIN];   // row k of the warp, staged
  __shared__ uint32_t s_mask[kPruneWarps][LM];
  __shared__ __align__(16) uint2 s_wt[32];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  griddep_launch_dependents();
  if (threadIdx.x < 16) window_rows(threadIdx.x, &s_wt[threadIdx.x], &s_wt[16 + threadIdx.x]);
  griddep_wait();                                      // inputs / outputs of the preceding kernel
  const int64_t groups = K / M;
  const int64_t mask_words = (K + 31) / 32;
  const bool vec_vals = Q8 ? (Kl % 32) == 0 : (Kl % 16) == 0;   // 16-byte output rows
  const uint32_t cpr = pg.cpr;
  const uint32_t drg = gridDim.x / cpr, dch = gridDim.x - drg * cpr;   // grid stride as (row group, chunk)
  uint32_t task = blockIdx.x;
  uint32_t rg = task / cpr, ch = task - rg * cpr;

  // row k of this warp in task (rg_, ch_) -> raw[k] (nothing for rows or
  // lanes past the operand)
  GroupRaw<LM, T> raw[2];
  auto load_row = [&](uint32_t rg_, uint32_t ch_, int k) {
    const int64_t r = static_cast<int64_t>(rg_) * 16 + 2 * warp + k;
    const int64_t gl = static_cast<int64_t>(ch_) * (32 * G) + lane * G;
    if (r < rows && gl < groups) load_lane<M, G, T>(src + r * ld + gl * M, groups - gl, raw[k]);
  };
  if (task < pg.tasks) {
    load_row(rg, ch, 0);
    load_row(rg, ch, 1);
  }
  __syncthreads();                                     // s_wt
  uint32_t tb = 0;                                     // s_nib buffer of this task
  while (task < pg.tasks) {
    uint8_t (*s_nib)[WIN] = s_nib_buf[tb];
    const uint32_t next = task + gridDim.x;
    uint32_t rg_n = rg + drg, ch_n = ch + dch;
    if (ch_n >= cpr) { ch_n -= cpr; ++rg_n; }
    const bool has_next = next < pg.tasks;
    const int64_t g0 = static_cast<int64_t>(ch) * (32 * G), gl = g0 + static_cast<int64_t>(lane) * G;
    const int ng = static_cast<int>((groups - g0) < 32 * G ? (groups - g0) : 32 * G);
    const int64_t r0 = static_cast<int64_t>(rg) * 16;
    if (r0 + 16 > rows || ng != 32 * G) {
      // a partial task: padding rows and windows carry the index pair (0, 1)
      for (int i = threadIdx.x; i < 16 * WIN / 4; i += blockDim.x)
        reinterpret_cast<uint32_t*>(&s_nib[0][0])[i] = 0x04040404u;
      __syncthreads();                                 // padding in place before any row writes
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int it = 2 * warp + k;
      const int64_t r = r0 + it;
      if (r < rows) {
        // the bulk store that last read this staging row (one task ago) is done reading
        if constexpr (kBulkRow) {
          if (lane == 0) bulk_wait_read1();
        }
        if (lane < LM) s_mask[warp][lane] = 0u;
        __syncwarp();
        float inv = 1.0f;
        if constexpr (Q8) inv = __frcp_rn(row_scale[r]);
        double st[2] = {0.0, 0.0};                     // transform mode: kept sums of this lane
        if (gl < groups) {
          uint32_t vals[NWL];
          uint8_t nibs[NWL];
          uint32_t keep = 0u;
          if constexpr (sizeof(T) == 2) {
            uint32_t PL[LM / 2];
#pragma unroll
            for (int p = 0; p < LM / 2; ++p) {
              const uint4& q = raw[k].v[p / 4];
              PL[p] = (p % 4 == 0) ? q.x : (p % 4 == 1) ? q.y : (p % 4 == 2) ? q.z : q.w;
            }
            if constexpr (XF) {
              if (row_shift != nullptr) {
                const float mu = row_shift[r];
#pragma unroll
                for (int p = 0; p < LM / 2; ++p) {
                  const __nv_bfloat162 h = __floats2bfloat162_rn(__fsub_rn(__uint_as_float(PL[p] << 16), mu),
                                                                 __fsub_rn(__uint_as_float(PL[p] & 0xFFFF0000u), mu));
                  PL[p] = *reinterpret_cast<const uint32_t*>(&h);
                }
              }
            }
#pragma unroll
            for (int j = 0; j < G; ++j) {
              uint32_t P[M / 2];
#pragma unroll
              for (int p = 0; p < M / 2; ++p) P[p] = PL[j * (M / 2) + p];
              uint32_t vj[NW];
              uint8_t nj[NW];
              const uint32_t kj = compress_group_bf16<M>(P, N, s_wt, vj, nj);
              const bool valid = (G == 1) || (gl + j < groups);
#pragma unroll
              for (int w = 0; w < NW; ++w) { vals[j * NW + w] = vj[w]; nibs[j * NW + w] = valid ? nj[w] : 0x4; }
              if (valid) keep |= (M == 32 ? kj : (kj & ((1u << M) - 1u))) << (j * M);
            }
          } else {
            keep = compress_group<M, T>(raw[k], N, vals, nibs);
          }
          if constexpr (XF) {
            if (stats != nullptr) {
              // kept values: both slots of every window of the valid groups
              // (padded slots hold +0.0)
#pragma unroll
              for (int w = 0; w < NWL; ++w) {
                if ((G == 1) || (gl + w / NW < groups)) {
                  const double a = __uint_as_float(vals[w] << 16), b = __uint_as_float(vals[w] & 0xFFFF0000u);
                  st[0] += a + b;
                  st[1] += a * a + b * b;
                }
              }
            }
          }
#pragma unroll
          for (int w = 0; w < NWL; ++w) {
            // staging slot of lane window w (group w / NW of the lane, window w % NW)
            int pos = lane * NWL + w;
            if constexpr (SPLIT) {
              const int j = w / NW, wi = w % NW;
              pos = (wi % 2 == 0) ? lane * G * NE + j * NE + wi / 2 : WIN_E + lane * G * NO + j * NO + wi / 2;
            }
            if constexpr (Q8) {
              reinterpret_cast<uint16_t*>(&s_val[warp][kBulkRow ? k : 0][0])[pos] = static_cast<uint16_t>(
                  e4m3x2(__fmul_rn(elem_f32(static_cast<uint16_t>(vals[w] & 0xFFFFu)), inv),
                         __fmul_rn(elem_f32(static_cast<uint16_t>(vals[w] >> 16)), inv)));
            } else {
              s_val[warp][kBulkRow ? k : 0][pos] = vals[w];
            }
            s_nib[it][pos] = nibs[w];
          }
          if (mask_out != nullptr)
            atomicOr(&s_mask[warp][(lane * LM) / 32],
                     (LM == 32 ? keep : (keep & ((1u << LM) - 1u))) << ((lane * LM) % 32));
        }
        // raw[k] is consumed: request this warp's row k of the next task
        if (has_next) load_row(rg_n, ch_n, k);
        // A whole task row (16-byte aligned start and size) leaves as one
        // bulk copy issued by lane 0 (or as 16-byte stores when short); a
        // partial one is copied element by element.
        const bool bulk = kBulkRow && vec_vals && ng == 32 * G;
        if (bulk) fence_proxy_async_smem();            // this lane's staging stores -> the copy engine
        __syncwarp();
        if constexpr (Q8) {
          uint16_t* vrow = static_cast<uint16_t*>(vals_out) + r * (Kl / 4) + g0 * NW;
          const uint16_t* sv16 = reinterpret_cast<const uint16_t*>(&s_val[warp][kBulkRow ? k : 0][0]);
          if (bulk) {
            if (lane == 0) bulk_store(vrow, sv16, WIN * 2);
          } else if (vec_vals && ng == 32 * G) {
            const uint4* sv = reinterpret_cast<const uint4*>(sv16);
            uint4* dv = reinterpret_cast<uint4*>(vrow);
            for (int i = lane; i < WIN / 8; i += 32) dv[i] = sv[i];
          } else {
            for (int i = lane; i < ng * NW; i += 32) vrow[i] = sv16[i];
          }
        } else if constexpr (SPLIT) {
          // the even run and the odd run of the task row, each to its region
          uint32_t* vrow = static_cast<uint32_t*>(vals_out) + r * (Kl / 4);
          uint32_t* ve = vrow + g0 * NE;
          uint32_t* vo = vrow + K / 4 + g0 * NO;
          const uint32_t* sv = &s_val[warp][kBulkRow ? k : 0][0];
          if (bulk) {
            if (lane == 0) {
              bulk_store(ve, sv, WIN_E * 4);
              bulk_store(vo, sv + WIN_E, (WIN - WIN_E) * 4);
            }
          } else {
            for (int i = lane; i < ng * NE; i += 32) ve[i] = sv[i];
            for (int i = lane; i < ng * NO; i += 32) vo[i] = sv[WIN_E + i];
          }
        } else {
          uint32_t* vrow = static_cast<uint32_t*>(vals_out) + r * (Kl / 4) + g0 * NW;
          if (bulk) {
            if (lane == 0) bulk_store(vrow, &s_val[warp][kBulkRow ? k : 0][0], WIN * 4);
          } else if (vec_vals && ng == 32 * G) {
            const uint4* sv = reinterpret_cast<const uint4*>(&s_val[warp][kBulkRow ? k : 0][0]);
            uint4* dv = reinterpret_cast<uint4*>(vrow);
            for (int i = lane; i < WIN / 4; i += 32) dv[i] = sv[i];
          } else {
            for (int i = lane; i < ng * NW; i += 32) vrow[i] = s_val[warp][kBulkRow ? k : 0][i];
          }
        }
        if (mask_out != nullptr && lane < LM) {
          const int64_t wi = static_cast<int64_t>(ch) * LM + lane;
          if (wi < mask_words) mask_out[r * mask_words + wi] = s_mask[warp][lane];
        }
        if constexpr (XF) {
          if (stats != nullptr) {
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) st[i] += __shfl_xor_sync(0xFFFFFFFFu, st[i], o);
            if (lane == 0) reinterpret_cast<double2*>(stats)[r * cpr + ch] = make_double2(st[0], st[1]);
          }
        }
        __syncwarp();
      } else if (has_next) {
        load_row(rg_n, ch_n, k);
      }
      // one bulk group per (task, row k), empty or not, so that a wait for
      // all but the newest group always covers this staging row's last copy
      if constexpr (kBulkRow) {
        if (lane == 0) bulk_commit();
      }
    }
    __syncthreads();
    // metadata: NWL blocks x 16 lane rows of 16 bytes.  Lane row L (0..15) of
    // block b holds rows L%8 and L%8+8 of the 16, windows 32b + 8c + 4(L/8) + 0..3
    // in word c (low half: first row, high half: second row).
    const int64_t rb = rg / 8;
    const int sub = static_cast<int>(rg % 8);
    if constexpr (Q8) {
      // 8-bit image: row `row` of the task, windows 32b .. 32b+31 -> 16 bytes
      for (int i = threadIdx.x; i < NWL * 16; i += blockDim.x) {
        const int b = i / 16, row = i % 16;
        const int64_t kb = static_cast<int64_t>(ch) * NWL + b;
        if (kb >= KB) continue;
        uint32_t wds[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t lo = *reinterpret_cast<const uint32_t*>(&s_nib[row][32 * b + 8 * c]);
          const uint32_t hi = *reinterpret_cast<const uint32_t*>(&s_nib[row][32 * b + 8 * c + 4]);
          wds[c] = __byte_perm(lo | (lo >> 4), hi | (hi >> 4), 0x6420);
        }
        *reinterpret_cast<uint4*>(meta_out + (rb * KB + kb) * 2048 + (sub * 16 + row) * 16) =
            make_uint4(wds[0], wds[1], wds[2], wds[3]);
      }
    } else {
      for (int i = threadIdx.x; i < NWL * 16; i += blockDim.x) {
        const int b = i / 16, L = i % 16;
        int64_t kb = static_cast<int64_t>(ch) * NWL + b;
        if constexpr (SPLIT) {
          // even blocks below K/128 (padding blocks of a short last chunk are
          // dropped there), odd blocks from K/128 on
          if (b < NWLE) {
            kb = static_cast<int64_t>(ch) * NWLE + b;
            if (kb >= K / 128) continue;
          } else {
            kb = K / 128 + static_cast<int64_t>(ch) * (NWL - NWLE) + (b - NWLE);
          }
        }
        if (kb >= KB) continue;
        const int i8 = L % 8, h = L / 8;
        uint32_t wds[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int j = 32 * b + 8 * c + 4 * h;
          // four nibble bytes n0..n3 -> bytes 0 and 2 of x | x >> 4 hold n0 | n1 << 4 and n2 | n3 << 4
          const uint32_t lo = *reinterpret_cast<const uint32_t*>(&s_nib[i8][j]);
          const uint32_t hi = *reinterpret_cast<const uint32_t*>(&s_nib[i8 + 8][j]);
          wds[c] = __byte_perm(lo | (lo >> 4), hi | (hi >> 4), 0x6420);
        }
        *reinterpret_cast<uint4*>(meta_out + (rb * KB + kb) * 2048 + sub * 256 + L * 16) =
            make_uint4(wds[0], wds[1], wds[2], wds[3]);
      }
    }
    task = next;
    tb ^= 1u;
    rg = rg_n;
    ch = ch_n;
  }
  if constexpr (kBulkRow) {
    if (lane == 0) bulk_wait_all();                    // the staging rows stay until the copies are done
  }
}

// Lift: dst[r][g*4(n-1) + 4w + j] = src[r][g*2n + 2w + j].  A CTA lifts one
// segment of kLiftElems input elements of kLiftRows rows: the segments are
// brought into shared memory (as bf16) with 16-byte loads, all in flight
// together, then each thread writes whole 16-byte chunks of the lifted rows --
// two windows of four -- so that every warp store covers 512 contiguous
// bytes.  Row blocks beyond the grid's y extent are taken in a loop.
constexpr int kLiftElems = 2048;
constexpr int kLiftRows = 4;

__device__ __forceinline__ void to_bf16_words(const uint4& u, uint16_t* out, const uint16_t*) {
  *reinterpret_cast<uint4*>(out) = u;
}
__device__ __forceinline__ void to_bf16_words(const uint4& u, uint16_t* out, const uint32_t*) {
  const uint32_t a = to_bf16_bits(u.x), b = to_bf16_bits(u.y), c = to_bf16_bits(u.z), d = to_bf16_bits(u.w);
  *reinterpret_cast<uint2*>(out) = make_uint2(a | (b << 16), c | (d << 16));
}

template <int M, typename T>
__global__ void __launch_bounds__(256)
k_lift(const T* __restrict__ src, int64_t rows, int64_t K, int64_t ld,
       uint16_t* __restrict__ dst, int64_t Kl) {
  constexpr int NW = M / 2 - 1;                          // windows per group
  constexpr int PV = 16 / static_cast<int>(sizeof(T));   // elements per 16-byte load
  __shared__ __align__(16) uint16_t s_x[kLiftRows][kLiftElems];
  const int64_t e0 = static_cast<int64_t>(blockIdx.x) * kLiftElems;
  const int n_in = static_cast<int>(K - e0 < kLiftElems ? K - e0 : kLiftElems);   // a multiple of M
  const int nwin = n_in / M * NW;
  griddep_launch_dependents();
  griddep_wait();
  for (int64_t r0 = static_cast<int64_t>(blockIdx.y) * kLiftRows; r0 < rows;
       r0 += static_cast<int64_t>(gridDim.y) * kLiftRows) {
    const int nr = static_cast<int>(rows - r0 < kLiftRows ? rows - r0 : kLiftRows);
    if (nr == kLiftRows && n_in == kLiftElems) {
      // whole block: every load of the kLiftRows rows issued before any store
      constexpr int J = kLiftElems / (256 * PV);
      uint4 u[kLiftRows][J];
#pragma unroll
      for (int k = 0; k < kLiftRows; ++k)
#pragma unroll
        for (int j = 0; j < J; ++j)
          u[k][j] = __ldg(reinterpret_cast<const uint4*>(src + (r0 + k) * ld + e0 + (threadIdx.x + 256 * j) * PV));
#pragma unroll
      for (int k = 0; k < kLiftRows; ++k)
#pragma unroll
        for (int j = 0; j < J; ++j) to_bf16_words(u[k][j], &s_x[k][(threadIdx.x + 256 * j) * PV], src);
    } else {
#pragma unroll
    for (int k = 0; k < kLiftRows; ++k) {
      if (k < nr) {
        const T* row = src + (r0 + k) * ld + e0;
        for (int i = threadIdx.x * PV; i < n_in; i += blockDim.x * PV) {
          if (i + PV <= n_in) {
            to_bf16_words(__ldg(reinterpret_cast<const uint4*>(row + i)), &s_x[k][i], row);
          } else if constexpr (sizeof(T) == 2) {         // a bf16 row ending in half a 16-byte word
            *reinterpret_cast<uint2*>(&s_x[k][i]) = __ldg(reinterpret_cast<const uint2*>(row + i));
          }
        }
      }
    }
    }
    __syncthreads();
    for (int k = 0; k < nr; ++k) {
      const uint32_t* s_w = reinterpret_cast<const uint32_t*>(&s_x[k][0]);
      uint16_t* out = dst + (r0 + k) * Kl + e0 / M * 4 * NW;
      for (int c = threadIdx.x; 2 * c < nwin; c += blockDim.x) {
        const int w0 = 2 * c, w1 = 2 * c + 1;
        const int s0 = (w0 / NW) * M + 2 * (w0 % NW);    // even element index: a 4-byte boundary
        const uint32_t a0 = s_w[s0 / 2], a1 = s_w[s0 / 2 + 1];
        if (w1 < nwin) {
          const int s1 = (w1 / NW) * M + 2 * (w1 % NW);
          reinterpret_cast<uint4*>(out)[c] = make_uint4(a0, a1, s_w[s1 / 2], s_w[s1 / 2 + 1]);
        } else {
          reinterpret_cast<uint2*>(out)[2 * c] = make_uint2(a0, a1);
        }
      }
    }
    __syncthreads();                                     // s_x is refilled for the next row block
  }
}

// ------------------------------------------------------------- hybrid prep

// Odd-window lift in place (the split window order): x [rows][ld] holds X in
// columns [0, K); columns [K, K') receive, group by group, the odd windows of
// X.  Odd window o of a group covers its elements 4o + 2 .. 4o + 5, i.e. its
// 32-bit words 2o + 1, 2o + 2, so a group's odd windows are its words 1 ..
// 2(M/4 - 1): the group without its first and last two elements.  A thread
// takes pairs of groups of one row (K % 128 == 0 keeps the group count even),
// several pairs' 16-byte loads in flight before their 16-byte stores.
template <int M>
__global__ void __launch_bounds__(256) k_lift_odd(uint16_t* x, int64_t rows, int64_t K, int64_t ld) {
  static_assert(M % 8 == 0 && M >= 8, "two groups make whole 16-byte loads and stores");
  constexpr int NO = M / 4 - 1;                   // odd windows per group
  constexpr int U = M == 8 ? 4 : (M == 16 ? 2 : 1);   // group pairs per thread and step, loads in flight together
  griddep_launch_dependents();
  griddep_wait();                                      // X may come from the preceding kernel
  const int64_t pairs = K / M / 2;                     // group pairs per row
  const int64_t total = rows * pairs;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t base = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; base < total;
       base += U * stride) {
    uint32_t w[U][M];                                  // U pairs of groups, M / 2 words per group
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t idx = base + u * stride;
      if (idx < total) {
        const int64_t r = idx / pairs, t = idx - r * pairs;
        const uint4* src = reinterpret_cast<const uint4*>(x + r * ld + t * 2 * M);
#pragma unroll
        for (int i = 0; i < M / 4; ++i) {
          const uint4 q = src[i];
          w[u][4 * i] = q.x; w[u][4 * i + 1] = q.y; w[u][4 * i + 2] = q.z; w[u][4 * i + 3] = q.w;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t idx = base + u * stride;
      if (idx < total) {
        const int64_t r = idx / pairs, t = idx - r * pairs;
        uint32_t o[4 * NO];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int k = 0; k < 2 * NO; ++k) o[h * 2 * NO + k] = w[u][h * (M / 2) + 1 + k];
        uint4* dst = reinterpret_cast<uint4*>(x + r * ld + K + t * 8 * NO);
#pragma unroll
        for (int i = 0; i < NO; ++i) dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
      }
    }
  }
}

// colnorm[c] = sum over rows r ascending of w[r][c]^2, fp64 (each square of a
// bf16 value is exact in fp64, so fused and unfused updates agree).
__global__ void k_colnorm_f64(const uint16_t* __restrict__ w, int64_t O, int64_t K,
                              double* __restrict__ colnorm) {
  griddep_wait();
  const int64_t c = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (c >= K) return;
  double s = 0.0;
  for (int64_t r = 0; r < O; ++r) {
    const double v = static_cast<double>(__uint_as_float(static_cast<uint32_t>(w[r * K + c]) << 16));
    s += v * v;
  }
  colnorm[c] = s;
}

// Column c is dense iff fewer than D columns beat it (larger energy, or equal
// energy and lower index).
__global__ void k_hybrid_rank(const double* __restrict__ colnorm, int64_t K, int64_t D,
                              uint8_t* __restrict__ is_dense) {
  griddep_wait();
  const int64_t c = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (c >= K) return;
  const double e = colnorm[c];
  int64_t beaten_by = 0;
  for (int64_t c2 = 0; c2 < K; ++c2) {
    const double e2 = colnorm[c2];
    beaten_by += (e2 > e || (e2 == e && c2 < c)) ? 1 : 0;
  }
  is_dense[c] = beaten_by < D ? 1 : 0;
}

// perm = [sparse columns ascending | dense columns ascending].
__global__ void k_hybrid_perm(const uint8_t* __restrict__ is_dense, int64_t K, int64_t D,
                              int32_t* __restrict__ perm) {
  griddep_wait();
  const int64_t c = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (c >= K) return;
  const uint8_t mine = is_dense[c];
  int64_t before = 0;
  for (int64_t c2 = 0; c2 < c; ++c2) before += (is_dense[c2] == mine) ? 1 : 0;
  perm[mine ? (K - D) + before : before] = static_cast<int32_t>(c);
}

// dst_lo[r][i] = src[r][perm[i]] for i < split, dst_hi[r][i - split] for the rest.
__global__ void k_gather_cols(const uint16_t* __restrict__ src, int64_t rows, int64_t K,
                              const int32_t* __restrict__ perm, int64_t split,
                              uint16_t* __restrict__ dst_lo, uint16_t* __restrict__ dst_hi) {
  const int64_t total = rows * K;
  griddep_launch_dependents();
  griddep_wait();
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = t / K, i = t % K;
    const uint16_t v = src[r * K + perm[i]];
    if (i < split) dst_lo[r * split + i] = v;
    else dst_hi[r * (K - split) + (i - split)] = v;
  }
}

// Bounded-wait self test: waits on a barrier nobody arrives on.
__global__ void k_expire_wait(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, 0xDEB0u, limit_ns);
}

}  // namespace nm
