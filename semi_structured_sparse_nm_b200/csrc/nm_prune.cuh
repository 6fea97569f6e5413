// nm_prune.cuh -- prune + window-compress, lift, and the offline hybrid
// selection kernels.  HBM-bound SIMT code: 128-bit coalesced loads, integer
// magnitude keys, results written in the layouts the GEMM consumes.
#pragma once
#include "nm_device.cuh"

namespace nm {

// Loads M consecutive elements (16-bit or 32-bit) of one group into registers
// with 8- or 16-byte vector loads.  The group start is 8-byte aligned for
// M = 4 bf16, 16-byte aligned otherwise (checked by the host).
template <int M, typename T>
__device__ __forceinline__ void load_group(const T* __restrict__ p, T (&x)[M]) {
  constexpr int BYTES = M * static_cast<int>(sizeof(T));
  if constexpr (BYTES % 16 == 0) {
    constexpr int V = BYTES / 16;
    constexpr int PER = 16 / static_cast<int>(sizeof(T));
#pragma unroll
    for (int v = 0; v < V; ++v) {
      uint4 u = __ldg(reinterpret_cast<const uint4*>(p) + v);
      const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
      for (int i = 0; i < PER; ++i) x[v * PER + i] = e[i];
    }
  } else {
    static_assert(BYTES == 8, "group of 8 bytes expected");
    uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
    for (int i = 0; i < M; ++i) x[i] = e[i];
  }
}

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

// One CTA per row (rows past `rows`, up to the 128-row padding of the
// metadata image, only write padding).  Each thread takes whole groups:
//   1. keys -> ranks -> keep bits (entry i kept iff fewer than N entries beat it);
//   2. greedy windows: window w takes the not yet placed kept entries among
//      positions 2w..2w+3 in ascending order, at most two;
//   3. the two values of window j go to vals[r][2j..2j+1] as one 32-bit store,
//      its index pair (i0 | i1 << 2) to a shared nibble row;
// then the CTA writes its row's nibbles into the metadata image, four windows
// (one 16-bit word) at a time.
template <int M, typename T>
__global__ void __launch_bounds__(128)
k_prune_compress(const T* __restrict__ src, int64_t rows, int64_t K, int64_t ld, int N,
                 uint32_t* __restrict__ mask_out, uint32_t* __restrict__ vals_out,
                 uint8_t* __restrict__ meta_out, int64_t Kl, int64_t KB) {
  constexpr int NW = M / 2 - 1;                 // windows per group (1 for 2:4)
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* s_nib = smem;                                             // KB*32 nibbles
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(smem + ((KB * 32 + 15) / 16) * 16);

  const int64_t r = blockIdx.x;
  const int64_t groups = K / M;
  const int64_t nwin = Kl / 4;
  const int64_t mask_words = (K + 31) / 32;
  const int tid = threadIdx.x;

  if (r < rows) {
    if (mask_out != nullptr)
      for (int64_t i = tid; i < mask_words; i += blockDim.x) s_mask[i] = 0u;
    for (int64_t j = nwin + tid; j < KB * 32; j += blockDim.x) s_nib[j] = 0x4;
    __syncthreads();
    const T* row = src + r * ld;
    for (int64_t g = tid; g < groups; g += blockDim.x) {
      T x[M];
      load_group<M, T>(row + g * M, x);
      // ranks by unique keys
      uint32_t keep = 0u;
#pragma unroll
      for (int i = 0; i < M; ++i) {
        const auto ki = order_key(x[i], i);
        int beaten_by = 0;
#pragma unroll
        for (int j = 0; j < M; ++j) beaten_by += (order_key(x[j], j) > ki) ? 1 : 0;
        keep |= (beaten_by < N ? 1u : 0u) << i;
      }
      // windows
      uint32_t placed = 0u;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        int held = 0, i0 = 0, i1 = 1;
        uint16_t v0 = 0, v1 = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int i = 2 * w + j;
          const bool take = ((keep >> i) & 1u) && !((placed >> i) & 1u) && held < 2;
          if (take) {
            const uint16_t b = to_bf16_bits(x[i]);
            if (held == 0) { i0 = j; v0 = b; } else { i1 = j; v1 = b; }
            placed |= 1u << i;
            ++held;
          }
        }
        if (held == 0) {
          i0 = 0; i1 = 1; v0 = 0; v1 = 0;
        } else if (held == 1) {
          const int a = i0, pad = (a == 0) ? 1 : 0;
          if (pad < a) { i1 = a; v1 = v0; i0 = pad; v0 = 0; }
          else { i1 = pad; v1 = 0; }
        }
        const int64_t jw = g * NW + w;
        vals_out[r * (Kl / 4) + jw] = static_cast<uint32_t>(v0) | (static_cast<uint32_t>(v1) << 16);
        s_nib[jw] = static_cast<uint8_t>(i0 | (i1 << 2));
      }
      if (mask_out != nullptr) {
        const int64_t bit = g * M;
        atomicOr(&s_mask[bit / 32], (M == 32 ? keep : (keep & ((1u << M) - 1u))) << (bit % 32));
      }
    }
    __syncthreads();
    if (mask_out != nullptr)
      for (int64_t i = tid; i < mask_words; i += blockDim.x) mask_out[r * mask_words + i] = s_mask[i];
  } else {
    for (int64_t j = tid; j < KB * 32; j += blockDim.x) s_nib[j] = 0x4;
    __syncthreads();
  }

  // metadata image: row m of row-block rb, four windows 4q..4q+3 per 16-bit word
  const int64_t rb = r / 128;
  const int m = static_cast<int>(r % 128);
  for (int64_t q = tid; q < KB * 8; q += blockDim.x) {
    const int64_t j = 4 * q;
    const int64_t kb = j / 32;
    const int jj = static_cast<int>(j % 32);
    const int c = jj / 8, h = (jj % 8) / 4;
    const uint16_t word = static_cast<uint16_t>(s_nib[j] | (s_nib[j + 1] << 4) |
                                                (s_nib[j + 2] << 8) | (s_nib[j + 3] << 12));
    const int lane = (m % 8) + 8 * h + 16 * (m / 16);
    const int64_t byte = (rb * KB + kb) * 2048 + lane * 16 + c * 4 + 2 * ((m / 8) % 2);
    *reinterpret_cast<uint16_t*>(meta_out + byte) = word;
  }
}

// Lift: dst[r][g*4(n-1) + 4w + j] = src[r][g*2n + 2w + j]; one thread per group.
template <int M, typename T>
__global__ void __launch_bounds__(256)
k_lift(const T* __restrict__ src, int64_t rows, int64_t K, int64_t ld,
       uint16_t* __restrict__ dst, int64_t Kl) {
  constexpr int NW = M / 2 - 1;
  const int64_t groups = K / M;
  const int64_t total = rows * groups;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = t / groups, g = t % groups;
    T x[M];
    load_group<M, T>(src + r * ld + g * M, x);
    uint2* out = reinterpret_cast<uint2*>(dst + r * Kl + g * 4 * NW);
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      uint2 v;
      v.x = static_cast<uint32_t>(to_bf16_bits(x[2 * w])) |
            (static_cast<uint32_t>(to_bf16_bits(x[2 * w + 1])) << 16);
      v.y = static_cast<uint32_t>(to_bf16_bits(x[2 * w + 2])) |
            (static_cast<uint32_t>(to_bf16_bits(x[2 * w + 3])) << 16);
      out[w] = v;
    }
  }
}

// ------------------------------------------------------------- hybrid prep

// colnorm[c] = sum over rows r ascending of w[r][c]^2, fp64 (each square of a
// bf16 value is exact in fp64, so fused and unfused updates agree).
__global__ void k_colnorm_f64(const uint16_t* __restrict__ w, int64_t O, int64_t K,
                              double* __restrict__ colnorm) {
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
