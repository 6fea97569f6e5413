// nm_fp8.cuh -- the 8-bit (E4M3) operand preparation.
//
// SlideSparse runs its online path as one fused kernel that quantises each
// token of the dense operand and writes it lifted; the weights are packed
// offline.  Here:
//   k_quant_lift_fp8  per row: amax, scale = amax / 448, codes of x / scale,
//                     written in the lifted window order (one pass over X);
//   k_row_scale_fp8   per row of W: scale = amax / 448;
//   k_quant_vals_fp8  codes of the compressed (kept) values with their row's
//                     scale;
//   k_meta_f16_to_8   the 16-bit metadata image re-laid as the 8-bit one
//                     (row-major: row m, window j of a 128 x 128-K block at
//                     byte 16 m + j / 2, low nibble for even j).
// Scales are IEEE fp32: scale = amax / 448 (correctly rounded division) and
// its reciprocal 1 / scale (correctly rounded); a value's code is taken from
// the fp32 product x * (1 / scale), nearest-even with saturation to +-448
// (cvt.rn.satfinite).
#pragma once
#include "nm_device.cuh"

namespace nm {

// Block-wide maximum of a non-negative value (256 threads).
__device__ __forceinline__ float block_max_256(float v, float* s_red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = s_red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) m = fmaxf(m, s_red[i]);
  return m;
}

__device__ __forceinline__ float fp8_scale_of(float amax) {
  return amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
}

// Per-token quantise + lift.  One warp per row, eight rows per CTA.  Lane l
// takes a contiguous run of groups (a multiple of four), so that its lifted
// codes are one contiguous run of whole 16-byte words.  Pass 1 reduces |x|
// over the lane's groups (16-byte loads) and the warp's lanes to the row
// maximum; pass 2 reads the groups again (from L1) four at a time, converts
// each element once -- code = e4m3(x * (1 / scale)) -- and forms each
// group's n-1 windows codes[r][g*4(n-1) + 4w + j] = code[g*2n + 2w + j] by
// byte permutes of the packed codes, stored as 16-byte words.
template <int M, typename T>
__device__ __forceinline__ void load_group_words(const T* __restrict__ p, uint32_t (&wd)[M * sizeof(T) / 4]) {
  constexpr int BYTES = M * static_cast<int>(sizeof(T));
  if constexpr (BYTES >= 16) {
#pragma unroll
    for (int v = 0; v < BYTES / 16; ++v) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(p) + v);
      wd[4 * v] = u.x; wd[4 * v + 1] = u.y; wd[4 * v + 2] = u.z; wd[4 * v + 3] = u.w;
    }
  } else {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    wd[0] = u.x; wd[1] = u.y;
  }
}

// element e of a group held as 32-bit words, as fp32
template <typename T, int WORDS>
__device__ __forceinline__ float group_elem(const uint32_t (&wd)[WORDS], int e) {
  if constexpr (sizeof(T) == 2) {
    const uint32_t w = wd[e / 2];
    return __uint_as_float((e % 2 == 0) ? (w << 16) : (w & 0xFFFF0000u));
  } else {
    return __uint_as_float(wd[e]);
  }
}

// The group's codes (four per word) and its NW window words.
template <int M, typename T>
__device__ __forceinline__ void quant_group_windows(const uint32_t (&wd)[M * sizeof(T) / 4], float inv,
                                                    uint32_t* win) {
  constexpr int NW = M / 2 - 1;
  constexpr int WORDS = M * static_cast<int>(sizeof(T)) / 4;
  uint32_t q[M / 4];
#pragma unroll
  for (int c = 0; c < M / 4; ++c) {
    const float f0 = group_elem<T, WORDS>(wd, 4 * c), f1 = group_elem<T, WORDS>(wd, 4 * c + 1);
    const float f2 = group_elem<T, WORDS>(wd, 4 * c + 2), f3 = group_elem<T, WORDS>(wd, 4 * c + 3);
    q[c] = e4m3x2(__fmul_rn(f0, inv), __fmul_rn(f1, inv)) | (e4m3x2(__fmul_rn(f2, inv), __fmul_rn(f3, inv)) << 16);
  }
  // window w = codes 2w .. 2w+3: word w/2 when w is even, else the upper
  // half of word (w-1)/2 and the lower half of the next one
#pragma unroll
  for (int w = 0; w < NW; ++w) win[w] = (w % 2 == 0) ? q[w / 2] : __byte_perm(q[w / 2], q[w / 2 + 1], 0x5432);
}

constexpr int kQuantWarps = 8;

// One warp per row; the grid's CTAs hold up to kQuantWarps warps (fewer for
// short batches, so that a few rows still spread over as many SMs).  Lane l
// takes groups l, l + 32, l + 64, ... so that each load instruction of the
// warp reads 32 consecutive groups.  With G > 0 the lane's groups (at most G)
// stay in registers between the maximum and the conversion; G = 0 reads them
// twice (the second time from L1).
template <int M, typename T, int G>
__global__ void __launch_bounds__(kQuantWarps * 32)
k_quant_lift_fp8(const T* __restrict__ src, int64_t rows, int64_t K, int64_t ld,
                 uint8_t* __restrict__ codes, float* __restrict__ scale_out, int64_t Kl) {
  constexpr int NW = M / 2 - 1;
  constexpr int WORDS = M * static_cast<int>(sizeof(T)) / 4;     // 32-bit words of one group
  griddep_launch_dependents();
  griddep_wait();
  const int wpb = blockDim.x / 32;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t groups = K / M;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * wpb + warp; r < rows; r += static_cast<int64_t>(gridDim.x) * wpb) {
    const T* row = src + r * ld;
    uint32_t* out = reinterpret_cast<uint32_t*>(codes + r * Kl);
    float amax = 0.0f;
    if constexpr (G > 0) {
      uint32_t wd[G][WORDS];
#pragma unroll
      for (int k = 0; k < G; ++k) {
        const int64_t g = lane + 32 * k;
        if (g < groups) {
          load_group_words<M, T>(row + g * M, wd[k]);
#pragma unroll
          for (int e = 0; e < M; ++e) amax = fmaxf(amax, fabsf(group_elem<T, WORDS>(wd[k], e)));
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      const float sc = fp8_scale_of(amax);
      const float inv = __frcp_rn(sc);
      if (lane == 0) scale_out[r] = sc;
#pragma unroll
      for (int k = 0; k < G; ++k) {
        const int64_t g = lane + 32 * k;
        if (g < groups) {
          uint32_t win[NW];
          quant_group_windows<M, T>(wd[k], inv, win);
#pragma unroll
          for (int w = 0; w < NW; ++w) out[g * NW + w] = win[w];
        }
      }
    } else {
      for (int64_t g = lane; g < groups; g += 32) {
        uint32_t wd[WORDS];
        load_group_words<M, T>(row + g * M, wd);
#pragma unroll
        for (int e = 0; e < M; ++e) amax = fmaxf(amax, fabsf(group_elem<T, WORDS>(wd, e)));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      const float sc = fp8_scale_of(amax);
      const float inv = __frcp_rn(sc);
      if (lane == 0) scale_out[r] = sc;
      for (int64_t g = lane; g < groups; g += 32) {
        uint32_t wd[WORDS], win[NW];
        load_group_words<M, T>(row + g * M, wd);
        quant_group_windows<M, T>(wd, inv, win);
#pragma unroll
        for (int w = 0; w < NW; ++w) out[g * NW + w] = win[w];
      }
    }
  }
}

// Groups per lane held in registers (at most 256 bytes of a row per lane),
// or 0 for the two-pass form.
__host__ __device__ constexpr int quant_groups_in_regs(int M, int elem_bytes) { return 256 / (M * elem_bytes); }

// scale[r] = amax(w[r][:]) / 448 for bf16 rows of length K (row stride ld).
__global__ void __launch_bounds__(256)
k_row_scale_fp8(const uint16_t* __restrict__ w, int64_t rows, int64_t K, int64_t ld, float* __restrict__ scale_out) {
  __shared__ float s_red[8];
  griddep_launch_dependents();
  griddep_wait();
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const uint16_t* row = w + r * ld;
    float amax = 0.0f;
    for (int64_t i = threadIdx.x; i < K; i += 256) amax = fmaxf(amax, fabsf(elem_f32(row[i])));
    const float sc = fp8_scale_of(block_max_256(amax, s_red));
    if (threadIdx.x == 0) scale_out[r] = sc;
    __syncthreads();
  }
}

// codes[r][i] = e4m3(vals[r][i] * (1 / scale[r])) for bf16 compressed values,
// nv values per row (a multiple of 8): eight values per thread.
__global__ void __launch_bounds__(256)
k_quant_vals_fp8(const uint16_t* __restrict__ vals, int64_t rows, int64_t nv, const float* __restrict__ scale,
                 uint8_t* __restrict__ codes) {
  griddep_launch_dependents();
  griddep_wait();
  const int64_t per_row = nv / 8, total = rows * per_row;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = t / per_row;
    const float inv = __frcp_rn(scale[r]);
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(vals) + t);
    const uint16_t* e = reinterpret_cast<const uint16_t*>(&u);
    uint32_t wd[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t lo = e4m3x2(__fmul_rn(elem_f32(e[4 * h]), inv), __fmul_rn(elem_f32(e[4 * h + 1]), inv));
      const uint32_t hi = e4m3x2(__fmul_rn(elem_f32(e[4 * h + 2]), inv), __fmul_rn(elem_f32(e[4 * h + 3]), inv));
      wd[h] = lo | (hi << 16);
    }
    reinterpret_cast<uint2*>(codes)[t] = make_uint2(wd[0], wd[1]);
  }
}

// The 16-bit metadata image (per 128 x 128-K block: row m, window j at lane
// (m%8) + 8((j%8)/4) + 16(m/16), word j/8, nibble (j%4) + 4((m/8)%2)) re-laid
// as the 8-bit image (row m, window j at byte 16 m + j/2, low nibble for even
// j).  One thread per (block, row).
__global__ void __launch_bounds__(256)
k_meta_f16_to_8(const uint8_t* __restrict__ in, int64_t blocks, uint8_t* __restrict__ out) {
  griddep_launch_dependents();
  griddep_wait();
  const int64_t total = blocks * 128;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t blk = t / 128;
    const int m = static_cast<int>(t % 128);
    const uint8_t* b = in + blk * 2048;
    uint32_t wd[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int lane = (m % 8) + 8 * ((j % 8) / 4) + 16 * (m / 16);
      const int nb = (j % 4) + 4 * ((m / 8) % 2);
      const uint32_t q = (b[lane * 16 + (j / 8) * 4 + nb / 2] >> (4 * (nb % 2))) & 0xFu;
      wd[j / 8] |= q << (4 * (j % 8));
    }
    reinterpret_cast<uint4*>(out + blk * 2048)[m] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
  }
}

}  // namespace nm
