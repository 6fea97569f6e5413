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

// Per-token quantise + lift.  One CTA per row.  Pass 1 reduces |x| over the
// row to its maximum (16-byte loads, block reduction); pass 2 takes one group
// of M elements per thread (read again, now from L1), converts each element
// once -- code = e4m3(x * (1 / scale)) -- and forms the group's n-1 windows
// codes[r][g*4(n-1) + 4w + j] = code[g*2n + 2w + j] by byte permutes of the
// packed codes, one 4-byte store per window.
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

template <int M, typename T>
__global__ void __launch_bounds__(256)
k_quant_lift_fp8(const T* __restrict__ src, int64_t rows, int64_t K, int64_t ld,
                 uint8_t* __restrict__ codes, float* __restrict__ scale_out, int64_t Kl) {
  constexpr int NW = M / 2 - 1;
  constexpr int PV = 16 / static_cast<int>(sizeof(T));
  constexpr int WORDS = M * static_cast<int>(sizeof(T)) / 4;     // 32-bit words of one group
  __shared__ float s_red[8];
  griddep_launch_dependents();
  griddep_wait();
  const int64_t groups = K / M;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const T* row = src + r * ld;
    float amax = 0.0f;
    for (int64_t i = static_cast<int64_t>(threadIdx.x) * PV; i < K; i += 256 * PV) {
      if (i + PV <= K) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(row + i));
        const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
        for (int j = 0; j < PV; ++j) amax = fmaxf(amax, fabsf(elem_f32(e[j])));
      } else if constexpr (sizeof(T) == 2) {           // a bf16 row ending in half a 16-byte word
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(row + i));
        const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) amax = fmaxf(amax, fabsf(elem_f32(e[j])));
      }
    }
    const float sc = fp8_scale_of(block_max_256(amax, s_red));
    const float inv = __frcp_rn(sc);
    if (threadIdx.x == 0) scale_out[r] = sc;
    uint32_t* out = reinterpret_cast<uint32_t*>(codes + r * Kl);
    for (int64_t g = threadIdx.x; g < groups; g += 256) {
      uint32_t wd[WORDS];
      load_group_words<M, T>(row + g * M, wd);
      uint32_t q[M / 4];                               // codes of the group, four per word
#pragma unroll
      for (int c = 0; c < M / 4; ++c) {
        float f[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int e = 4 * c + j;
          if constexpr (sizeof(T) == 2) {
            const uint32_t w = wd[e / 2];
            f[j] = __uint_as_float((e % 2 == 0) ? (w << 16) : (w & 0xFFFF0000u));
          } else {
            f[j] = __uint_as_float(wd[e]);
          }
        }
        q[c] = e4m3x2(__fmul_rn(f[0], inv), __fmul_rn(f[1], inv)) |
               (e4m3x2(__fmul_rn(f[2], inv), __fmul_rn(f[3], inv)) << 16);
      }
      // window w = codes 2w .. 2w+3: word w/2 when w is even, else the upper
      // half of word (w-1)/2 and the lower half of the next one
#pragma unroll
      for (int w = 0; w < NW; ++w)
        out[g * NW + w] = (w % 2 == 0) ? q[w / 2] : __byte_perm(q[w / 2], q[w / 2 + 1], 0x5432);
    }
    __syncthreads();                                   // s_red is reused by the next row
  }
}

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
