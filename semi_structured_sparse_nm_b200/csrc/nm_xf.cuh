// nm_xf.cuh -- the per-token corrections around the activation prune.
//
// D-PTS (dynamic shift): the token is centred on its mean before the prune,
//   mu[t] = fl32((sum_k x[t][k]) / K), the sum in fp64; the prune kernel's
//   transform mode prunes xs = bf16(fl32(x - mu)), and the GEMM epilogue adds
//   the shift back as mu[t] * s[o], s[o] = fl32(sum_k W[o][k]) (fp64 sum).
// VAR: the survivors of token t are rescaled by
//   alpha[t] = sqrt(var(x[t]) / var(kept xs[t])), var(u) = E[u^2] - E[u]^2
//   over all K entries; k_row_prep_bf16 leaves the fp64 moments of x, the
//   prune kernel's transform mode per-(row, chunk) fp64 sums of the kept
//   entries, k_xf_finalize adds those up, and the GEMM epilogue multiplies
//   the accumulator by alpha[t].
// Sums of bf16 values whose magnitudes span fewer than 53 - 8 - log2(K)
// binades are exact in fp64, so mu and s do not depend on the order in which
// the threads add.
#pragma once
#include "nm_device.cuh"

namespace nm {

// Sum and sum of squares of a bf16 row [0, K) in fp64, one warp per row:
// lane l takes the 16-byte words l, l + 32, ... (eight loads in flight per
// step), lane 0 the elements past the last whole word; every lane ends with
// the warp's totals.
__device__ __forceinline__ void row_sums_warp(const uint16_t* __restrict__ row, int64_t K, int lane,
                                              double& s, double& q) {
  const int64_t words = K / 8;
  double sh[4] = {0.0, 0.0, 0.0, 0.0}, qh[4] = {0.0, 0.0, 0.0, 0.0};   // four independent chains
  for (int64_t w0 = lane; w0 < words; w0 += 32 * 8) {
    uint4 u[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (w0 + 32 * j < words) u[j] = __ldg(reinterpret_cast<const uint4*>(row) + w0 + 32 * j);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (w0 + 32 * j < words) {
        const uint32_t wd[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const double a = __uint_as_float(wd[h] << 16), b = __uint_as_float(wd[h] & 0xFFFF0000u);
          sh[h] += a + b;
          qh[h] = fma(a, a, fma(b, b, qh[h]));
        }
      }
    }
  }
  s += (sh[0] + sh[1]) + (sh[2] + sh[3]);
  q += (qh[0] + qh[1]) + (qh[2] + qh[3]);
  if (lane == 0)
    for (int64_t k = words * 8; k < K; ++k) {
      const double a = elem_f32(row[k]);
      s += a;
      q += a * a;
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    q += __shfl_xor_sync(0xFFFFFFFFu, q, o);
  }
}

// out[r] = fl32(sum_k w[r][k]) (fp64 sum), one warp per row.
__global__ void __launch_bounds__(256)
k_row_sum_bf16(const uint16_t* __restrict__ w, int64_t rows, int64_t K, int64_t ld, float* __restrict__ out) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x % 32;
  for (int64_t r = blockIdx.x * 8 + threadIdx.x / 32; r < rows; r += static_cast<int64_t>(gridDim.x) * 8) {
    double s = 0.0, q = 0.0;
    row_sums_warp(w + r * ld, K, lane, s, q);
    if (lane == 0) out[r] = static_cast<float>(s);
  }
}

// Token statistics before the prune, one warp per row, one pass: the fp64
// sum and sum of squares of the incoming token.  With the shift,
// mu = fl32(sum / K) -> row_shift[r]; with VAR, moments[r] = {sum, sum of
// squares} (the variance a shift does not change).
__global__ void __launch_bounds__(256)
k_row_prep_bf16(const uint16_t* __restrict__ src, int64_t rows, int64_t K, int64_t ld, int shift,
                float* __restrict__ row_shift, double* __restrict__ moments) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x % 32;
  for (int64_t r = blockIdx.x * 8 + threadIdx.x / 32; r < rows; r += static_cast<int64_t>(gridDim.x) * 8) {
    double s = 0.0, q = 0.0;
    row_sums_warp(src + r * ld, K, lane, s, q);
    if (lane == 0) {
      if (shift) row_shift[r] = static_cast<float>(s / static_cast<double>(K));
      if (moments != nullptr) reinterpret_cast<double2*>(moments)[r] = make_double2(s, q);
    }
  }
}

// Per row, one warp: alpha = sqrt(var_in / var_kept) from moments[r] =
// {sum x, sum x^2} and the prune's partial sums of the kept entries
// kept[r][c] = {sum, sum of squares} (c = 0 .. chunks-1); 1 without VAR or
// when the kept token has no variance.  Without the shift, row_shift is set
// to 0.
__global__ void __launch_bounds__(256)
k_xf_finalize(const double* __restrict__ moments, const double* __restrict__ kept, int64_t rows, int64_t chunks,
              int64_t K, int zero_shift, float* __restrict__ row_scale, float* __restrict__ row_shift) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x % 32;
  const int64_t r = blockIdx.x * 8 + threadIdx.x / 32;
  if (r >= rows) return;
  float a = 1.0f;
  if (moments != nullptr) {
    double sp = 0.0, qp = 0.0;
    for (int64_t c = lane; c < chunks; c += 32) {
      const double2 p = reinterpret_cast<const double2*>(kept)[r * chunks + c];
      sp += p.x;
      qp += p.y;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sp += __shfl_xor_sync(0xFFFFFFFFu, sp, o);
      qp += __shfl_xor_sync(0xFFFFFFFFu, qp, o);
    }
    const double2 m = reinterpret_cast<const double2*>(moments)[r];
    const double kd = static_cast<double>(K);
    const double mi = m.x / kd, mp = sp / kd;
    const double vi = m.y / kd - mi * mi, vp = qp / kd - mp * mp;
    if (vp > 0.0) a = static_cast<float>(sqrt(vi / vp));
  }
  if (lane == 0) {
    row_scale[r] = a;
    if (zero_shift) row_shift[r] = 0.0f;
  }
}

}  // namespace nm
