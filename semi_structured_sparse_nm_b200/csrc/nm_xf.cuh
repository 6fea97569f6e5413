// nm_xf.cuh -- the per-token corrections around the activation prune.
//
// D-PTS (dynamic shift): the token is centred on its mean before the prune,
//   mu[t] = fl32((sum_k x[t][k]) / K), the sum in fp64; the prune kernel's
//   transform mode prunes xs = bf16(fl32(x - mu)), and the GEMM epilogue adds
//   the shift back as mu[t] * s[o], s[o] = fl32(sum_k W[o][k]) (fp64 sum).
// VAR: the survivors of token t are rescaled by
//   alpha[t] = sqrt(var(xs[t]) / var(kept xs[t])), var(u) = E[u^2] - E[u]^2
//   over all K entries; the prune kernel's transform mode leaves per-(row,
//   chunk) fp64 partial sums, k_xf_finalize adds them in chunk order, and the
//   GEMM epilogue multiplies the accumulator by alpha[t].
// Sums of bf16 values whose magnitudes span fewer than 53 - 8 - log2(K)
// binades are exact in fp64, so mu and s do not depend on the order in which
// the threads add.
#pragma once
#include "nm_device.cuh"

namespace nm {

// out[r] = fl32(sum_k src[r][k]) (MEAN: fl32(sum / K)), the sum in fp64; one
// CTA of 256 threads per row, 16-byte loads.
template <bool MEAN>
__global__ void __launch_bounds__(256)
k_row_sum_bf16(const uint16_t* __restrict__ src, int64_t rows, int64_t K, int64_t ld, float* __restrict__ out) {
  __shared__ double s_red[8];
  griddep_launch_dependents();
  griddep_wait();
  const int64_t K8 = K / 8 * 8;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const uint16_t* row = src + r * ld;
    double s = 0.0;
    for (int64_t i = static_cast<int64_t>(threadIdx.x) * 8; i < K8; i += 256 * 8) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(row + i));
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        s += static_cast<double>(__uint_as_float(w[j] << 16)) + static_cast<double>(__uint_as_float(w[j] & 0xFFFF0000u));
    }
    if (threadIdx.x == 0)
      for (int64_t i = K8; i < K; ++i) s += static_cast<double>(elem_f32(row[i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
      double t = 0.0;
#pragma unroll
      for (int i = 0; i < 8; ++i) t += s_red[i];
      out[r] = MEAN ? static_cast<float>(t / static_cast<double>(K)) : static_cast<float>(t);
    }
    __syncthreads();                                   // s_red is reused by the next row
  }
}

// Per row: alpha = sqrt(var_in / var_kept) from the prune's partial sums
// stats[r][c] = {sum xs, sum xs^2, sum kept, sum kept^2} (c = 0 .. chunks-1,
// added in that order); 1 without VAR or when the kept token has no
// variance.  Without the shift, row_shift is set to 0.
__global__ void k_xf_finalize(const double* __restrict__ stats, int64_t rows, int64_t chunks, int64_t K, int var,
                              int zero_shift, float* __restrict__ row_scale, float* __restrict__ row_shift) {
  griddep_launch_dependents();
  griddep_wait();
  const int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (r >= rows) return;
  float a = 1.0f;
  if (var) {
    double s = 0.0, q = 0.0, sp = 0.0, qp = 0.0;
    for (int64_t c = 0; c < chunks; ++c) {
      const double* p = stats + (r * chunks + c) * 4;
      s += p[0]; q += p[1]; sp += p[2]; qp += p[3];
    }
    const double kd = static_cast<double>(K);
    const double mi = s / kd, mp = sp / kd;
    const double vi = q / kd - mi * mi, vp = qp / kd - mp * mp;
    if (vp > 0.0) a = static_cast<float>(sqrt(vi / vp));
  }
  row_scale[r] = a;
  if (zero_shift) row_shift[r] = 0.0f;
}

}  // namespace nm
