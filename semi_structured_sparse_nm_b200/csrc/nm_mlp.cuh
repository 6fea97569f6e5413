// nm_mlp.cuh -- the GLU-MLP mapping of the hybrid format.
//
// One set of intermediate indices stays dense in all three projections.  The
// indices are ranked by the summed fp64 energies of the up and gate rows and
// the down column, permuted into [sparse ascending | dense ascending], and
// the projections are packed so that the permutation is absorbed inside the
// MLP:
//   up, gate   output-split: rows [up_s; gate_s] 2:4 along the model
//              dimension, rows [up_d; gate_d] dense -- one GEMM whose output
//              columns come out as [up_s | gate_s | up_d | gate_d];
//   h          silu(gate) * up, written in the permuted order [sparse | dense];
//   down       input-split on h: its first Is input columns 2:4 (in the
//              permuted order), the last D dense.
// Offline kernels here: row energies (sequential, k ascending, as the column
// energies of nm_prune.cuh), the summed score, the row gather of up and gate.
// Online: the SiLU gate.
#pragma once
#include "nm_device.cuh"

namespace nm {

// rownorm[r] = sum_{k ascending} w[r][k]^2 (fp64), one thread per row.
__global__ void k_rownorm_f64(const uint16_t* __restrict__ w, int64_t O, int64_t K, double* __restrict__ rownorm) {
  griddep_launch_dependents();
  griddep_wait();
  const int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (r >= O) return;
  const uint16_t* row = w + r * K;
  double s = 0.0;
  for (int64_t k = 0; k < K; ++k) {
    const double v = static_cast<double>(elem_f32(row[k]));
    s += v * v;
  }
  rownorm[r] = s;
}

// score[i] = (a[i] + b[i]) + c[i] in fp64, in that order.
__global__ void k_add3_f64(const double* __restrict__ a, const double* __restrict__ b, const double* __restrict__ c,
                           int64_t n, double* __restrict__ out) {
  griddep_launch_dependents();
  griddep_wait();
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i < n) out[i] = (a[i] + b[i]) + c[i];
}

// Row gather of up and gate by the permutation: for j < Is,
// sparse[j] = up[perm[j]] and sparse[Is + j] = gate[perm[j]]; for j >= Is,
// dense[j - Is] = up[perm[j]] and dense[D + j - Is] = gate[perm[j]].  Rows of
// d bf16 (d a multiple of 8), one 16-byte chunk per thread step.
__global__ void k_gather_rows_ug(const uint16_t* __restrict__ up, const uint16_t* __restrict__ gate, int64_t d,
                                 const int32_t* __restrict__ perm, int64_t I, int64_t Is,
                                 uint16_t* __restrict__ sparse, uint16_t* __restrict__ dense) {
  griddep_launch_dependents();
  griddep_wait();
  const int64_t D = I - Is, chunks = d / 8, total = 2 * I * chunks;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = t / chunks, c = t % chunks;
    const bool is_gate = row >= I;
    const int64_t j = is_gate ? row - I : row;
    const uint16_t* src = (is_gate ? gate : up) + static_cast<int64_t>(perm[j]) * d;
    uint16_t* dst = j < Is ? sparse + ((is_gate ? Is : 0) + j) * d : dense + ((is_gate ? D : 0) + (j - Is)) * d;
    reinterpret_cast<uint4*>(dst)[c] = __ldg(reinterpret_cast<const uint4*>(src) + c);
  }
}

// h[t][j] = silu(g) * u in fp32 (silu(z) = z / (1 + e^-z)), bf16 in and out,
// from the up/gate product Y [B x 2I] with columns [up_s | gate_s | up_d |
// gate_d]: for j < Is, u = Y[t][j], g = Y[t][Is + j]; for j >= Is,
// u = Y[t][2 Is + j - Is], g = Y[t][2 Is + D + j - Is].  Eight outputs per
// thread step (Is and D are multiples of 8).
__global__ void k_silu_mul(const uint16_t* __restrict__ y, int64_t B, int64_t I, int64_t Is,
                           uint16_t* __restrict__ h) {
  griddep_launch_dependents();
  griddep_wait();
  const int64_t D = I - Is, per_row = I / 8, total = B * per_row;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = t / per_row, j = (t % per_row) * 8;
    const uint16_t* yr = y + b * 2 * I;
    const int64_t ju = j < Is ? j : 2 * Is + (j - Is);
    const int64_t jg = j < Is ? Is + j : 2 * Is + D + (j - Is);
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(yr + ju));
    const uint4 g = __ldg(reinterpret_cast<const uint4*>(yr + jg));
    const uint16_t* ue = reinterpret_cast<const uint16_t*>(&u);
    const uint16_t* ge = reinterpret_cast<const uint16_t*>(&g);
    uint32_t out[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float g0 = elem_f32(ge[2 * k]), g1 = elem_f32(ge[2 * k + 1]);
      const float h0 = g0 / (1.0f + expf(-g0)) * elem_f32(ue[2 * k]);
      const float h1 = g1 / (1.0f + expf(-g1)) * elem_f32(ue[2 * k + 1]);
      __nv_bfloat162 p = __floats2bfloat162_rn(h0, h1);
      out[k] = *reinterpret_cast<uint32_t*>(&p);
    }
    reinterpret_cast<uint4*>(h + b * I + j)[0] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

}  // namespace nm
