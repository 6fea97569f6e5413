// nm_peak.cuh -- tensor-core rate probe.
//
// Grounds the roofline denominators of the GEMMs: every SM pair issues a run
// of tcgen05 MMAs (cta_group::2, M = 256, N = 256) from operands that stay in
// shared memory, with no loads and no epilogue, so the launch time is the
// tensor pipe's own rate at the clocks of the moment.  The operand values are
// a fixed pattern; the accumulator is never read.
//   MODE 0: bf16 dense       (kind::f16,      K = 16 per MMA)
//   MODE 1: bf16 2:4 sparse  (kind::f16 .sp,  K = 32 per MMA)
//   MODE 2: E4M3 2:4 sparse  (kind::f8f6f4 .sp, K = 64 per MMA)
// Shared-memory layout per CTA, as in the 2-CTA GEMM's stages: A 128 rows x
// 128 B (128-byte swizzle), B two 128-byte-wide halves of 128 rows, metadata
// two 2048-byte blocks.
#pragma once
#include "nm_device.cuh"
#include "nm_gemm2.cuh"

namespace nm {

constexpr int kProbeN = 256;
constexpr int kProbeA = 128 * 128;                  // 16 KB
constexpr int kProbeB = 2 * (kProbeN / 2) * 128;    // 32 KB
constexpr int kProbeE = 2 * 2048;
constexpr int kProbeSmem = kProbeA + kProbeB + kProbeE + 1024 + 64;
// launched with more dynamic shared memory than two CTAs can share, so that
// each SM holds one CTA and its whole tensor memory
constexpr int kProbeSmemLaunch = 160 * 1024;

template <int MODE>
__global__ void __launch_bounds__(128, 1) k_mma_probe(int iters) {
  extern __shared__ uint8_t smem_probe_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_probe_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kProbeA;
  uint8_t* sE = sB + kProbeB;
  uint64_t* done_bar = reinterpret_cast<uint64_t*>(sE + kProbeE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  const int warp = threadIdx.x / 32;
  const bool leader = cluster_rank_2() == 0;

  // operand pattern: bf16 / E4M3 values near one; metadata nibbles 0x4 (entries 0 and 1)
  const uint32_t word = MODE == 2 ? 0x38383838u : 0x3F803F80u;
  for (int i = threadIdx.x; i < (kProbeA + kProbeB) / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(sA)[i] = word;
  for (int i = threadIdx.x; i < kProbeE / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(sE)[i] = 0x44444444u;
  if (threadIdx.x == 0) {
    mbar_init(done_bar, 1);
    fence_mbar_init();
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // generic stores -> tensor-core reads
  if (warp == 1) { tmem_alloc2(tmem_slot, 512); tmem_relinquish2(); }
  tc_fence_before();
  __syncthreads();
  cluster_barrier();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 1 && leader && elect_one()) {
    const uint32_t e_col = tmem + 256;
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    if constexpr (MODE == 1) {
      tc_cp_pair_128x128b(e_col, desc_plain_128x16(smem_u32(sE)));
    } else if constexpr (MODE == 2) {
      tc_cp_pair_128x128b(e_col, desc_plain_128x16(smem_u32(sE)));
      tc_cp_pair_128x128b(e_col + 4, desc_plain_128x16(smem_u32(sE + 2048)));
    }
    const uint32_t idesc = MODE == 2 ? idesc_e4m3(256, kProbeN, true) : idesc_bf16(256, kProbeN, MODE == 1);
#pragma unroll 1
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
        const uint64_t ad = desc_sw128_kmajor(a0 + 32u * kk);
        if constexpr (MODE == 0) {
          tc_mma_pair(tmem, ad, desc_sw128_kmajor(b0 + 32u * kk), idesc, acc);
        } else if constexpr (MODE == 1) {
          const uint64_t bd = desc_sw128_kmajor(b0 + (kk / 2) * (kProbeN / 2 * 128) + (kk % 2) * 64);
          tc_mma_sp_pair(tmem, ad, bd, e_col + (kk & ~1), idesc | static_cast<uint32_t>(kk & 1), acc);
        } else {
          const uint64_t bd = desc_sw128_kmajor(b0 + (kk / 2) * (kProbeN / 2 * 128) + (kk % 2) * 64);
          tc_mma_sp_pair_e4m3(tmem, ad, bd, e_col + 2u * kk, idesc, acc);
        }
      }
    }
    tc_commit_pair(done_bar);
  }
  // both CTAs: the leader's commit arrives on each CTA's barrier
  if (threadIdx.x == 0) mbar_wait(done_bar, 0u, nullptr, 0xFEA0u);
  __syncthreads();
  tc_fence_before();
  cluster_barrier();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem, 512);
  }
}

}  // namespace nm
