// nm_api.cu -- the C ABI declared in include/nmsparse.h.  Host-side
// validation, tensor-map encoding, tile/split selection and launches.  One
// translation unit: the kernels are included from the .cuh files so that the
// device status word is a single symbol.
#include <cudaTypedefs.h>

#include <algorithm>
#include <utility>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "nm_device.cuh"
#include "nm_gemm.cuh"
#include "nm_gemm2.cuh"
#include "nm_prune.cuh"
#include "nm_fp8.cuh"
#include "nm_mlp.cuh"
#include "nm_xf.cuh"
#include "nm_peak.cuh"
#include "nmsparse.h"

namespace {

thread_local int g_last_cuda_error = 0;
// Test hook (nm_debug_fail_next_launch): the next kernel launch on this
// thread returns this error instead of launching (0: none).
thread_local int g_fail_next_launch = 0;
// Name of the GEMM kernel instantiation most recently launched on this
// thread (nm_last_gemm_kernel).
thread_local char g_last_gemm[64] = "";

cudaError_t injected_launch_error() {
  const int c = g_fail_next_launch;
  g_fail_next_launch = 0;
  return static_cast<cudaError_t>(c);
}

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return NM_ERR_CUDA;
}

#define NM_CUDA_TRY(expr)                        \
  do {                                           \
    cudaError_t _e = (expr);                     \
    if (_e != cudaSuccess) return cuda_fail(_e); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
bool m_supported(int M) { return M == 4 || M == 8 || M == 16 || M == 32; }
int num_sms();

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2D bf16 tensor [outer][inner], row pitch row_bytes, box box_inner x
// box_outer, 128-byte swizzle, zero fill out of bounds.
int make_tmap(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t row_bytes,
              uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B,
              CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto fn = encode_fn();
  if (fn == nullptr) return cuda_fail(cudaErrorNotSupported);
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return NM_OK;
}

// Launch with programmatic stream serialisation: the kernel may start while
// the preceding kernel in the stream finishes; every kernel of this library
// waits (griddepcontrol.wait) before it touches memory the preceding kernel
// may own.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (g_fail_next_launch != 0) return injected_launch_error();
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// The same launch without programmatic serialisation: the kernel starts only
// after everything queued before it on the stream (kernels, copies, event
// waits) has completed.
template <typename... KArgs, typename... Args>
cudaError_t launch_plain(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                         Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = nullptr;
  cfg.numAttrs = 0;
  if (g_fail_next_launch != 0) return injected_launch_error();
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ----------------------------------------------------------------- GEMM
struct GemmPlan {
  const void* a_s = nullptr;  // compressed sparse A [rows_a][ks_lift/2]
  const void* a_d = nullptr;  // dense A [rows_a][kd]
  const void* b = nullptr;    // B [rows_b][ks_lift + kd]
  int64_t rows_a = 0, rows_b = 0, ks_lift = 0, kd = 0;
  const uint8_t* meta = nullptr;
  void* y = nullptr;
  int64_t ldy = 0;
  int out_fp32 = 0, transpose = 0;
  int a_static = 0;           // A is a weight: may be read before the preceding kernel ends
  int64_t out_split_rows = -1;  // output-split: A rows [0, this) sparse (a_s), the rest dense (a_d)
  const float* row_scale = nullptr;   // bf16 affine epilogue: y = acc * row_scale[a] + row_shift[a] * col_sum[b]
  const float* row_shift = nullptr;
  const float* col_sum = nullptr;
  int fp8 = 0;                // 8-bit (E4M3) operands, rescaled by scale_a[row] * scale_b[column]
  const float* scale_a = nullptr;
  const float* scale_b = nullptr;
  const void* lift_x = nullptr;  // in-GEMM lift: B = lift(lift_x), raw bf16 [rows_b][lift_k], row stride lift_ldx
  int64_t lift_ldx = 0, lift_k = 0;
  int lift_m = 0;
  void* ws = nullptr;            // optional scratch: the split last round's partial tiles (stream-K tail)
  size_t ws_bytes = 0;
};

// Scratch bound of the split last round on SM pairs: at most one 256 x 256
// fp32 partial tile per SM pair.
size_t sk_workspace_bound() { return static_cast<size_t>(std::max(1, num_sms() / 2)) * 256 * 256 * 4; }

// Ring depths of the in-GEMM lift kernel (compile-time instantiations), in
// order of preference: 6 stages of A (about half the k-range of the 6:8
// decode product, whose ring no longer has to hold B), else 4.
constexpr int kLiftRings[2] = {6, 4};

// Shared-memory plan of the in-GEMM lift for one launch shape: the largest
// raw-X box count and k-block count over the splits, and the layout
// [ring of A + metadata | receive buffer | barriers | raw X boxes | panel].
struct LiftSmem {
  int boxes = 0, kb = 0, ring = 0, raw_off = 0, panel_off = 0, bytes = 0;
};
constexpr int kMaxDynSmem = 232448;   // 227 KB per CTA on sm_100

template <int BN>
bool plan_lift_smem(int64_t kb_total, int splits, int64_t K, int M, LiftSmem* out) {
  using Cfg = nm::GemmCfg<BN, false>;
  const int L = 2 * (M - 2);                        // lifted columns per group: 4 (M/2 - 1)
  const int64_t k_lift = (K / M) * L;
  LiftSmem ls;
  for (int sp = 0; sp < splits; ++sp) {
    const int64_t b0 = kb_total * sp / splits, b1 = kb_total * (sp + 1) / splits;
    ls.kb = std::max<int>(ls.kb, static_cast<int>(b1 - b0));
    const int64_t j_lo = b0 * 128, j_hi = std::min<int64_t>(b1 * 128, k_lift);
    const int64_t c_base = ((j_lo / L) * M) & ~int64_t(7);
    const int64_t c_end = j_hi > j_lo ? ((j_hi - 1) / L + 1) * M : c_base;
    ls.boxes = std::max<int>(ls.boxes, static_cast<int>(ceil_div(c_end - c_base, int64_t(256))));
  }
  const int raw_bytes = ls.boxes * BN * 512, panel_bytes = ls.kb * Cfg::kBBytes;
  for (int r : kLiftRings) {
    const int fixed = r * (nm::kABytes + Cfg::kEStage) + Cfg::kRecvBytes + 256;
    ls.raw_off = static_cast<int>(ceil_div(int64_t(fixed), int64_t(1024)) * 1024);
    ls.panel_off = static_cast<int>(ceil_div(int64_t(ls.raw_off + raw_bytes), int64_t(1024)) * 1024);
    ls.bytes = 1024 + ls.panel_off + panel_bytes;
    ls.ring = r;
    if (ls.bytes <= kMaxDynSmem) { *out = ls; return true; }
  }
  return false;
}

template <int BN, bool FP8 = false>
int launch_gemm_bn(const GemmPlan& p, int splits, cudaStream_t st) {
  using Cfg = nm::GemmCfg<BN, FP8>;
  CUtensorMap ta_s, ta_d, tb;
  const int64_t kb_sparse = ceil_div(p.ks_lift, FP8 ? 256 : 128);
  const int64_t kb_dense = ceil_div(p.kd, 64);
  int rc;
  if (FP8) {
    // 8-bit codes: A stored [rows_a][K'/2] bytes, B lifted [rows_b][K'] bytes,
    // boxes of 128 bytes; sparse k-blocks only
    if ((rc = make_tmap(&ta_s, p.a_s, p.ks_lift / 2, p.rows_a, p.ks_lift / 2, 128, nm::kBM,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_DATA_TYPE_UINT8)) != NM_OK) return rc;
    if ((rc = make_tmap(&tb, p.b, p.ks_lift, p.rows_b, p.ks_lift, 128, BN, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_DATA_TYPE_UINT8)) != NM_OK) return rc;
    ta_d = ta_s;
  } else {
  // output-split: the sparse and the dense A are separate matrices over the
  // same B columns [0, K)
  const bool osplit = p.out_split_rows >= 0;
  const int64_t rows_s = osplit ? p.out_split_rows : p.rows_a;
  const int64_t rows_d = osplit ? p.rows_a - p.out_split_rows : p.rows_a;
  const int64_t b_cols = osplit ? p.ks_lift : p.ks_lift + p.kd;
  if (kb_sparse > 0 && rows_s > 0) {
    if ((rc = make_tmap(&ta_s, p.a_s, p.ks_lift / 2, rows_s, p.ks_lift, 64, nm::kBM)) != NM_OK) return rc;
  }
  if (kb_dense > 0 && rows_d > 0) {
    if ((rc = make_tmap(&ta_d, p.a_d, p.kd, rows_d, p.kd * 2, 64, nm::kBM)) != NM_OK) return rc;
  }
  if (kb_sparse == 0 || rows_s == 0) ta_s = ta_d;
  if (kb_dense == 0 || rows_d == 0) ta_d = ta_s;
  if (p.lift_x != nullptr) {
    // in-GEMM lift: tmB maps the raw activation, boxes of 256 columns x BN rows
    if ((rc = make_tmap(&tb, p.lift_x, p.lift_k, p.rows_b, p.lift_ldx * 2, 256, BN,
                        CU_TENSOR_MAP_SWIZZLE_NONE)) != NM_OK) return rc;
  } else if ((rc = make_tmap(&tb, p.b, b_cols, p.rows_b, b_cols * 2, 64, BN)) != NM_OK) {
    return rc;
  }
  }

  nm::GemmArgs args{};
  args.rows_a = p.rows_a;
  args.rows_b = p.rows_b;
  args.kb_sparse = static_cast<int>(kb_sparse);
  args.kb_dense = static_cast<int>(kb_dense);
  args.k_dense_x0 = p.ks_lift;
  args.meta = p.meta;
  args.meta_kb = FP8 ? ceil_div(p.ks_lift, 128) : kb_sparse;
  args.Y = p.y;
  args.ldy = p.ldy;
  args.out_fp32 = p.out_fp32;
  args.transpose_out = p.transpose;
  args.splits = splits;
  args.a_static = p.a_static;
  args.out_split_tiles = p.out_split_rows >= 0 ? static_cast<int>(p.out_split_rows / nm::kBM) : -1;
  args.row_scale = FP8 ? p.scale_a : p.row_scale;
  args.col_scale = FP8 ? p.scale_b : nullptr;
  args.row_shift = p.row_shift;
  args.col_sum = p.col_sum;
  args.fp8_last_half = (FP8 && p.ks_lift % 256 != 0) ? 1 : 0;
  int smem = Cfg::kSmemBytes;
  if (p.out_split_rows >= 0) args.k_dense_x0 = 0;
  // in-GEMM lift: its own instantiation (ring of 6 or 4 stages of A) and
  // parameter type
  nm::LiftArgs largs{};
  int lift_ring = 0;
  if (p.lift_x != nullptr) {
    if constexpr (FP8 || BN > 32) {
      return NM_ERR_UNSUPPORTED;
    } else {
      LiftSmem ls;
      if (!plan_lift_smem<BN>(kb_sparse, splits, p.lift_k, p.lift_m, &ls)) return NM_ERR_UNSUPPORTED;
      static_cast<nm::GemmArgs&>(largs) = args;
      largs.lift_m = p.lift_m;
      largs.lift_k = p.lift_k;
      largs.lift_boxes = ls.boxes;
      largs.lift_kb = ls.kb;
      largs.lift_raw_off = ls.raw_off;
      largs.lift_panel_off = ls.panel_off;
      lift_ring = ls.ring;
      smem = ls.bytes;
    }
  }

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(ceil_div(p.rows_a, nm::kBM)),
                     static_cast<unsigned>(ceil_div(p.rows_b, BN)), static_cast<unsigned>(splits));
  cfg.blockDim = dim3(192, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  // Programmatic dependent launch: the kernel may start while the preceding
  // kernel in the stream finishes; it waits for it (griddepcontrol.wait)
  // before touching anything but the static weight operand.
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (splits > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = static_cast<unsigned>(splits);
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  if (lift_ring > 0)
    std::snprintf(g_last_gemm, sizeof(g_last_gemm), "k_nm_gemm<%d,lift%d>", BN, lift_ring);
  else
    std::snprintf(g_last_gemm, sizeof(g_last_gemm), "k_nm_gemm<%d%s>", BN, FP8 ? ",fp8" : "");
  auto launch = [&](auto kern, const auto& a) -> int {
    NM_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    if (g_fail_next_launch != 0) NM_CUDA_TRY(injected_launch_error());
    NM_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, ta_s, ta_d, tb, a));
    NM_CUDA_TRY(cudaGetLastError());
    return NM_OK;
  };
  if constexpr (!FP8 && BN <= 32) {
    if (lift_ring == 6) return launch(nm::k_nm_gemm<BN, false, 6>, largs);
    if (lift_ring == 4) return launch(nm::k_nm_gemm<BN, false, 4>, largs);
  }
  return launch(nm::k_nm_gemm<BN, FP8>, args);
}

// uint8 [rows][16] view of a metadata image, box of one 128-row block.
// The metadata image as rows of 128 bytes: one 2048-byte block (the
// tensor-memory image of 128 operand rows) is a box of 16 such rows, fetched
// as 16 requests of 128 bytes.
int make_tmap_meta(CUtensorMap* m, const void* base, int64_t blocks) {
  auto fn = encode_fn();
  if (fn == nullptr) return cuda_fail(cudaErrorNotSupported);
  cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(blocks * 16)};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {128, 16};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return NM_OK;
}

// Number of 2-CTA clusters of this kernel that fit on the device at once.
template <int BN, int NACC, int MSUB, bool FP8 = false, bool LIFT = false>
int resident_pairs() {
  using Cfg = nm::Gemm2Cfg<BN, NACC, MSUB, FP8>;
  auto kern = nm::k_nm_gemm_2cta<BN, NACC, MSUB, FP8, LIFT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem) != cudaSuccess) {
    cudaGetLastError();
    return num_sms() / 2;
  }
  cudaLaunchConfig_t q{};
  q.gridDim = dim3(2, 1, 1);
  q.blockDim = dim3(LIFT ? nm::kLiftThreads2 : 192, 1, 1);
  q.dynamicSmemBytes = Cfg::kSmem;
  cudaLaunchAttribute qa[1];
  qa[0].id = cudaLaunchAttributeClusterDimension;
  qa[0].val.clusterDim.x = 2;
  qa[0].val.clusterDim.y = 1;
  qa[0].val.clusterDim.z = 1;
  q.attrs = qa;
  q.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &q) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = num_sms() / 2;
  }
  return n;
}

// Persistent 2-CTA kernel for pure-sparse products whose A side is a whole
// number of 256-row blocks.
template <int BN, int NACC, int MSUB, bool FP8 = false, bool LIFT = false>
int launch_gemm_2cta(const GemmPlan& p, cudaStream_t st) {
  using Cfg = nm::Gemm2Cfg<BN, NACC, MSUB, FP8>;
  if (LIFT != (p.lift_x != nullptr)) return NM_ERR_UNSUPPORTED;
  CUtensorMap ta, tb, te, ty, tad;
  int rc;
  // k-blocks: 128 lifted K (bf16) or 256 (8-bit, the last one possibly 128)
  const int64_t kb = ceil_div(p.ks_lift, FP8 ? 256 : 128);
  const int64_t kb_dense = ceil_div(p.kd, 64);
  // bf16 outputs leave through TMA stores of 32 x 32 staging tiles: Y[a][b]
  // row-major (64-byte swizzled tile), or Y[b][a] for the transposed product
  const bool y_ok = !p.out_fp32 && (p.ldy % 8) == 0 && (reinterpret_cast<uintptr_t>(p.y) & 15u) == 0;
  const int tma_store = !y_ok ? 0 : (p.transpose ? 2 : 1);
  if (tma_store == 1) {
    if ((rc = make_tmap(&ty, p.y, p.rows_b, p.rows_a, p.ldy * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B)) != NM_OK)
      return rc;
  } else if (tma_store == 2) {
    if ((rc = make_tmap(&ty, p.y, p.rows_a, p.rows_b, p.ldy * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE)) != NM_OK)
      return rc;
  }
  const int64_t meta_kb = ceil_div(p.ks_lift, 128);     // 128-K metadata blocks per 128 rows
  if (FP8) {
    if ((rc = make_tmap(&ta, p.a_s, p.ks_lift / 2, p.rows_a, p.ks_lift / 2, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_DATA_TYPE_UINT8)) != NM_OK) return rc;
    if ((rc = make_tmap_meta(&te, p.meta, ceil_div(p.rows_a, 128) * meta_kb)) != NM_OK) return rc;
    if ((rc = make_tmap(&tb, p.b, p.ks_lift, p.rows_b, p.ks_lift, 128, BN / 2, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_DATA_TYPE_UINT8)) != NM_OK) return rc;
    tad = ta;
  } else {
  // output-split: the 2:4 rows and the dense rows are separate matrices over
  // the same B columns [0, K)
  const bool osplit = p.out_split_rows >= 0;
  const int64_t rows_s = osplit ? p.out_split_rows : p.rows_a;
  const int64_t rows_d = osplit ? p.rows_a - p.out_split_rows : p.rows_a;
  const int64_t b_cols = osplit ? p.ks_lift : p.ks_lift + p.kd;
  const bool has_s = kb > 0 && rows_s > 0, has_d = kb_dense > 0 && rows_d > 0;
  if (has_s) {
    if ((rc = make_tmap(&ta, p.a_s, p.ks_lift / 2, rows_s, p.ks_lift, 64, 128)) != NM_OK) return rc;
    if ((rc = make_tmap_meta(&te, p.meta, ceil_div(rows_s, 128) * kb)) != NM_OK) return rc;
  }
  if (has_d) {
    if ((rc = make_tmap(&tad, p.a_d, p.kd, rows_d, p.kd * 2, 64, 128)) != NM_OK) return rc;
  }
  if (!has_s) { ta = tad; te = tad; }
  if (!has_d) tad = ta;
  if (LIFT) {
    tb = ta;                                         // B is written by the lift warps; any valid map
  } else if ((rc = make_tmap(&tb, p.b, b_cols, p.rows_b, b_cols * 2, 64, BN / 2)) != NM_OK) {
    return rc;
  }
  }
  nm::Gemm2Args a{};
  a.rows_a = p.rows_a;
  a.rows_b = p.rows_b;
  a.kb = static_cast<int>(kb);
  a.kb_dense = static_cast<int>(kb_dense);
  a.k_dense_x0 = p.ks_lift;
  a.meta_kb = meta_kb;
  a.scale_a = FP8 ? p.scale_a : p.row_scale;
  a.scale_b = p.scale_b;
  a.shift_a = p.row_shift;
  a.sum_b = p.col_sum;
  a.last_half = (FP8 && p.ks_lift % 256 != 0) ? 1 : 0;
  a.out_split_tiles = p.out_split_rows >= 0 ? static_cast<int>(p.out_split_rows / (256 * MSUB)) : -1;
  if (p.out_split_rows >= 0) a.k_dense_x0 = 0;
  a.tiles_m = static_cast<int>(ceil_div(p.rows_a, 256 * MSUB));
  a.tiles_n = static_cast<int>(ceil_div(p.rows_b, BN));
  a.Y = p.y;
  a.ldy = p.ldy;
  a.out_fp32 = p.out_fp32;
  a.transpose_out = p.transpose;
  a.tma_store = tma_store;
  if (!tma_store) ty = ta;                             // unused; any valid map
  const int tiles = a.tiles_m * a.tiles_n;
  auto kern = nm::k_nm_gemm_2cta<BN, NACC, MSUB, FP8, LIFT>;
  NM_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem));
  cudaLaunchConfig_t cfg{};
  // A persistent grid larger than the number of co-resident SM pairs would
  // run its last clusters after the others: size it by the occupancy query.
  static int resident = 0;
  if (resident == 0) resident = resident_pairs<BN, NACC, MSUB, FP8, LIFT>();
  const int clusters = std::max(1, std::min(tiles, resident));
  // Split last round (stream-K tail): when the tiles leave a last persistent
  // round in which fewer than half the SM pairs would work, and the caller
  // gave scratch, each of that round's L tiles is split along K into
  // clusters / L parts, run by otherwise idle pairs; k_sk_fixup adds the
  // parts in order.  A part keeps at least 16 k-blocks: the partial tiles
  // cost a write and a read of 256 x BN fp32 each, which a shorter part does
  // not pay back (measured on B200: 6:8 prefill, 48 k-blocks in 9 parts,
  // 10 us of fixup for 3 us saved), and the parts' units must fit the
  // scratch.  Plain bf16/fp32 outputs of pure 2:4 products only (no dense
  // k-blocks, output split or epilogue scaling); 256- and 512-row tiles.
  a.sk_full = tiles;
  a.sk_parts = 0;
  a.sk_ws = nullptr;
  if (p.ws != nullptr && aligned16(p.ws) && !FP8 && p.out_split_rows < 0 && p.kd == 0 &&
      p.row_scale == nullptr && p.row_shift == nullptr) {
    const int R = tiles / clusters, L = tiles - R * clusters;
    // a last round made only of the last, partial column of tiles is short
    // already (its tiles carry fewer rows of B): no split
    const bool tail_partial = (p.rows_b % BN) != 0 && (tiles - L) / a.tiles_m == a.tiles_n - 1;
    if (R >= 1 && L > 0 && !tail_partial) {
      // parts also limited by the scratch: L x parts units of 256 MSUB x BN fp32
      const size_t unit_bytes = static_cast<size_t>(256) * MSUB * BN * 4;
      const int64_t fit = static_cast<int64_t>(p.ws_bytes / (unit_bytes * static_cast<size_t>(L)));
      const int parts = static_cast<int>(std::min<int64_t>(std::min<int64_t>(clusters / L, kb / 16), fit));
      const size_t need = static_cast<size_t>(L) * parts * unit_bytes;
      if (parts >= 2 && p.ws_bytes >= need) {
        a.sk_full = R * clusters;
        a.sk_parts = parts;
        a.sk_ws = static_cast<float*>(p.ws);
      }
    }
  }
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
  cfg.blockDim = dim3(LIFT ? nm::kLiftThreads2 : 192, 1, 1);
  cfg.dynamicSmemBytes = Cfg::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  std::snprintf(g_last_gemm, sizeof(g_last_gemm), "k_nm_gemm_2cta<%d,%d,%d%s>", BN, NACC, MSUB,
                FP8 ? ",fp8" : (LIFT ? ",lift" : ""));
  if (g_fail_next_launch != 0) NM_CUDA_TRY(injected_launch_error());
  if constexpr (LIFT) {
    nm::Gemm2LiftArgs la{};
    static_cast<nm::Gemm2Args&>(la) = a;
    la.lift_x = static_cast<const uint16_t*>(p.lift_x);
    la.lift_ldx = p.lift_ldx;
    la.lift_k = p.lift_k;
    la.lift_m = p.lift_m;
    NM_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, ta, tb, te, ty, tad, la));
  } else {
    NM_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, ta, tb, te, ty, tad, a));
  }
  NM_CUDA_TRY(cudaGetLastError());
  if (a.sk_parts > 1) {
    const size_t n = std::strlen(g_last_gemm);
    std::snprintf(g_last_gemm + n, sizeof(g_last_gemm) - n, "+split%d", a.sk_parts);
    const int tail = tiles - a.sk_full;
    const int64_t total = static_cast<int64_t>(tail) * 64 * MSUB * BN;     // 4-output quads
    const int64_t blocks = std::min<int64_t>(ceil_div(total, int64_t(256)), int64_t(num_sms()) * 8);
    NM_CUDA_TRY(launch_pdl(nm::k_sk_fixup, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st,
                           static_cast<const float*>(a.sk_ws), a.sk_full, a.sk_parts, tail, a.tiles_m, 256 * MSUB,
                           BN, p.rows_a, p.rows_b, p.y, p.ldy, p.out_fp32, p.transpose));
    NM_CUDA_TRY(cudaGetLastError());
  }
  return NM_OK;
}
int pick_bn(int64_t rows_b) {
  if (rows_b <= 16) return 16;
  if (rows_b <= 32) return 32;
  if (rows_b <= 64) return 64;
  return 128;
}

int num_sms() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      sms = 148;
  }
  return sms;
}

// Split-K only when the output tiles cannot cover the SMs; powers of two up to
// 8 (the cluster holds the splits of one tile).
int pick_splits(int64_t tiles, int64_t kb_total) {
  int s = 1;
  while (s < 8 && tiles * (s * 2) <= num_sms() && kb_total >= (s * 2) * 4) s *= 2;
  return s;
}

// Kernel choice.  NMSPARSE_GEMM pins one variant where it applies:
// "1cta", "2cta224", "2cta192", "2cta256", "2cta128", "2cta224x2", "2cta192x2",
// "2cta160x2", "2cta128x2";
// unset or "auto" picks by shape.
int run_gemm(const GemmPlan& p, cudaStream_t st) {
  const char* env = std::getenv("NMSPARSE_GEMM");
  const std::string mode = env != nullptr ? env : "auto";
  // an output-split product needs whole 256-row tiles on both sides of the split
  const bool osplit = p.out_split_rows >= 0;
  const bool eligible2 = (!osplit || p.out_split_rows % 256 == 0) && (p.ks_lift + p.kd) > 0 &&
                         p.rows_a % 256 == 0 && (p.kd == 0 || p.ks_lift % 128 == 0);
  const bool eligible4 = eligible2 && !osplit && p.rows_a % 512 == 0;
  // SM pairs the 2-CTA kernel would occupy with 128-wide tiles
  const int64_t pairs128 = (p.rows_a / 256) * ceil_div(p.rows_b, int64_t(128));
  if (eligible2 && mode != "1cta") {
    if (mode == "2cta224") return launch_gemm_2cta<224, 2, 1>(p, st);
    if (mode == "2cta192") return launch_gemm_2cta<192, 2, 1>(p, st);
    if (mode == "2cta256") return launch_gemm_2cta<256, 1, 1>(p, st);
    if (mode == "2cta128") return launch_gemm_2cta<128, 2, 1>(p, st);
    if (eligible4 && mode == "2cta224x2") return launch_gemm_2cta<224, 1, 2>(p, st);
    if (eligible4 && mode == "2cta192x2") return launch_gemm_2cta<192, 1, 2>(p, st);
    if (eligible4 && mode == "2cta160x2") return launch_gemm_2cta<160, 1, 2>(p, st);
    if (eligible4 && mode == "2cta128x2") return launch_gemm_2cta<128, 1, 2>(p, st);
    // products with dense k-blocks (hybrid, output-split, dense comparator)
    // on SM pairs; a narrow product with too few tiles to occupy half of the
    // SMs runs on single CTAs with split-K instead
    if (p.kd > 0 && p.rows_b >= 512) return launch_gemm_2cta<224, 2, 1>(p, st);
    if (p.kd > 0 && p.rows_b >= 64 && 4 * pairs128 >= num_sms()) return launch_gemm_2cta<128, 2, 1>(p, st);
    if (p.rows_b >= 512 && p.ks_lift >= 512) {
      // Both 2:4 operands stream through shared memory, whose port bounds this
      // kernel well before the tensor pipe does; measured on B200, the 224-wide
      // tile with two accumulators (epilogue overlapped) is best except for
      // long reductions on narrow outputs, where the 256-wide tile's fewer
      // rounds outweigh its exposed epilogue.
      if (p.rows_b <= 8192 && p.ks_lift >= 16384) return launch_gemm_2cta<256, 1, 1>(p, st);
      return launch_gemm_2cta<224, 2, 1>(p, st);
    }
  }
  const int bn = pick_bn(p.rows_b);
  const int64_t tiles = ceil_div(p.rows_a, nm::kBM) * ceil_div(p.rows_b, bn);
  const int64_t kb_total = ceil_div(p.ks_lift, 128) + ceil_div(p.kd, 64);
  const int splits = pick_splits(tiles, kb_total);
  switch (bn) {
    case 16: return launch_gemm_bn<16>(p, splits, st);
    case 32: return launch_gemm_bn<32>(p, splits, st);
    case 64: return launch_gemm_bn<64>(p, splits, st);
    default: return launch_gemm_bn<128>(p, splits, st);
  }
}

// --------------------------------------------------------------- prune
// early = false launches without programmatic serialisation (the prune then
// waits for copies and event waits queued before it, not only for kernels).
template <typename T, bool Q8 = false, bool XF = false, bool SPLIT = false>
int launch_prune(const T* src, int64_t rows, int64_t K, int64_t ld, int N, int M, uint32_t* mask,
                 void* vals, void* meta, cudaStream_t st, const float* row_scale = nullptr,
                 const float* row_shift = nullptr, double* stats = nullptr, bool early = true) {
  const int64_t Kl = nm_lifted_k(K, M);
  const int64_t KB = ceil_div(Kl, 128);
  const int64_t rows_pad = ceil_div(rows, 128) * 128;
  const int64_t cpr = ceil_div(K / M, 32 * nm::prune_groups_per_lane(M, sizeof(T)));
  const int64_t tasks = (rows_pad / 16) * cpr;
  if (tasks >= (int64_t(1) << 31)) return NM_ERR_UNSUPPORTED;
  // persistent grid: the resident CTAs of every SM take the tasks in turn
  const int64_t per_sm = nm::prune_min_blocks(M, sizeof(T));
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(tasks, int64_t(num_sms()) * per_sm));
  const dim3 grid(static_cast<unsigned>(blocks)), block(nm::kPruneWarps * 32);
  nm::PruneGrid pg{static_cast<uint32_t>(cpr), static_cast<uint32_t>(tasks)};
  auto v = static_cast<uint32_t*>(vals);
  auto e = static_cast<uint8_t*>(meta);
  auto go = [&](auto kern) {
    return early ? launch_pdl(kern, grid, block, 0, st, src, rows, K, ld, N, mask, v, e, Kl, KB, pg, row_scale,
                              row_shift, stats)
                 : launch_plain(kern, grid, block, 0, st, src, rows, K, ld, N, mask, v, e, Kl, KB, pg, row_scale,
                                row_shift, stats);
  };
  cudaError_t err;
  if constexpr (SPLIT) {
    switch (M) {
      case 8: err = go(nm::k_prune_compress<8, T, false, false, true>); break;
      case 16: err = go(nm::k_prune_compress<16, T, false, false, true>); break;
      case 32: err = go(nm::k_prune_compress<32, T, false, false, true>); break;
      default: return NM_ERR_UNSUPPORTED;
    }
  } else {
    switch (M) {
      case 4: err = go(nm::k_prune_compress<4, T, Q8, XF>); break;
      case 8: err = go(nm::k_prune_compress<8, T, Q8, XF>); break;
      case 16: err = go(nm::k_prune_compress<16, T, Q8, XF>); break;
      case 32: err = go(nm::k_prune_compress<32, T, Q8, XF>); break;
      default: return NM_ERR_UNSUPPORTED;
    }
  }
  NM_CUDA_TRY(err);
  NM_CUDA_TRY(cudaGetLastError());
  return NM_OK;
}

template <typename T>
int launch_lift(const T* src, int64_t rows, int64_t K, int64_t ld, int M, void* dst, cudaStream_t st) {
  const int64_t Kl = nm_lifted_k(K, M);
  // one CTA per (block of nm::kLiftRows rows, segment of nm::kLiftElems input
  // elements); row blocks beyond the grid's y extent are taken in a loop
  const int64_t segs = ceil_div(K, int64_t(nm::kLiftElems));
  const int64_t rblocks = ceil_div(rows, int64_t(nm::kLiftRows));
  auto d = static_cast<uint16_t*>(dst);
  const dim3 grid(static_cast<unsigned>(segs), static_cast<unsigned>(std::min<int64_t>(rblocks, 65535))), block(256);
  cudaError_t err;
  switch (M) {
    case 4: err = launch_pdl(nm::k_lift<4, T>, grid, block, 0, st, src, rows, K, ld, d, Kl); break;
    case 8: err = launch_pdl(nm::k_lift<8, T>, grid, block, 0, st, src, rows, K, ld, d, Kl); break;
    case 16: err = launch_pdl(nm::k_lift<16, T>, grid, block, 0, st, src, rows, K, ld, d, Kl); break;
    case 32: err = launch_pdl(nm::k_lift<32, T>, grid, block, 0, st, src, rows, K, ld, d, Kl); break;
    default: return NM_ERR_UNSUPPORTED;
  }
  NM_CUDA_TRY(err);
  NM_CUDA_TRY(cudaGetLastError());
  return NM_OK;
}

int launch_lift_odd(uint16_t* x, int64_t rows, int64_t K, int64_t ld, int M, cudaStream_t st) {
  const int64_t total = rows * (K / M / 2);
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(ceil_div(total, int64_t(256)), int64_t(num_sms()) * 16));
  const dim3 grid(static_cast<unsigned>(blocks)), block(256);
  cudaError_t err;
  switch (M) {
    case 8: err = launch_pdl(nm::k_lift_odd<8>, grid, block, 0, st, x, rows, K, ld); break;
    case 16: err = launch_pdl(nm::k_lift_odd<16>, grid, block, 0, st, x, rows, K, ld); break;
    case 32: err = launch_pdl(nm::k_lift_odd<32>, grid, block, 0, st, x, rows, K, ld); break;
    default: return NM_ERR_UNSUPPORTED;
  }
  NM_CUDA_TRY(err);
  NM_CUDA_TRY(cudaGetLastError());
  return NM_OK;
}

int check_prune_args(const void* src, nm_dtype dt, int64_t rows, int64_t K, int64_t ld, int N, int M,
                     const void* vals, const void* meta) {
  if (dt != NM_BF16 && dt != NM_FP32) return NM_ERR_INVALID_ARG;
  if (rows < 0 || K <= 0 || M <= 0 || ld < K || N < 0 || N > M) return NM_ERR_INVALID_ARG;
  if (K % M != 0) return NM_ERR_INVALID_ARG;
  if (!m_supported(M)) return NM_ERR_UNSUPPORTED;
  if (N > (M == 4 ? 2 : M - 2)) return NM_ERR_UNSUPPORTED;
  if (rows == 0) return NM_OK;                 // empty operand: nothing to read or write
  if (src == nullptr || vals == nullptr || meta == nullptr) return NM_ERR_INVALID_ARG;
  const int64_t esz = dt == NM_BF16 ? 2 : 4;
  if (!aligned16(src) || !aligned16(vals) || !aligned16(meta) || (ld * esz) % 16 != 0) return NM_ERR_ALIGNMENT;
  return NM_OK;
}

}  // namespace

extern "C" {

int64_t nm_lifted_k(int64_t K, int M) {
  if (M < 4 || M % 2 != 0 || K <= 0 || K % M != 0) return -1;
  return K / M * 4 * (M / 2 - 1);
}

size_t nm_meta_bytes(int64_t rows, int64_t K, int M) {
  const int64_t Kl = nm_lifted_k(K, M);
  if (Kl < 0 || rows < 0) return 0;
  return static_cast<size_t>(ceil_div(rows, 128) * ceil_div(Kl, 128) * 2048);
}

int nm_prune_compress(const void* src, nm_dtype dt, int64_t rows, int64_t K, int64_t ld, int N, int M,
                      uint32_t* mask_out, void* vals_out, void* meta_out, void* stream) {
  int rc = check_prune_args(src, dt, rows, K, ld, N, M, vals_out, meta_out);
  if (rc != NM_OK) return rc;
  if (mask_out != nullptr && !aligned16(mask_out)) return NM_ERR_ALIGNMENT;
  if (rows == 0) return NM_OK;
  auto st = static_cast<cudaStream_t>(stream);
  if (dt == NM_BF16)
    return launch_prune(static_cast<const uint16_t*>(src), rows, K, ld, N, M, mask_out, vals_out, meta_out, st);
  return launch_prune(static_cast<const uint32_t*>(src), rows, K, ld, N, M, mask_out, vals_out, meta_out, st);
}

int slide_decompose(const void* w, nm_dtype dt, int64_t rows, int64_t K, int N, int M, uint32_t* mask_out,
                    void* vals_out, void* meta_out, void* stream) {
  if (!(N == M - 2 || (M == 4 && N == 2))) return NM_ERR_UNSUPPORTED;
  return nm_prune_compress(w, dt, rows, K, K, N, M, mask_out, vals_out, meta_out, stream);
}

int slide_decompose_split(const void* w, int64_t rows, int64_t K, int N, int M, uint32_t* mask_out, void* vals_out,
                          void* meta_out, void* stream) {
  int rc = check_prune_args(w, NM_BF16, rows, K, K, N, M, vals_out, meta_out);
  if (rc != NM_OK) return rc;
  if (N != M - 2 || M < 8 || M % 4 != 0 || K % 128 != 0) return NM_ERR_UNSUPPORTED;
  if (mask_out != nullptr && !aligned16(mask_out)) return NM_ERR_ALIGNMENT;
  if (rows == 0) return NM_OK;
  return launch_prune<uint16_t, false, false, true>(static_cast<const uint16_t*>(w), rows, K, K, N, M, mask_out,
                                                     vals_out, meta_out, static_cast<cudaStream_t>(stream));
}

int nm_lift_odd(void* x, int64_t rows, int64_t K, int64_t ld, int M, void* stream) {
  if (rows < 0 || K <= 0 || M <= 0 || K % M != 0) return NM_ERR_INVALID_ARG;
  if (M < 8 || M % 4 != 0 || !m_supported(M) || K % 128 != 0) return NM_ERR_UNSUPPORTED;
  if (ld < nm_lifted_k(K, M)) return NM_ERR_INVALID_ARG;
  if (rows == 0) return NM_OK;
  if (x == nullptr) return NM_ERR_INVALID_ARG;
  if (!aligned16(x) || (ld * 2) % 16 != 0) return NM_ERR_ALIGNMENT;
  return launch_lift_odd(static_cast<uint16_t*>(x), rows, K, ld, M, static_cast<cudaStream_t>(stream));
}

int nm_lift(const void* src, nm_dtype dt, int64_t rows, int64_t K, int64_t ld, int M, void* dst, void* stream) {
  if (dt != NM_BF16 && dt != NM_FP32) return NM_ERR_INVALID_ARG;
  if (rows < 0 || K <= 0 || M <= 0 || ld < K || K % M != 0) return NM_ERR_INVALID_ARG;
  if (!m_supported(M)) return NM_ERR_UNSUPPORTED;
  if (rows == 0) return NM_OK;
  if (src == nullptr || dst == nullptr) return NM_ERR_INVALID_ARG;
  const int64_t esz = dt == NM_BF16 ? 2 : 4;
  if (!aligned16(src) || !aligned16(dst) || (ld * esz) % 16 != 0 || (nm_lifted_k(K, M) % 8) != 0)
    return NM_ERR_ALIGNMENT;
  if (rows == 0) return NM_OK;
  auto st = static_cast<cudaStream_t>(stream);
  if (dt == NM_BF16) return launch_lift(static_cast<const uint16_t*>(src), rows, K, ld, M, dst, st);
  return launch_lift(static_cast<const uint32_t*>(src), rows, K, ld, M, dst, st);
}

size_t nm_sparse_gemm_workspace_size(const nm_sparse_operand* S, int64_t rows_d, nm_side side) {
  (void)side;
  // products on SM pairs (whole 256-row tiles of the sparse operand, at
  // least 512 rows of the dense one) may split their last round; the split-K
  // of the single-CTA kernel keeps its partial sums in the cluster's shared
  // memory
  if (S == nullptr || S->rows <= 0 || S->rows % 256 != 0 || rows_d < 512) return 0;
  return sk_workspace_bound();
}

}  // extern "C"

namespace {

// Validates a sparse x lifted-dense product and fills its plan; NM_OK with
// *empty set when there is nothing to compute.
int sparse_plan(const nm_sparse_operand* S, const void* D, int64_t rows_d, nm_side side, void* Y,
                nm_dtype out_dt, GemmPlan* plan, bool* empty) {
  *empty = false;
  if (S == nullptr) return NM_ERR_INVALID_ARG;
  if (side != NM_ACT && side != NM_WEIGHT) return NM_ERR_INVALID_ARG;
  if (out_dt != NM_BF16 && out_dt != NM_FP32) return NM_ERR_INVALID_ARG;
  if (S->rows < 0 || rows_d < 0 || S->K <= 0 || S->M <= 0 || S->K % S->M != 0) return NM_ERR_INVALID_ARG;
  if (!m_supported(S->M)) return NM_ERR_UNSUPPORTED;
  if (S->K_lift != nm_lifted_k(S->K, S->M)) return NM_ERR_INVALID_ARG;
  if (S->K_lift % 16 != 0) return NM_ERR_UNSUPPORTED;
  if (S->rows == 0 || rows_d == 0) { *empty = true; return NM_OK; }
  if (D == nullptr || Y == nullptr || S->vals == nullptr || S->meta == nullptr) return NM_ERR_INVALID_ARG;
  if (!aligned16(S->vals) || !aligned16(S->meta) || !aligned16(D) || !aligned16(Y)) return NM_ERR_ALIGNMENT;
  GemmPlan& p = *plan;
  p.a_s = S->vals;
  p.b = D;
  p.rows_a = S->rows;
  p.rows_b = rows_d;
  p.ks_lift = S->K_lift;
  p.kd = 0;
  p.meta = static_cast<const uint8_t*>(S->meta);
  p.y = Y;
  p.out_fp32 = out_dt == NM_FP32;
  p.transpose = side == NM_WEIGHT;
  p.ldy = side == NM_ACT ? rows_d : S->rows;
  p.a_static = side == NM_WEIGHT;
  return NM_OK;
}

int64_t prune_chunks(int64_t K, int M) { return ceil_div(K / M, 32 * nm::prune_groups_per_lane(M, 2)); }

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// In-GEMM lift (slide_gemm): the single-CTA kernel's tile width and split
// for rows_x activation rows, and whether the lifted panel fits its shared
// memory.
template <int BN>
bool slide_fused_fits(const nm_sparse_operand* W, int splits) {
  const int64_t kb_total = ceil_div(W->K_lift, int64_t(128));
  LiftSmem ls;
  return plan_lift_smem<BN>(kb_total, splits, W->K, W->M, &ls);
}

// In-GEMM lift on SM pairs (prefill shapes): the weight in whole 256-row
// tiles, at least 64 activation rows, and the 32-bit window arithmetic of the
// lift warps.  Returns the tile width (0: not this path).
int slide_pair_bn(const nm_sparse_operand* W, int64_t rows_x) {
  if (W->rows % 256 != 0 || rows_x < 64 || W->K_lift / 4 >= (int64_t(1) << 31)) return 0;
  if (rows_x < 512) return 128;
  if (rows_x <= 8192 && W->K_lift >= 16384) return 256;
  return 224;
}

bool slide_fused_plan(const nm_sparse_operand* W, int64_t rows_x, int* bn, int* splits) {
  if (rows_x > 32 || W->K_lift >= (int64_t(1) << 24)) return false;   // the kernel's 32-bit window math
  *bn = pick_bn(rows_x);
  *splits = pick_splits(ceil_div(W->rows, int64_t(nm::kBM)), ceil_div(W->K_lift, int64_t(128)));
  return *bn == 16 ? slide_fused_fits<16>(W, *splits) : slide_fused_fits<32>(W, *splits);
}


}  // namespace

extern "C" {

int nm_sparse_gemm(const nm_sparse_operand* S, const void* D, int64_t rows_d, nm_side side, void* Y,
                   nm_dtype out_dt, void* ws, size_t ws_bytes, void* stream) {
  GemmPlan p;
  bool empty = false;
  const int rc = sparse_plan(S, D, rows_d, side, Y, out_dt, &p, &empty);
  if (rc != NM_OK || empty) return rc;
  p.ws = ws;
  p.ws_bytes = ws != nullptr ? ws_bytes : 0;
  return run_gemm(p, static_cast<cudaStream_t>(stream));
}

size_t slide_gemm_workspace_size(const nm_sparse_operand* W, int64_t rows_x) {
  if (W == nullptr || rows_x <= 0 || W->rows <= 0 || W->K <= 0 || W->M <= 0 || !m_supported(W->M) ||
      W->K % W->M != 0 || W->K_lift != nm_lifted_k(W->K, W->M))
    return 0;
  int bn = 0, splits = 0;
  if (slide_fused_plan(W, rows_x, &bn, &splits)) return 0;
  // SM pairs: optional scratch for a split last round (the lift needs none)
  if (slide_pair_bn(W, rows_x) != 0) return rows_x >= 512 ? sk_workspace_bound() : 0;
  return static_cast<size_t>(ceil_div(rows_x * W->K_lift * 2, int64_t(16)) * 16);
}

int slide_gemm(const nm_sparse_operand* W, const void* X, int64_t rows_x, int64_t ldx, void* Y, nm_dtype out_dt,
               void* ws, size_t ws_bytes, void* stream) {
  if (W == nullptr || rows_x < 0 || ldx < W->K) return NM_ERR_INVALID_ARG;
  GemmPlan p;
  bool empty = false;
  int rc = sparse_plan(W, X, rows_x, NM_WEIGHT, Y, out_dt, &p, &empty);
  if (rc != NM_OK || empty) return rc;
  if ((ldx * 2) % 16 != 0) return NM_ERR_ALIGNMENT;
  auto st = static_cast<cudaStream_t>(stream);
  int bn = 0, splits = 0;
  if (slide_fused_plan(W, rows_x, &bn, &splits)) {
    p.b = nullptr;
    p.lift_x = X;
    p.lift_ldx = ldx;
    p.lift_k = W->K;
    p.lift_m = W->M;
    return bn == 16 ? launch_gemm_bn<16>(p, splits, st) : launch_gemm_bn<32>(p, splits, st);
  }
  if ((bn = slide_pair_bn(W, rows_x)) != 0) {
    // prefill shapes: the lift warps of the SM-pair kernel write B from X
    if (ldx % 2 != 0) return NM_ERR_ALIGNMENT;
    p.ws = ws;
    p.ws_bytes = ws != nullptr ? ws_bytes : 0;
    p.b = nullptr;
    p.lift_x = X;
    p.lift_ldx = ldx;
    p.lift_k = W->K;
    p.lift_m = W->M;
    if (bn == 128) return launch_gemm_2cta<128, 2, 1, false, true>(p, st);
    if (bn == 256) return launch_gemm_2cta<256, 1, 1, false, true>(p, st);
    return launch_gemm_2cta<224, 2, 1, false, true>(p, st);
  }
  // lift into the workspace, then the plain product
  if (ws == nullptr || ws_bytes < slide_gemm_workspace_size(W, rows_x)) return NM_ERR_WORKSPACE;
  if (!aligned16(ws)) return NM_ERR_ALIGNMENT;
  if ((rc = nm_lift(X, NM_BF16, rows_x, W->K, ldx, W->M, ws, stream)) != NM_OK) return rc;
  p.b = ws;
  return run_gemm(p, st);
}

// ------------------------------------------------ per-token corrections

// VAR scratch: the token moments (rows x 2 fp64, padded to 256 bytes), then
// the kept sums of every (row, chunk) (rows x chunks x 2 fp64).
int64_t xf_moments_bytes(int64_t rows) { return ceil_div(rows * 16, int64_t(256)) * 256; }

size_t nm_prune_compress_xf_workspace_size(int64_t rows, int64_t K, int M) {
  if (rows <= 0 || K <= 0 || !m_supported(M) || K % M != 0) return 0;
  return static_cast<size_t>(xf_moments_bytes(rows) + rows * prune_chunks(K, M) * 16);
}

int nm_prune_compress_xf(const void* src, int64_t rows, int64_t K, int64_t ld, int N, int M, unsigned flags,
                         uint32_t* mask_out, void* vals_out, void* meta_out, float* row_scale_out,
                         float* row_shift_out, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_prune_args(src, NM_BF16, rows, K, ld, N, M, vals_out, meta_out);
  if (rc != NM_OK) return rc;
  if ((flags & ~(NM_XF_SHIFT | NM_XF_VAR)) != 0u) return NM_ERR_INVALID_ARG;
  if (rows == 0) return NM_OK;
  if (row_scale_out == nullptr || row_shift_out == nullptr) return NM_ERR_INVALID_ARG;
  if ((mask_out != nullptr && !aligned16(mask_out)) || !aligned4(row_scale_out) || !aligned4(row_shift_out))
    return NM_ERR_ALIGNMENT;
  const bool shift = (flags & NM_XF_SHIFT) != 0u, var = (flags & NM_XF_VAR) != 0u;
  if (var) {
    if (ws == nullptr || ws_bytes < nm_prune_compress_xf_workspace_size(rows, K, M)) return NM_ERR_WORKSPACE;
    if (!aligned16(ws)) return NM_ERR_ALIGNMENT;
  }
  auto st = static_cast<cudaStream_t>(stream);
  const auto* x = static_cast<const uint16_t*>(src);
  double* moments = var ? static_cast<double*>(ws) : nullptr;
  double* kept = var ? reinterpret_cast<double*>(static_cast<uint8_t*>(ws) + xf_moments_bytes(rows)) : nullptr;
  const dim3 wgrid(static_cast<unsigned>(std::min<int64_t>(ceil_div(rows, int64_t(8)), int64_t(1) << 30))),
      block(256);
  if (shift || var)   // token mean and / or moments, one warp per row
    NM_CUDA_TRY(launch_pdl(nm::k_row_prep_bf16, wgrid, block, 0, st, x, rows, K, ld, shift ? 1 : 0, row_shift_out,
                           moments));
  if ((rc = launch_prune<uint16_t, false, true>(x, rows, K, ld, N, M, mask_out, vals_out, meta_out, st, nullptr,
                                                shift ? row_shift_out : nullptr, kept)) != NM_OK)
    return rc;
  NM_CUDA_TRY(launch_pdl(nm::k_xf_finalize, wgrid, block, 0, st, static_cast<const double*>(moments),
                         static_cast<const double*>(kept), rows, prune_chunks(K, M), K, shift ? 0 : 1, row_scale_out,
                         row_shift_out));
  return NM_OK;
}

int nm_row_sums(const void* w, int64_t rows, int64_t K, int64_t ld, float* sums_out, void* stream) {
  if (rows < 0 || K <= 0 || ld < K) return NM_ERR_INVALID_ARG;
  if (rows == 0) return NM_OK;
  if (w == nullptr || sums_out == nullptr) return NM_ERR_INVALID_ARG;
  if (!aligned16(w) || (ld * 2) % 16 != 0 || !aligned4(sums_out)) return NM_ERR_ALIGNMENT;
  const dim3 grid(static_cast<unsigned>(std::min<int64_t>(ceil_div(rows, int64_t(8)), int64_t(1) << 30))), block(256);
  NM_CUDA_TRY(launch_pdl(nm::k_row_sum_bf16, grid, block, 0, static_cast<cudaStream_t>(stream),
                         static_cast<const uint16_t*>(w), rows, K, ld, sums_out));
  return NM_OK;
}

int nm_sparse_gemm_xf(const nm_sparse_operand* X, const void* W_lift, int64_t rows_w, const float* row_scale,
                      const float* row_shift, const float* w_row_sums, void* Y, nm_dtype out_dt, void* stream) {
  GemmPlan p;
  bool empty = false;
  const int rc = sparse_plan(X, W_lift, rows_w, NM_ACT, Y, out_dt, &p, &empty);
  if (rc != NM_OK || empty) return rc;
  if (row_scale == nullptr || row_shift == nullptr || w_row_sums == nullptr) return NM_ERR_INVALID_ARG;
  if (!aligned4(row_scale) || !aligned4(row_shift) || !aligned4(w_row_sums)) return NM_ERR_ALIGNMENT;
  p.row_scale = row_scale;
  p.row_shift = row_shift;
  p.col_sum = w_row_sums;
  return run_gemm(p, static_cast<cudaStream_t>(stream));
}


// ------------------------------------------------------------ 8-bit (E4M3)

int nm_quant_lift_fp8(const void* src, nm_dtype dt, int64_t rows, int64_t K, int64_t ld, int M,
                      uint8_t* codes_out, float* scale_out, void* stream) {
  if (dt != NM_BF16 && dt != NM_FP32) return NM_ERR_INVALID_ARG;
  if (rows < 0 || K <= 0 || M <= 0 || ld < K || K % M != 0) return NM_ERR_INVALID_ARG;
  if (!m_supported(M)) return NM_ERR_UNSUPPORTED;
  const int64_t esz = dt == NM_BF16 ? 2 : 4;
  const int64_t Kl = nm_lifted_k(K, M);
  if (Kl % 16 != 0) return NM_ERR_UNSUPPORTED;
  if (rows == 0) return NM_OK;
  if (src == nullptr || codes_out == nullptr || scale_out == nullptr) return NM_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(codes_out) || (ld * esz) % 16 != 0 ||
      (reinterpret_cast<uintptr_t>(scale_out) & 3u) != 0)
    return NM_ERR_ALIGNMENT;
  auto st = static_cast<cudaStream_t>(stream);
  // one warp per row; CTAs of up to eight warps, fewer when there are few
  // rows (so that they spread over the SMs); a grid of at most eight CTAs per
  // SM loops over the rows
  const int wpb = static_cast<int>(std::min<int64_t>(nm::kQuantWarps, std::max<int64_t>(1, rows / num_sms())));
  const int64_t ctas = std::min<int64_t>(ceil_div(rows, int64_t(wpb)), int64_t(num_sms()) * 8);
  const dim3 grid(static_cast<unsigned>(ctas)), block(wpb * 32);
  const int64_t gpl = ceil_div(K / M, int64_t(32));             // groups per lane
  cudaError_t err;
  // the lane's groups stay in registers when there are at most GR of them
#define NM_QL(MM, TT)                                                                                       \
  {                                                                                                         \
    constexpr int GR = nm::quant_groups_in_regs(MM, sizeof(TT));                                            \
    if (gpl <= GR)                                                                                          \
      err = launch_pdl(nm::k_quant_lift_fp8<MM, TT, GR>, grid, block, 0, st, static_cast<const TT*>(src), rows, \
                       K, ld, codes_out, scale_out, Kl);                                                    \
    else                                                                                                    \
      err = launch_pdl(nm::k_quant_lift_fp8<MM, TT, 0>, grid, block, 0, st, static_cast<const TT*>(src), rows, \
                       K, ld, codes_out, scale_out, Kl);                                                    \
  }
  if (dt == NM_BF16) {
    switch (M) {
      case 4: NM_QL(4, uint16_t) break;
      case 8: NM_QL(8, uint16_t) break;
      case 16: NM_QL(16, uint16_t) break;
      default: NM_QL(32, uint16_t) break;
    }
  } else {
    switch (M) {
      case 4: NM_QL(4, uint32_t) break;
      case 8: NM_QL(8, uint32_t) break;
      case 16: NM_QL(16, uint32_t) break;
      default: NM_QL(32, uint32_t) break;
    }
  }
#undef NM_QL
  NM_CUDA_TRY(err);
  NM_CUDA_TRY(cudaGetLastError());
  return NM_OK;
}

int nm_prune_compress_fp8(const void* src, int64_t rows, int64_t K, int64_t ld, int N, int M,
                          uint32_t* mask_out, uint8_t* codes_out, float* scale_out, uint8_t* meta_out,
                          void* stream) {
  int rc = check_prune_args(src, NM_BF16, rows, K, ld, N, M, codes_out, meta_out);
  if (rc != NM_OK) return rc;
  const int64_t Kl = nm_lifted_k(K, M);
  if (Kl % 16 != 0) return NM_ERR_UNSUPPORTED;
  if (mask_out != nullptr && !aligned16(mask_out)) return NM_ERR_ALIGNMENT;
  if (rows == 0) return NM_OK;
  if (scale_out == nullptr) return NM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(scale_out) & 3u) != 0) return NM_ERR_ALIGNMENT;
  auto st = static_cast<cudaStream_t>(stream);
  // per-token scales first, then the prune writes the kept values' codes
  const unsigned rgrid = static_cast<unsigned>(std::min<int64_t>(rows, int64_t(1) << 30));
  NM_CUDA_TRY(launch_pdl(nm::k_row_scale_fp8, dim3(rgrid), dim3(256), 0, st,
                         static_cast<const uint16_t*>(src), rows, K, ld, scale_out));
  return launch_prune<uint16_t, true>(static_cast<const uint16_t*>(src), rows, K, ld, N, M, mask_out, codes_out,
                                      meta_out, st, scale_out);
}

size_t slide_decompose_fp8_workspace_size(int64_t rows, int64_t K, int M) {
  const int64_t Kl = nm_lifted_k(K, M);
  if (Kl < 0 || rows < 0) return 0;
  const size_t vals = static_cast<size_t>(ceil_div(rows * (Kl / 2) * 2, int64_t(256)) * 256);
  return vals + nm_meta_bytes(rows, K, M);
}

int slide_decompose_fp8(const void* w, int64_t rows, int64_t K, int N, int M, uint8_t* vals_out,
                        float* scale_out, uint8_t* meta_out, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_prune_args(w, NM_BF16, rows, K, K, N, M, vals_out, meta_out);
  if (rc != NM_OK) return rc;
  const int64_t Kl = nm_lifted_k(K, M);
  if (Kl % 16 != 0) return NM_ERR_UNSUPPORTED;
  if (rows == 0) return NM_OK;
  if (scale_out == nullptr || ws == nullptr) return NM_ERR_INVALID_ARG;
  if (ws_bytes < slide_decompose_fp8_workspace_size(rows, K, M)) return NM_ERR_WORKSPACE;
  if (!aligned16(ws) || (reinterpret_cast<uintptr_t>(scale_out) & 3u) != 0) return NM_ERR_ALIGNMENT;
  auto st = static_cast<cudaStream_t>(stream);
  auto wv = static_cast<uint8_t*>(ws);
  uint8_t* wm = wv + (slide_decompose_fp8_workspace_size(rows, K, M) - nm_meta_bytes(rows, K, M));
  // 16-bit windows first (the same pruning and window split), then 8-bit codes and metadata
  if ((rc = launch_prune(static_cast<const uint16_t*>(w), rows, K, K, N, M, nullptr, wv, wm, st)) != NM_OK) return rc;
  const unsigned rgrid = static_cast<unsigned>(std::min<int64_t>(rows, int64_t(1) << 30));
  NM_CUDA_TRY(launch_pdl(nm::k_row_scale_fp8, dim3(rgrid), dim3(256), 0, st,
                         static_cast<const uint16_t*>(w), rows, K, K, scale_out));
  const int64_t chunks = rows * (Kl / 16);
  const unsigned vgrid = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(ceil_div(chunks, 256), int64_t(1) << 30)));
  NM_CUDA_TRY(launch_pdl(nm::k_quant_vals_fp8, dim3(vgrid), dim3(256), 0, st,
                         reinterpret_cast<const uint16_t*>(wv), rows, Kl / 2, static_cast<const float*>(scale_out),
                         vals_out));
  const int64_t blocks = ceil_div(rows, int64_t(128)) * ceil_div(Kl, int64_t(128));
  const unsigned mgrid = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(ceil_div(blocks * 128, 256), int64_t(1) << 30)));
  NM_CUDA_TRY(launch_pdl(nm::k_meta_f16_to_8, dim3(mgrid), dim3(256), 0, st,
                         static_cast<const uint8_t*>(wm), blocks, meta_out));
  NM_CUDA_TRY(cudaGetLastError());
  return NM_OK;
}

int nm_sparse_gemm_fp8(const nm_sparse_operand* S, const float* S_scale, const void* D, const float* D_scale,
                       int64_t rows_d, nm_side side, void* Y, nm_dtype out_dt, void* stream) {
  if (S == nullptr) return NM_ERR_INVALID_ARG;
  if (side != NM_ACT && side != NM_WEIGHT) return NM_ERR_INVALID_ARG;
  if (out_dt != NM_BF16 && out_dt != NM_FP32) return NM_ERR_INVALID_ARG;
  if (S->rows < 0 || rows_d < 0 || S->K <= 0 || S->M <= 0 || S->K % S->M != 0) return NM_ERR_INVALID_ARG;
  if (!m_supported(S->M)) return NM_ERR_UNSUPPORTED;
  if (S->K_lift != nm_lifted_k(S->K, S->M)) return NM_ERR_INVALID_ARG;
  if (S->K_lift % 128 != 0) return NM_ERR_UNSUPPORTED;
  const char* env = std::getenv("NMSPARSE_GEMM");
  const std::string mode = env != nullptr ? env : "auto";
  // decode-shaped products (a few rows of B) and NMSPARSE_GEMM=1cta take the
  // single-CTA kernel (any row count); the SM-pair kernel needs whole
  // 256-row blocks of the sparse operand
  const bool single = mode == "1cta" || (mode == "auto" && rows_d <= 64);
  if (!single && S->rows % 256 != 0) return NM_ERR_UNSUPPORTED;
  if (S->rows == 0 || rows_d == 0) return NM_OK;
  if (D == nullptr || Y == nullptr || S->vals == nullptr || S->meta == nullptr || S_scale == nullptr ||
      D_scale == nullptr)
    return NM_ERR_INVALID_ARG;
  if (!aligned16(S->vals) || !aligned16(S->meta) || !aligned16(D) || !aligned16(Y) ||
      (reinterpret_cast<uintptr_t>(S_scale) & 3u) != 0 || (reinterpret_cast<uintptr_t>(D_scale) & 3u) != 0)
    return NM_ERR_ALIGNMENT;
  GemmPlan p;
  p.a_s = S->vals;
  p.b = D;
  p.rows_a = S->rows;
  p.rows_b = rows_d;
  p.ks_lift = S->K_lift;
  p.kd = 0;
  p.meta = static_cast<const uint8_t*>(S->meta);
  p.y = Y;
  p.out_fp32 = out_dt == NM_FP32;
  p.transpose = side == NM_WEIGHT;
  p.ldy = side == NM_ACT ? rows_d : S->rows;
  p.a_static = side == NM_WEIGHT;
  p.fp8 = 1;
  p.scale_a = S_scale;
  p.scale_b = D_scale;
  auto st = static_cast<cudaStream_t>(stream);
  // Decode-shaped products (a few rows of B: tokens of a weight-sparse
  // product) run on single CTAs, 128 rows of A per tile, with cluster split-K
  // over the reduction.
  if (single) {
    const int bn1 = pick_bn(p.rows_b);
    const int64_t tiles1 = ceil_div(p.rows_a, int64_t(nm::kBM)) * ceil_div(p.rows_b, int64_t(bn1));
    const int splits = pick_splits(tiles1, ceil_div(p.ks_lift, int64_t(256)));
    switch (bn1) {
      case 16: return launch_gemm_bn<16, true>(p, splits, st);
      case 32: return launch_gemm_bn<32, true>(p, splits, st);
      case 64: return launch_gemm_bn<64, true>(p, splits, st);
      default: return launch_gemm_bn<128, true>(p, splits, st);
    }
  }
  if (p.rows_a % 512 == 0) {
    // 512-row tiles (two 256-row MMAs per k-slice share the B stage)
    if (mode == "2cta192x2") return launch_gemm_2cta<192, 1, 2, true>(p, st);
    if (mode == "2cta160x2") return launch_gemm_2cta<160, 1, 2, true>(p, st);
    if (mode == "2cta128x2") return launch_gemm_2cta<128, 1, 2, true>(p, st);
  }
  int bn = 0;
  if (mode == "2cta224") bn = 224;
  if (mode == "2cta192") bn = 192;
  if (mode == "2cta160") bn = 160;
  if (mode == "2cta128") bn = 128;
  if (bn == 0) {
    // Tile width by waves over the SM pairs: cost = waves * (BN + 48), the
    // 48 standing for a tile's fixed share (measured: 192 wide at 4096 rows
    // of B, 160 at 2048, 128 at 512).
    const int64_t pairs = std::max(1, num_sms() / 2);
    const int64_t tiles_m = ceil_div(p.rows_a, int64_t(256));
    int64_t best = -1;
    for (int cand : {224, 192, 160, 128}) {
      const int64_t waves = ceil_div(tiles_m * ceil_div(p.rows_b, int64_t(cand)), pairs);
      const int64_t cost = waves * (cand + 48);
      if (best < 0 || cost < best) { best = cost; bn = cand; }
    }
  }
  switch (bn) {
    case 192: return launch_gemm_2cta<192, 2, 1, true>(p, st);
    case 160: return launch_gemm_2cta<160, 2, 1, true>(p, st);
    case 128: return launch_gemm_2cta<128, 2, 1, true>(p, st);
    default: return launch_gemm_2cta<224, 2, 1, true>(p, st);
  }
}

int nm_dense_gemm(const void* A, int64_t rows_a, const void* B, int64_t rows_b, int64_t K, void* Y,
                  nm_dtype out_dt, void* stream) {
  if (out_dt != NM_BF16 && out_dt != NM_FP32) return NM_ERR_INVALID_ARG;
  if (rows_a < 0 || rows_b < 0 || K <= 0) return NM_ERR_INVALID_ARG;
  if (K % 16 != 0) return NM_ERR_UNSUPPORTED;
  if (rows_a == 0 || rows_b == 0) return NM_OK;
  if (A == nullptr || B == nullptr || Y == nullptr) return NM_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(Y)) return NM_ERR_ALIGNMENT;
  GemmPlan p;
  p.a_d = A;
  p.b = B;
  p.rows_a = rows_a;
  p.rows_b = rows_b;
  p.ks_lift = 0;
  p.kd = K;
  p.y = Y;
  p.ldy = rows_b;
  p.out_fp32 = out_dt == NM_FP32;
  return run_gemm(p, static_cast<cudaStream_t>(stream));
}

int64_t hybrid_dense_count(int64_t K, double dense_frac) {
  if (K <= 0) return 0;
  if (dense_frac <= 0.0) return 0;
  if (dense_frac >= 1.0) return K;
  return 4 * static_cast<int64_t>((dense_frac * static_cast<double>(K)) / 4.0);
}

size_t hybrid_prepare_workspace_size(int64_t O, int64_t K) {
  if (O <= 0 || K <= 0) return 0;
  const int64_t colnorm = K * 8, flags = ceil_div(K, 256) * 256, wsp = O * K * 2;
  return static_cast<size_t>(ceil_div(colnorm, 256) * 256 + flags + wsp);
}

int hybrid_prepare(const void* w, int64_t O, int64_t K, double dense_frac, nm_hybrid_weight* out, void* ws,
                   size_t ws_bytes, void* stream) {
  if (w == nullptr || out == nullptr || out->perm == nullptr) return NM_ERR_INVALID_ARG;
  if (O <= 0 || K <= 0 || K % 8 != 0) return NM_ERR_INVALID_ARG;
  const int64_t D = hybrid_dense_count(K, dense_frac);
  const int64_t Ks = K - D;
  if (out->O != O || out->K != K || out->K_dense != D) return NM_ERR_INVALID_ARG;
  if (Ks % 128 != 0) return NM_ERR_UNSUPPORTED;
  if (Ks > 0 && (out->vals_s == nullptr || out->meta_s == nullptr)) return NM_ERR_INVALID_ARG;
  if (D > 0 && out->W_d == nullptr) return NM_ERR_INVALID_ARG;
  if (ws == nullptr || ws_bytes < hybrid_prepare_workspace_size(O, K)) return NM_ERR_WORKSPACE;
  if (!aligned16(w) || !aligned16(ws) || !aligned16(out->perm) ||
      (Ks > 0 && (!aligned16(out->vals_s) || !aligned16(out->meta_s))) || (D > 0 && !aligned16(out->W_d)))
    return NM_ERR_ALIGNMENT;
  auto st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  double* colnorm = reinterpret_cast<double*>(base);
  uint8_t* is_dense = base + ceil_div(K * 8, 256) * 256;
  uint16_t* wsp = reinterpret_cast<uint16_t*>(is_dense + ceil_div(K, 256) * 256);
  const unsigned cb = static_cast<unsigned>(ceil_div(K, 128));
  NM_CUDA_TRY(launch_pdl(nm::k_colnorm_f64, dim3(cb), dim3(128), 0, st, static_cast<const uint16_t*>(w), O, K,
                         colnorm));
  NM_CUDA_TRY(launch_pdl(nm::k_hybrid_rank, dim3(cb), dim3(128), 0, st, static_cast<const double*>(colnorm), K, D,
                         is_dense));
  NM_CUDA_TRY(launch_pdl(nm::k_hybrid_perm, dim3(cb), dim3(128), 0, st, static_cast<const uint8_t*>(is_dense), K,
                         D, out->perm));
  const int64_t gblocks = std::max<int64_t>(1, std::min<int64_t>(ceil_div(O * K, 256), int64_t(num_sms()) * 16));
  NM_CUDA_TRY(launch_pdl(nm::k_gather_cols, dim3(static_cast<unsigned>(gblocks)), dim3(256), 0, st,
                         static_cast<const uint16_t*>(w), O, K, static_cast<const int32_t*>(out->perm), Ks, wsp,
                         static_cast<uint16_t*>(out->W_d)));
  if (Ks > 0) return launch_prune(wsp, O, Ks, Ks, 2, 4, nullptr, out->vals_s, out->meta_s, st);
  return NM_OK;
}

size_t hybrid_gemm_workspace_size(const nm_hybrid_weight* W, int64_t B) {
  if (W == nullptr || B <= 0) return 0;
  return static_cast<size_t>(ceil_div(B * W->K * 2, 256) * 256);
}

int hybrid_gemm(const void* X, int64_t B, const nm_hybrid_weight* W, void* Y, nm_dtype out_dt, void* ws,
                size_t ws_bytes, void* stream) {
  if (X == nullptr || W == nullptr || Y == nullptr) return NM_ERR_INVALID_ARG;
  if (out_dt != NM_BF16 && out_dt != NM_FP32) return NM_ERR_INVALID_ARG;
  if (B < 0 || W->O <= 0 || W->K <= 0 || W->K_dense < 0 || W->K_dense > W->K || W->K % 8 != 0)
    return NM_ERR_INVALID_ARG;
  const int64_t Ks = W->K - W->K_dense;
  if (Ks % 128 != 0) return NM_ERR_UNSUPPORTED;
  if (Ks > 0 && (W->vals_s == nullptr || W->meta_s == nullptr)) return NM_ERR_INVALID_ARG;
  if (W->K_dense > 0 && W->W_d == nullptr) return NM_ERR_INVALID_ARG;
  if (B == 0) return NM_OK;
  const bool gather = W->perm != nullptr;
  if (gather && (ws == nullptr || ws_bytes < hybrid_gemm_workspace_size(W, B))) return NM_ERR_WORKSPACE;
  if (!aligned16(X) || !aligned16(Y) || (gather && !aligned16(ws)) || (Ks > 0 && !aligned16(W->vals_s)) ||
      (W->K_dense > 0 && !aligned16(W->W_d)))
    return NM_ERR_ALIGNMENT;
  auto st = static_cast<cudaStream_t>(stream);
  const uint16_t* xp = static_cast<const uint16_t*>(X);
  if (gather) {
    uint16_t* g = static_cast<uint16_t*>(ws);
    const int64_t gblocks = std::max<int64_t>(1, std::min<int64_t>(ceil_div(B * W->K, 256), int64_t(num_sms()) * 4));
    NM_CUDA_TRY(launch_pdl(nm::k_gather_cols, dim3(static_cast<unsigned>(gblocks)), dim3(256), 0, st,
                           static_cast<const uint16_t*>(X), B, W->K, static_cast<const int32_t*>(W->perm), W->K, g,
                           static_cast<uint16_t*>(nullptr)));
    xp = g;
  }
  GemmPlan p;
  p.a_s = W->vals_s;
  p.a_d = W->W_d;
  p.b = xp;
  p.rows_a = W->O;
  p.rows_b = B;
  p.ks_lift = Ks;
  p.kd = W->K_dense;
  p.meta = static_cast<const uint8_t*>(W->meta_s);
  p.y = Y;
  p.ldy = W->O;
  p.out_fp32 = out_dt == NM_FP32;
  p.transpose = 1;
  p.a_static = 1;
  return run_gemm(p, st);
}

// --------------------------------------------------------- hybrid GLU MLP

int64_t spense_dense_count(int64_t I, double dense_frac) {
  if (I <= 0 || dense_frac <= 0.0) return 0;
  if (dense_frac >= 1.0) return I;
  return 256 * static_cast<int64_t>((dense_frac * static_cast<double>(I)) / 256.0);
}

size_t spense_mlp_prepare_workspace_size(int64_t d, int64_t I) {
  if (d <= 0 || I <= 0) return 0;
  const int64_t vec = ceil_div(I * 8, int64_t(256)) * 256;                 // one fp64 vector of I
  const int64_t flags = ceil_div(I, int64_t(256)) * 256;
  const int64_t ug = ceil_div(2 * I * d * 2, int64_t(256)) * 256;          // gathered sparse up/gate rows
  const int64_t dn = ceil_div(d * I * 2, int64_t(256)) * 256;              // gathered sparse down columns
  return static_cast<size_t>(4 * vec + flags + ug + dn);
}

int spense_mlp_prepare(const void* w_up, const void* w_gate, const void* w_down, double dense_frac,
                       nm_spense_mlp* out, void* ws, size_t ws_bytes, void* stream) {
  if (w_up == nullptr || w_gate == nullptr || w_down == nullptr || out == nullptr || out->perm == nullptr)
    return NM_ERR_INVALID_ARG;
  const int64_t d = out->d, I = out->I, D = spense_dense_count(I, dense_frac), Is = I - D;
  if (d <= 0 || I <= 0 || out->D != D) return NM_ERR_INVALID_ARG;
  if (d % 128 != 0 || I % 256 != 0) return NM_ERR_UNSUPPORTED;
  if (Is > 0 && (out->ug_vals == nullptr || out->ug_meta == nullptr || out->down_vals == nullptr ||
                 out->down_meta == nullptr))
    return NM_ERR_INVALID_ARG;
  if (D > 0 && (out->ug_dense == nullptr || out->down_dense == nullptr)) return NM_ERR_INVALID_ARG;
  if (ws == nullptr || ws_bytes < spense_mlp_prepare_workspace_size(d, I)) return NM_ERR_WORKSPACE;
  if (!aligned16(w_up) || !aligned16(w_gate) || !aligned16(w_down) || !aligned16(ws) || !aligned16(out->perm) ||
      (Is > 0 && (!aligned16(out->ug_vals) || !aligned16(out->ug_meta) || !aligned16(out->down_vals) ||
                  !aligned16(out->down_meta))) ||
      (D > 0 && (!aligned16(out->ug_dense) || !aligned16(out->down_dense))))
    return NM_ERR_ALIGNMENT;
  auto st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  const int64_t vec = ceil_div(I * 8, int64_t(256)) * 256;
  double* rn_up = reinterpret_cast<double*>(base);
  double* rn_gate = reinterpret_cast<double*>(base + vec);
  double* cn_down = reinterpret_cast<double*>(base + 2 * vec);
  double* score = reinterpret_cast<double*>(base + 3 * vec);
  uint8_t* is_dense = base + 4 * vec;
  uint16_t* ug_sp = reinterpret_cast<uint16_t*>(is_dense + ceil_div(I, int64_t(256)) * 256);
  uint16_t* dn_sp = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(ug_sp) +
                                                ceil_div(2 * I * d * 2, int64_t(256)) * 256);
  const auto* up = static_cast<const uint16_t*>(w_up);
  const auto* gate = static_cast<const uint16_t*>(w_gate);
  const auto* down = static_cast<const uint16_t*>(w_down);
  const unsigned ib = static_cast<unsigned>(ceil_div(I, int64_t(128)));
  NM_CUDA_TRY(launch_pdl(nm::k_rownorm_f64, dim3(ib), dim3(128), 0, st, up, I, d, rn_up));
  NM_CUDA_TRY(launch_pdl(nm::k_rownorm_f64, dim3(ib), dim3(128), 0, st, gate, I, d, rn_gate));
  NM_CUDA_TRY(launch_pdl(nm::k_colnorm_f64, dim3(ib), dim3(128), 0, st, down, d, I, cn_down));
  NM_CUDA_TRY(launch_pdl(nm::k_add3_f64, dim3(ib), dim3(128), 0, st, static_cast<const double*>(rn_up),
                         static_cast<const double*>(rn_gate), static_cast<const double*>(cn_down), I, score));
  NM_CUDA_TRY(launch_pdl(nm::k_hybrid_rank, dim3(ib), dim3(128), 0, st, static_cast<const double*>(score), I, D,
                         is_dense));
  NM_CUDA_TRY(launch_pdl(nm::k_hybrid_perm, dim3(ib), dim3(128), 0, st, static_cast<const uint8_t*>(is_dense), I,
                         D, out->perm));
  const unsigned gb = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(ceil_div(2 * I * (d / 8), int64_t(256)),
                                                                                   int64_t(num_sms()) * 16)));
  NM_CUDA_TRY(launch_pdl(nm::k_gather_rows_ug, dim3(gb), dim3(256), 0, st, up, gate, d,
                         static_cast<const int32_t*>(out->perm), I, Is, ug_sp,
                         static_cast<uint16_t*>(out->ug_dense)));
  const unsigned cb = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(ceil_div(d * I, int64_t(256)),
                                                                                   int64_t(num_sms()) * 16)));
  NM_CUDA_TRY(launch_pdl(nm::k_gather_cols, dim3(cb), dim3(256), 0, st, down, d, I,
                         static_cast<const int32_t*>(out->perm), Is, dn_sp, static_cast<uint16_t*>(out->down_dense)));
  int rc;
  if (Is > 0) {
    if ((rc = launch_prune(static_cast<const uint16_t*>(ug_sp), 2 * Is, d, d, 2, 4, nullptr, out->ug_vals,
                           out->ug_meta, st)) != NM_OK)
      return rc;
    if ((rc = launch_prune(static_cast<const uint16_t*>(dn_sp), d, Is, Is, 2, 4, nullptr, out->down_vals,
                           out->down_meta, st)) != NM_OK)
      return rc;
  }
  return NM_OK;
}

size_t spense_mlp_workspace_size(const nm_spense_mlp* W, int64_t B) {
  if (W == nullptr || B <= 0 || W->I <= 0) return 0;
  return static_cast<size_t>(ceil_div(B * 2 * W->I * 2, int64_t(256)) * 256 + ceil_div(B * W->I * 2, int64_t(256)) * 256);
}

int spense_mlp(const void* X, int64_t B, const nm_spense_mlp* W, void* Y, void* ws, size_t ws_bytes, void* stream) {
  if (X == nullptr || W == nullptr || Y == nullptr) return NM_ERR_INVALID_ARG;
  const int64_t d = W->d, I = W->I, D = W->D, Is = I - D;
  if (B < 0 || d <= 0 || I <= 0 || D < 0 || D > I) return NM_ERR_INVALID_ARG;
  if (d % 128 != 0 || I % 256 != 0 || D % 256 != 0) return NM_ERR_UNSUPPORTED;
  // every packed weight the three launches read, checked before the first
  if (Is > 0 && (W->ug_vals == nullptr || W->ug_meta == nullptr || W->down_vals == nullptr ||
                 W->down_meta == nullptr))
    return NM_ERR_INVALID_ARG;
  if (D > 0 && (W->ug_dense == nullptr || W->down_dense == nullptr)) return NM_ERR_INVALID_ARG;
  if (B == 0) return NM_OK;
  if (ws == nullptr || ws_bytes < spense_mlp_workspace_size(W, B)) return NM_ERR_WORKSPACE;
  if (!aligned16(X) || !aligned16(Y) || !aligned16(ws) ||
      (Is > 0 && (!aligned16(W->ug_vals) || !aligned16(W->ug_meta) || !aligned16(W->down_vals) ||
                  !aligned16(W->down_meta))) ||
      (D > 0 && (!aligned16(W->ug_dense) || !aligned16(W->down_dense))))
    return NM_ERR_ALIGNMENT;
  auto st = static_cast<cudaStream_t>(stream);
  uint16_t* y_ug = static_cast<uint16_t*>(ws);
  uint16_t* h = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + ceil_div(B * 2 * I * 2, int64_t(256)) * 256);
  // up and gate: one output-split product, columns [up_s | gate_s | up_d | gate_d]
  GemmPlan p;
  p.a_s = W->ug_vals;
  p.a_d = W->ug_dense;
  p.meta = static_cast<const uint8_t*>(W->ug_meta);
  p.b = X;
  p.rows_a = 2 * I;
  p.rows_b = B;
  p.ks_lift = d;
  p.kd = d;
  p.out_split_rows = 2 * Is;
  p.y = y_ug;
  p.ldy = 2 * I;
  p.transpose = 1;
  p.a_static = 1;
  int rc;
  if ((rc = run_gemm(p, st)) != NM_OK) return rc;
  const unsigned sb = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(ceil_div(B * (I / 8), int64_t(256)),
                                                                                   int64_t(num_sms()) * 8)));
  NM_CUDA_TRY(launch_pdl(nm::k_silu_mul, dim3(sb), dim3(256), 0, st, static_cast<const uint16_t*>(y_ug), B, I, Is, h));
  // down: input-split on h, which is already in the permuted order
  nm_hybrid_weight dw{};
  dw.perm = nullptr;
  dw.vals_s = W->down_vals;
  dw.meta_s = W->down_meta;
  dw.W_d = W->down_dense;
  dw.O = d;
  dw.K = I;
  dw.K_dense = D;
  return hybrid_gemm(h, B, &dw, Y, NM_BF16, nullptr, 0, stream);
}

}  // extern "C"

// Scratch of hybrid_gemm_noalloc(): one fixed array per device, alive until
// the process exits.  Host code may not use its name as an address; the
// device address is looked up once per device below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[NM_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (cached).
int noalloc_scratch(void** out) {
  int dev = 0;
  NM_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return NM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    NM_CUDA_TRY(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return NM_OK;
}
}  // namespace

extern "C" {

int hybrid_gemm_noalloc(const void* X, int64_t B, const nm_hybrid_weight* W, void* Y, nm_dtype out_dt,
                        void* stream) {
  if (X == nullptr || W == nullptr || Y == nullptr || B < 0) return NM_ERR_INVALID_ARG;
  if (W->O <= 0 || W->K <= 0 || W->K_dense < 0 || W->K_dense > W->K) return NM_ERR_INVALID_ARG;
  // Only the gather (W->perm set) uses scratch: B x K bf16 values, B * K * 2
  // bytes, compared without forming the product (no overflow).
  void* ws = nullptr;
  if (W->perm != nullptr && B > 0) {
    if (B > static_cast<int64_t>(NM_NOALLOC_SCRATCH_BYTES / 2) / W->K) return NM_ERR_WORKSPACE;
    const int rc = noalloc_scratch(&ws);
    if (rc != NM_OK) return rc;
  }
  return hybrid_gemm(X, B, W, Y, out_dt, ws, ws != nullptr ? NM_NOALLOC_SCRATCH_BYTES : 0, stream);
}

// ------------------------------------------------ host-buffer pipeline

}  // extern "C"

namespace {
// The auxiliary stream of the chunked host-buffer pipeline (copies out) and
// the events that chain its two buffer slots, one set per device, created on
// first use and kept until the process exits.
struct HostPipe {
  bool ready = false;
  cudaStream_t s_in = nullptr, s_out = nullptr;
  // per buffer slot: X copied in, X consumed by the prune, GEMM done, Y copied out
  cudaEvent_t in[2] = {}, x_free[2] = {}, done[2] = {}, out[2] = {};
};
std::mutex g_pipe_mu;
HostPipe g_pipe[kMaxDevices];

int host_pipe(HostPipe** out) {
  int dev = 0;
  NM_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return NM_ERR_UNSUPPORTED;
  HostPipe& p = g_pipe[dev];
  if (!p.ready) {
    NM_CUDA_TRY(cudaStreamCreateWithFlags(&p.s_in, cudaStreamNonBlocking));
    NM_CUDA_TRY(cudaStreamCreateWithFlags(&p.s_out, cudaStreamNonBlocking));
    for (int b = 0; b < 2; ++b) {
      NM_CUDA_TRY(cudaEventCreateWithFlags(&p.in[b], cudaEventDisableTiming));
      NM_CUDA_TRY(cudaEventCreateWithFlags(&p.x_free[b], cudaEventDisableTiming));
      NM_CUDA_TRY(cudaEventCreateWithFlags(&p.done[b], cudaEventDisableTiming));
      NM_CUDA_TRY(cudaEventCreateWithFlags(&p.out[b], cudaEventDisableTiming));
    }
    p.ready = true;
  }
  *out = &p;
  return NM_OK;
}

// Default chunk of the host-buffer pipeline: 256 rows, or more when the
// chunk's product would otherwise leave more than half the SM pairs idle
// (256-row tiles x 224-wide columns), so that the math of a chunk stays well
// below the time of its copy in.
int64_t host_chunk_rows(int64_t T, int64_t O, int64_t chunk_rows) {
  if (chunk_rows > 0) return std::min(T, chunk_rows);
  const int64_t pairs = std::max(1, num_sms() / 2);
  const int64_t col_tiles = ceil_div(O, int64_t(224));
  const int64_t m_tiles = std::max<int64_t>(1, ceil_div(pairs, 2 * col_tiles));
  return std::min(T, 256 * m_tiles);
}

// Chunk c of the host-buffer pipeline: rows [r0, r0 + rows).  Chunks of Tc
// rows, the last one what is left; with the default chunk size a last chunk
// of 256 rows or more is split into (F - 128, 128), so that the work after the
// final copy in (the last chunk's prune, product and copy out) is short.
struct HostChunks {
  int64_t T, Tc, n;                               // rows, chunk rows, chunks
  bool split_tail;
};
HostChunks host_chunks(int64_t T, int64_t Tc, bool default_chunk) {
  const int64_t n = ceil_div(T, Tc);
  const int64_t last = T - (n - 1) * Tc;
  const bool split = default_chunk && last >= 256;
  return {T, Tc, split ? n + 1 : n, split};
}
void host_chunk_at(const HostChunks& h, int64_t c, int64_t* r0, int64_t* rows) {
  if (h.split_tail && c >= h.n - 2) {
    const int64_t last0 = (h.n - 2) * h.Tc;        // start of the chunk that was split
    if (c == h.n - 2) { *r0 = last0; *rows = h.T - last0 - 128; }
    else { *r0 = h.T - 128; *rows = 128; }
    return;
  }
  *r0 = c * h.Tc;
  *rows = std::min(h.Tc, h.T - *r0);
}

int64_t round256(int64_t b) { return ceil_div(b, int64_t(256)) * 256; }

// Bytes of one buffer slot: X chunk, compressed values, metadata, Y chunk.
int64_t host_slot_bytes(int64_t Tc, int64_t K, int M, int64_t O) {
  const int64_t Kl = nm_lifted_k(K, M);
  return round256(Tc * K * 2) + round256(Tc * (Kl / 2) * 2) +
         round256(static_cast<int64_t>(nm_meta_bytes(Tc, K, M))) + round256(Tc * O * 2);
}
}  // namespace

extern "C" {

size_t nm_act_sparse_linear_host_workspace_size(int64_t T, int64_t K, int N, int M, int64_t O, int64_t chunk_rows) {
  (void)N;
  if (T <= 0 || K <= 0 || O <= 0 || nm_lifted_k(K, M) < 0) return 0;
  const int64_t Tc = host_chunk_rows(T, O, chunk_rows);
  return static_cast<size_t>(2 * host_slot_bytes(Tc, K, M, O));
}

int nm_act_sparse_linear_host(const void* x_host, int64_t T, int64_t K, int N, int M, const void* w_lift, int64_t O,
                              void* y_host, int64_t chunk_rows, void* ws, size_t ws_bytes, void* stream) {
  if (T < 0 || K <= 0 || O <= 0 || chunk_rows < 0) return NM_ERR_INVALID_ARG;
  if (chunk_rows % 128 != 0) return NM_ERR_INVALID_ARG;
  const int64_t Tc = host_chunk_rows(T, O, chunk_rows);
  // the pattern and shapes are validated before anything is enqueued (the
  // placeholder address stands for the chunk buffers, which are never read here)
  void* const placeholder = reinterpret_cast<void*>(uintptr_t(256));
  int rc = check_prune_args(placeholder, NM_BF16, 1, K, K, N, M, placeholder, placeholder);
  if (rc != NM_OK) return rc;
  const int64_t Kl = nm_lifted_k(K, M);
  if (Kl % 16 != 0) return NM_ERR_UNSUPPORTED;
  if (T == 0) return NM_OK;
  if (x_host == nullptr || y_host == nullptr || w_lift == nullptr || ws == nullptr) return NM_ERR_INVALID_ARG;
  if (!aligned16(w_lift) || !aligned16(ws)) return NM_ERR_ALIGNMENT;
  if (ws_bytes < nm_act_sparse_linear_host_workspace_size(T, K, N, M, O, chunk_rows)) return NM_ERR_WORKSPACE;

  const int64_t slot = host_slot_bytes(Tc, K, M, O);
  uint8_t* base[2] = {static_cast<uint8_t*>(ws), static_cast<uint8_t*>(ws) + slot};
  auto st = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe* p = nullptr;
  if ((rc = host_pipe(&p)) != NM_OK) return rc;
  const HostChunks plan = host_chunks(T, Tc, chunk_rows == 0);
  const int64_t chunks = plan.n;
  // The caller's stream orders the call: both copy streams start after the
  // work queued on it so far.
  NM_CUDA_TRY(cudaEventRecord(p->done[0], st));
  NM_CUDA_TRY(cudaStreamWaitEvent(p->s_in, p->done[0], 0));
  NM_CUDA_TRY(cudaStreamWaitEvent(p->s_out, p->done[0], 0));
  NM_CUDA_TRY(cudaEventRecord(p->x_free[0], st));
  NM_CUDA_TRY(cudaEventRecord(p->x_free[1], st));
  NM_CUDA_TRY(cudaEventRecord(p->out[0], st));
  NM_CUDA_TRY(cudaEventRecord(p->out[1], st));
  auto enqueue_chunk = [&](int64_t c) -> int {
    const int b = static_cast<int>(c % 2);
    int64_t r0 = 0, rows = 0;
    host_chunk_at(plan, c, &r0, &rows);
    uint8_t* xd = base[b];
    uint8_t* vals = xd + round256(Tc * K * 2);
    uint8_t* meta = vals + round256(Tc * (Kl / 2) * 2);
    uint8_t* yd = meta + round256(static_cast<int64_t>(nm_meta_bytes(Tc, K, M)));
    // copy in on its own stream, once the prune of chunk c - 2 has read slot
    // b's X: it overlaps the prune and GEMM of chunk c - 1
    NM_CUDA_TRY(cudaStreamWaitEvent(p->s_in, p->x_free[b], 0));
    NM_CUDA_TRY(cudaMemcpyAsync(xd, static_cast<const uint8_t*>(x_host) + r0 * K * 2, static_cast<size_t>(rows * K * 2),
                                cudaMemcpyHostToDevice, p->s_in));
    NM_CUDA_TRY(cudaEventRecord(p->in[b], p->s_in));
    // prune and GEMM on the caller's stream, once X has landed and the copy
    // out of chunk c - 2 has read slot b's Y; the prune is launched without
    // programmatic serialisation, so it waits for the event, not only for the
    // preceding kernel
    NM_CUDA_TRY(cudaStreamWaitEvent(st, p->in[b], 0));
    NM_CUDA_TRY(cudaStreamWaitEvent(st, p->out[b], 0));
    int r = launch_prune(reinterpret_cast<const uint16_t*>(xd), rows, K, K, N, M, nullptr, vals, meta, st, nullptr,
                         nullptr, nullptr, /*early=*/false);
    if (r != NM_OK) return r;
    NM_CUDA_TRY(cudaEventRecord(p->x_free[b], st));
    nm_sparse_operand S{};
    S.vals = vals;
    S.meta = meta;
    S.rows = rows;
    S.K = K;
    S.N = N;
    S.M = M;
    S.K_lift = Kl;
    if ((r = nm_sparse_gemm(&S, w_lift, O, NM_ACT, yd, NM_BF16, nullptr, 0, stream)) != NM_OK) return r;
    NM_CUDA_TRY(cudaEventRecord(p->done[b], st));
    // copy out
    NM_CUDA_TRY(cudaStreamWaitEvent(p->s_out, p->done[b], 0));
    NM_CUDA_TRY(cudaMemcpyAsync(static_cast<uint8_t*>(y_host) + r0 * O * 2, yd, static_cast<size_t>(rows * O * 2),
                                cudaMemcpyDeviceToHost, p->s_out));
    NM_CUDA_TRY(cudaEventRecord(p->out[b], p->s_out));
    return NM_OK;
  };
  for (int64_t c = 0; c < chunks && rc == NM_OK; ++c) rc = enqueue_chunk(c);
  // `stream` reaches this point once every queued chunk has been copied out
  // (and, through them, every copy in); the join is made on the error path
  // too, so that no copy into y_host is still in flight when work queued
  // after this call on `stream` runs
  const cudaError_t j0 = cudaStreamWaitEvent(st, p->out[0], 0);
  const cudaError_t j1 = cudaStreamWaitEvent(st, p->out[1], 0);
  const cudaError_t j2 = cudaStreamWaitEvent(st, p->in[0], 0);
  const cudaError_t j3 = cudaStreamWaitEvent(st, p->in[1], 0);
  if (rc != NM_OK) return rc;
  NM_CUDA_TRY(j0);
  NM_CUDA_TRY(j1);
  NM_CUDA_TRY(j2);
  NM_CUDA_TRY(j3);
  return NM_OK;
}

const char* nm_status_string(int s) {
  switch (s) {
    case NM_OK: return "ok";
    case NM_ERR_INVALID_ARG: return "invalid argument";
    case NM_ERR_UNSUPPORTED: return "unsupported N:M pattern or shape";
    case NM_ERR_ALIGNMENT: return "pointer or leading dimension not 16-byte aligned";
    case NM_ERR_CUDA: return "CUDA error";
    case NM_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case NM_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int nm_last_cuda_error(void) { return g_last_cuda_error; }

const char* nm_last_gemm_kernel(void) { return g_last_gemm; }

int nm_get_device_error(void* stream) {
  NM_CUDA_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  unsigned v = 0;
  NM_CUDA_TRY(cudaMemcpyFromSymbol(&v, nm::g_status, sizeof(v)));
  if (v == 0) return NM_OK;
  const unsigned zero = 0;
  NM_CUDA_TRY(cudaMemcpyToSymbol(nm::g_status, &zero, sizeof(zero)));
  return static_cast<int>(v);
}

int nm_debug_fail_next_launch(int cuda_error) {
  if (cuda_error < 0) return NM_ERR_INVALID_ARG;
  g_fail_next_launch = cuda_error;
  return NM_OK;
}

int nm_debug_expire_wait(unsigned timeout_us, void* stream) {
  if (timeout_us == 0 || timeout_us > 10u * 1000u * 1000u) return NM_ERR_INVALID_ARG;
  nm::k_expire_wait<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(timeout_us) * 1000ull);
  NM_CUDA_TRY(cudaGetLastError());
  return NM_OK;
}

int nm_mma_rate_probe(int mode, int iters, double* flops_out, void* stream) {
  if (mode < 0 || mode > 2 || iters <= 0 || iters > 1000000 || flops_out == nullptr) return NM_ERR_INVALID_ARG;
  const int clusters = std::max(1, num_sms() / 2);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = nm::kProbeSmemLaunch;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static_assert(nm::kProbeSmem <= nm::kProbeSmemLaunch, "probe shared memory");
  cudaError_t e;
  switch (mode) {
    case 0:
      NM_CUDA_TRY(cudaFuncSetAttribute(nm::k_mma_probe<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, nm::kProbeSmemLaunch));
      e = cudaLaunchKernelEx(&cfg, nm::k_mma_probe<0>, iters);
      break;
    case 1:
      NM_CUDA_TRY(cudaFuncSetAttribute(nm::k_mma_probe<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, nm::kProbeSmemLaunch));
      e = cudaLaunchKernelEx(&cfg, nm::k_mma_probe<1>, iters);
      break;
    default:
      NM_CUDA_TRY(cudaFuncSetAttribute(nm::k_mma_probe<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, nm::kProbeSmemLaunch));
      e = cudaLaunchKernelEx(&cfg, nm::k_mma_probe<2>, iters);
      break;
  }
  NM_CUDA_TRY(e);
  NM_CUDA_TRY(cudaGetLastError());
  const double k = mode == 0 ? 16.0 : (mode == 1 ? 32.0 : 64.0);   // logical K per MMA
  *flops_out = static_cast<double>(clusters) * iters * 4.0 * 2.0 * 256.0 * nm::kProbeN * k;
  return NM_OK;
}

const char* nm_version(void) { return "nmsparse 0.1 (sm_100a)"; }

}  // extern "C"
