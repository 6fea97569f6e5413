/*
 * nmsparse.h -- C ABI of the B200 (sm_100a) N:M semi-structured sparse
 * linear-layer library.
 *
 * Conventions, for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    allocates no device memory; scratch space is passed in as `ws` with a
 *    size from the matching *_workspace_size() call.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *    asynchronous on that stream and return a status code; they validate all
 *    arguments before launching anything, and a call that returns an error
 *    has launched nothing and written no output.
 *  - Matrices are row-major.  "bf16" is IEEE bfloat16 (uint16 bit patterns),
 *    "fp32" is IEEE binary32.  The reduction dimension K is the contiguous
 *    one for every operand.
 *  - Pointers must be 16-byte aligned and leading dimensions multiples of 8
 *    elements (16 bytes for bf16 rows), else NM_ERR_ALIGNMENT.
 *  - Weight operands (the sparse operand of NM_WEIGHT products, the hybrid
 *    and GLU-MLP weights) may be read before a kernel waits for the work
 *    queued ahead of it.  Every kernel of this library lets the next one
 *    start early (programmatic dependent launch), so a run of library calls
 *    can be in flight together: a weight must not be written by a library
 *    call that may still be running.  Prepare weights ahead, and separate
 *    the preparation from their use by a stream synchronisation, an event
 *    wait or a copy (as offline preparation is).  Everything else waits for
 *    the preceding work.
 *
 * Terms.  An N:M pattern keeps the N entries of largest magnitude in every
 * aligned group of M consecutive entries along K, ties going to the lower
 * index.  For M = 2n the kept entries of a group are spread over n-1
 * overlapping windows of width 4 and stride 2 (2 entries each), which the
 * 2:4 sparse tensor cores execute; the dense operand is then "lifted" so that
 * lifted column g*4(n-1) + 4w + j is source column g*2n + 2w + j.  The lifted
 * width is K' = K * (2n-2) / n (K' = K for 2:4).
 *   [Motivating Next-Gen Accelerators with Flexible (N:M) Activation Sparsity
 *    via Benchmarking Lightweight Post-Training Sparsification Approaches,
 *    technical summary sections 1 and 2.A]
 *   [SlideSparse: Fast and Flexible (2N-2):2N Structured Sparsity, technical
 *    summary sections 2.A (sliding windows), 2.B (activation lifting),
 *    2.C (offline packer, online lift and 2:4 GEMM)]
 *   [SpenseGPT: Practical One-shot Pruning Enabling Sparse and Dense GEMMs for
 *    LLM Inference, technical summary sections 2.A (hybrid dense + 2:4 format,
 *    input-split) and 2.B (permuting the dense indices into one block)]
 */
#ifndef NMSPARSE_H
#define NMSPARSE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { NM_BF16 = 0, NM_FP32 = 1 } nm_dtype;

/* Which side of Y = X . W^T carries the sparse operand.
 * NM_ACT:    sparse = X [T x K], dense = lifted W [O x K'], Y [T x O].
 * NM_WEIGHT: sparse = W [O x K], dense = lifted X [T x K'], Y [T x O]
 *            (the product is formed as W . X^T and stored transposed). */
typedef enum { NM_ACT = 0, NM_WEIGHT = 1 } nm_side;

enum {
    NM_OK = 0,
    NM_ERR_INVALID_ARG = 1,    /* null pointer, negative size, K % M != 0, bad dtype */
    NM_ERR_UNSUPPORTED = 2,    /* N:M or shape outside what the kernels implement */
    NM_ERR_ALIGNMENT = 3,      /* pointer / leading dimension alignment */
    NM_ERR_CUDA = 4,           /* a CUDA call failed; see nm_last_cuda_error() */
    NM_ERR_DEVICE_TIMEOUT = 5, /* a kernel's bounded wait expired (nm_get_device_error) */
    NM_ERR_WORKSPACE = 6       /* ws NULL or ws_bytes below the required size */
};

/* A window-compressed sparse operand, as written by nm_prune_compress() or
 * slide_decompose().
 *   vals : bf16 [rows][K_lift/2]; window j of row r holds its two entries at
 *          vals[r][2j], vals[r][2j+1] (padding slots hold +0.0).
 *   meta : nm_meta_bytes(rows, K, M) bytes, the sparse-MMA metadata image
 *          (see nm_meta_bytes). */
typedef struct {
    const void *vals;
    const void *meta;
    int64_t rows;
    int64_t K;        /* original reduction length */
    int32_t N, M;
    int64_t K_lift;   /* nm_lifted_k(K, M) */
} nm_sparse_operand;

/* A hybrid dense + 2:4 weight W [O x K] (device buffers owned by the caller,
 * filled by hybrid_prepare()).
 *   perm   : int32 [K] = [sparse columns ascending | dense columns ascending]
 *   vals_s : bf16 [O][Ks/2], 2:4-compressed sparse block (Ks = K - K_dense,
 *            columns in perm order)
 *   meta_s : nm_meta_bytes(O, Ks, 4) bytes
 *   W_d    : bf16 [O][K_dense], the dense block (columns in perm order) */
typedef struct {
    int32_t *perm;
    void *vals_s;
    void *meta_s;
    void *W_d;
    int64_t O, K, K_dense;
} nm_hybrid_weight;

/* A GLU MLP y = (silu(x . W_gate^T) * (x . W_up^T)) . W_down^T in the
 * hybrid format (device buffers owned by the caller, filled by
 * spense_mlp_prepare()).  W_up, W_gate are [I x d], W_down is [d x I]; D of
 * the I intermediate indices stay dense (Is = I - D are 2:4).
 *   perm      : int32 [I] = [sparse indices ascending | dense ascending]
 *   ug_vals   : bf16 [2 Is][d/2], rows [up_s; gate_s] 2:4-compressed along d
 *   ug_meta   : nm_meta_bytes(2 Is, d, 4) bytes
 *   ug_dense  : bf16 [2 D][d], rows [up_d; gate_d]
 *   down_vals : bf16 [d][Is/2], W_down's sparse input columns (permuted order)
 *   down_meta : nm_meta_bytes(d, Is, 4) bytes
 *   down_dense: bf16 [d][D], W_down's dense input columns (permuted order) */
typedef struct {
    int32_t *perm;
    void *ug_vals;
    void *ug_meta;
    void *ug_dense;
    void *down_vals;
    void *down_meta;
    void *down_dense;
    int64_t d, I, D;
} nm_spense_mlp;

/* ------------------------------------------------------------------ sizes */

/* Lifted width K' = K*(M-2)/(M/2) for even M >= 4 (K' = K for M = 4);
 * -1 if M is odd, below 4, or does not divide K. */
int64_t nm_lifted_k(int64_t K, int M);

/* Bytes of the metadata image of a `rows` x K operand pruned N:M.  The image
 * is made of blocks of 128 rows x 128 lifted columns (2048 bytes, the
 * tensor-memory image of four sparse MMAs of K = 32): block (rb, kb) starts
 * at byte (rb * ceil(K'/128) + kb) * 2048; inside it, row m and window
 * q (0..31, four lifted columns each) hold their 4-bit index pair at lane
 * (m%8) + 8*((q%8)/4) + 16*(m/16), byte 4*(q/8) of that lane's 16 bytes,
 * nibble (q%4) + 4*((m/8)%2) of that 32-bit word.  Rows and windows past the
 * operand carry the pair (0,1).  0 on invalid arguments. */
size_t nm_meta_bytes(int64_t rows, int64_t K, int M);

/* ------------------------------------------------------------ prune steps */

/* Prunes `src` [rows x K] (row stride `ld` elements, dtype NM_BF16 or
 * NM_FP32) to N:M along K and writes its window-compressed form.
 * [Flexible (N:M) Activation Sparsity, technical summary §1 (N:M blocks:
 *  keep N of every M consecutive entries, chosen anew for every input) and
 *  §2.A (ACT: the absolute magnitude decides); SlideSparse, §2.A (the kept
 *  entries of a group of 2n spread over n-1 windows of width 4, stride 2).]
 *   mask_out : optional (may be NULL) uint32 [rows][ceil(K/32)]; bit k%32 of
 *              word k/32 is set iff entry k is kept.
 *   vals_out : bf16 [rows][K'/2] (fp32 inputs are rounded to nearest even).
 *   meta_out : nm_meta_bytes(rows, K, M) bytes.
 * Supported: M in {4, 8, 16, 32}; N <= 2 for M = 4, else 1 <= N <= M-2.
 * Magnitudes are compared as integers on the sign-cleared bit patterns. */
int nm_prune_compress(const void *src, nm_dtype dt, int64_t rows, int64_t K, int64_t ld,
                      int N, int M, uint32_t *mask_out, void *vals_out, void *meta_out,
                      void *stream);

/* The offline weight packer of the (2N-2):2N family: the same operation as
 * nm_prune_compress() restricted to N = M - 2 (6:8, 14:16, 30:32) or 2:4,
 * for a weight W [rows x K] with row stride K.
 * [SlideSparse, technical summary §2.A (sliding-window decomposition: n-1
 *  windows are necessary and sufficient for 2n-2 of 2n) and §2.C (the
 *  offline packer).] */
int slide_decompose(const void *w, nm_dtype dt, int64_t rows, int64_t K, int N, int M,
                    uint32_t *mask_out, void *vals_out, void *meta_out, void *stream);

/* [SlideSparse, technical summary §2.B (activation lifting: the dense
 *  operand is widened to K' = K (2n-2)/n so that every window meets its
 *  own copy of the columns it covers).]
 * Lifts the dense operand: dst[r][g*4(n-1) + 4w + j] = src[r][g*2n + 2w + j]
 * for M = 2n, src [rows x K] (row stride ld elements, bf16 or fp32),
 * dst bf16 [rows x K'] (row stride K').  M = 4 copies (and converts fp32).
 * K' must be a multiple of 8 (16-byte rows), else NM_ERR_ALIGNMENT. */
int nm_lift(const void *src, nm_dtype dt, int64_t rows, int64_t K, int64_t ld, int M,
            void *dst, void *stream);

/* The split window order (a layout of this library, for the (2N-2):2N
 * weight side).  Window w of group g covers elements g*2n + 2w .. + 3, so
 * a group's even windows 0, 2, ..., n-2 tile it and its odd windows overlap
 * them [SlideSparse, technical summary §2.A].  In the split order each row's
 * windows are every group's even windows, group by group, then every group's
 * odd windows; the lifted activations in that order are [X | the odd windows
 * of X], so the GEMM reads the raw activations for two thirds (6:8) of its
 * reduction and only the odd windows are materialised [§2.B-§2.C place the
 * lift inside the online kernel; this keeps X where it is instead].
 *
 * slide_decompose_split(): slide_decompose() with the windows of every row
 * in the split order: bf16 W [rows x K] (row stride K), N = M - 2 with
 * M = 8, 16 or 32, K a multiple of 128 (so that the even windows end on a
 * 128-K metadata block); else NM_ERR_UNSUPPORTED.  Outputs as
 * nm_prune_compress() (values [rows][K'/2], metadata image, optional mask);
 * the operand is multiplied by nm_sparse_gemm() (NM_WEIGHT) against lifted
 * activations in the same order, which nm_lift_odd() makes in place. */
int slide_decompose_split(const void *w, int64_t rows, int64_t K, int N, int M, uint32_t *mask_out,
                          void *vals_out, void *meta_out, void *stream);

/* nm_lift_odd(): x bf16 [rows x ld] holds X [rows x K] in its first K
 * columns; columns [K, K') receive the odd windows of X in the split order
 * (group g's odd window o = X[r][g*M + 4o + 2 .. + 5] at column
 * K + g*4(M/4 - 1) + 4o).  M = 8, 16 or 32 and K a multiple of 128 (else
 * NM_ERR_UNSUPPORTED); ld >= K' (else NM_ERR_INVALID_ARG); x 16-byte aligned
 * with 16-byte rows (else NM_ERR_ALIGNMENT).  With ld = K' the buffer is the
 * dense operand of nm_sparse_gemm() for a slide_decompose_split() weight. */
int nm_lift_odd(void *x, int64_t rows, int64_t K, int64_t ld, int M, void *stream);

/* ------------------------------------------------------------------- GEMM */

/* Y = sparse . dense^T (side NM_ACT) or its transpose (NM_WEIGHT), bf16
 * products accumulated in fp32 on the 2:4 sparse tensor cores.
 * [SlideSparse, technical summary §2.C (the windowed operand against the
 *  lifted one on 2:4 hardware; ideal speedup n/(n-1) over dense, §4).]
 *   S      : the compressed sparse operand (rows_s = S->rows).
 *   D      : bf16 lifted dense operand [rows_d][S->K_lift], row stride K_lift.
 *   Y      : NM_ACT -> [rows_s][rows_d]; NM_WEIGHT -> [rows_d][rows_s];
 *            row-major, dtype out_dt (NM_BF16 rounds to nearest even).
 *   ws     : optional scratch of nm_sparse_gemm_workspace_size() bytes,
 *            16-byte aligned (NULL, or fewer bytes: none).  Products on SM
 *            pairs whose tiles leave a last persistent round in which fewer
 *            than half the pairs would work split that round's tiles along K
 *            across the idle pairs, the parts' fp32 partial tiles going to ws
 *            and a second launch adding them in part order (stream-K tail);
 *            without ws that round runs whole.  The result is deterministic
 *            either way; the two schedules round the fp32 sums in different
 *            orders.  Its contents need no initialisation.
 * Requires K_lift % 16 == 0. */
size_t nm_sparse_gemm_workspace_size(const nm_sparse_operand *S, int64_t rows_d, nm_side side);
int nm_sparse_gemm(const nm_sparse_operand *S, const void *D, int64_t rows_d, nm_side side,
                   void *Y, nm_dtype out_dt, void *ws, size_t ws_bytes, void *stream);

/* The online half of the sliding-window method in one call: the activation
 * lift and the weight-sparse product, Y[rows_x][W->rows] = lift(X) . W_c^T
 * with lift() as in nm_lift().
 * [SlideSparse, technical summary §2.B (activation lifting: X is expanded
 *  to K' so that the windowed weight runs on 2:4 hardware) and §2.C (the
 *  online lift followed by the 2:4 GEMM).]
 *   W     : the packed weight (slide_decompose() or nm_prune_compress() of W).
 *   X     : raw bf16 activations [rows_x][W->K], row stride ldx elements
 *           (a multiple of 8), 16-byte aligned; NOT lifted.
 *   Y     : [rows_x][W->rows] row-major, dtype out_dt.
 *   ws    : slide_gemm_workspace_size() bytes, 16-byte aligned, or NULL when
 *           that size is 0.
 * Decode shapes run as ONE kernel -- rows_x <= 32 and the lifted panel of a
 * CTA's k-range fits its shared memory (16 rows at K = 4096 for 6:8 do; 32
 * rows need K of about 2048 or less): each CTA loads the raw columns of X
 * its k-range needs and writes their lift into shared memory itself, so the
 * lifted X never goes through global memory and no workspace is used.
 * Prefill shapes also run as ONE kernel -- W->rows a multiple of 256 and
 * rows_x >= 64: the SM-pair product, whose lift warps write every lifted B
 * stage into shared memory straight from X (global memory, no staging copy)
 * in place of the TMA load of a lifted copy.  slide_gemm_workspace_size()
 * returns 0 exactly for these two families of shapes.  Other shapes lift
 * into ws first and run nm_sparse_gemm().  Results equal nm_lift() followed
 * by nm_sparse_gemm() bit for bit (on the prefill path, with the tile width
 * that nm_sparse_gemm() picks for the same product: 128 below 512 rows of X,
 * else 224, or 256 when K' >= 16384 and rows_x <= 8192).  X may be written by
 * the preceding kernel in the stream; W follows the weight rule of
 * nm_sparse_gemm(); the prefill path needs ldx even. */
size_t slide_gemm_workspace_size(const nm_sparse_operand *W, int64_t rows_x);
int slide_gemm(const nm_sparse_operand *W, const void *X, int64_t rows_x, int64_t ldx, void *Y,
               nm_dtype out_dt, void *ws, size_t ws_bytes, void *stream);

/* Dense comparator on the same tensor-core pipeline: Y[rows_a][rows_b] =
 * A . B^T with A [rows_a x K], B [rows_b x K] bf16, K % 16 == 0. */
int nm_dense_gemm(const void *A, int64_t rows_a, const void *B, int64_t rows_b, int64_t K,
                  void *Y, nm_dtype out_dt, void *stream);

/* --------------------------------------------------------- 8-bit (E4M3) */

/* The 8-bit variant of the weight-sparse path: activations quantised per
 * token and lifted in one pass, weights packed offline with per-row scales,
 * and the sparse product run on the 8-bit sparse tensor cores (kind::f8f6f4,
 * E4M3 x E4M3, fp32 accumulate) with both scales applied in the epilogue.
 * [SlideSparse, technical summary §2.B (the lifting is fused into the
 *  per-token quantisation kernel that INT8/FP8 inference already runs) and
 *  §2.C (offline packer, online quantisation-slide kernel).]
 *
 * E4M3: the OCP 8-bit format with bias 7, 3 mantissa bits, largest finite
 * 448, no infinity.  Per row: amax = max |x|, scale = amax / 448 (fp32,
 * correctly rounded; 1 for an all-zero row), inv = 1 / scale (fp32, correctly
 * rounded), code = E4M3(x * inv) with the product rounded to fp32, then to
 * nearest even E4M3 and saturated to +-448.
 *
 * The 8-bit metadata image has the blocks of nm_meta_bytes() (128 rows x 128
 * lifted columns, 2048 bytes, block (rb, kb) at (rb * ceil(K'/128) + kb) *
 * 2048); inside a block row m and window q hold their index pair at byte
 * 16*m + q/2, low nibble for even q.  Rows and windows past the operand carry
 * the pair (0,1). */

/* Quantise + lift: codes_out [rows][K'] (row stride K', E4M3 codes in the
 * lifted order of nm_lift()), scale_out [rows] fp32.  src [rows x K], row
 * stride ld elements, NM_BF16 or NM_FP32.  K' must be a multiple of 16
 * (else NM_ERR_UNSUPPORTED); src and codes_out 16-byte aligned, scale_out
 * 4-byte aligned. */
int nm_quant_lift_fp8(const void *src, nm_dtype dt, int64_t rows, int64_t K, int64_t ld, int M,
                      uint8_t *codes_out, float *scale_out, void *stream);

/* Prune + compress in 8 bits (the activation-sparse side): per-row scale
 * scale_out[r] = amax(src[r]) / 448, then nm_prune_compress() of the bf16
 * src [rows x K] (row stride ld) with the kept values written as codes
 * E4M3(v * (1 / scale)) -- codes_out [rows][K'/2], two per window -- and the
 * metadata as the 8-bit image (meta_out, nm_meta_bytes(rows, K, M) bytes).
 * mask_out as in nm_prune_compress().  K' must be a multiple of 16. */
int nm_prune_compress_fp8(const void *src, int64_t rows, int64_t K, int64_t ld, int N, int M,
                          uint32_t *mask_out, uint8_t *codes_out, float *scale_out, uint8_t *meta_out,
                          void *stream);

/* Offline weight packer, 8-bit: slide_decompose() of the bf16 weight
 * W [rows x K] (row stride K), then per row scale = amax(W[r]) / 448 and the
 * kept values' codes E4M3(v * (1 / scale)).  vals_out [rows][K'/2] codes,
 * scale_out [rows], meta_out the 8-bit image (nm_meta_bytes(rows, K, M)
 * bytes).  ws: slide_decompose_fp8_workspace_size() bytes of scratch (the
 * 16-bit windows).  K' must be a multiple of 16. */
size_t slide_decompose_fp8_workspace_size(int64_t rows, int64_t K, int M);
int slide_decompose_fp8(const void *w, int64_t rows, int64_t K, int N, int M, uint8_t *vals_out,
                        float *scale_out, uint8_t *meta_out, void *ws, size_t ws_bytes, void *stream);

/* Y = (S . D^T) * S_scale[row of S] * D_scale[row of D], or its transpose
 * (side NM_WEIGHT), with S the packed 8-bit sparse operand (S->vals codes,
 * S->meta the 8-bit image) and D the lifted codes [rows_d][S->K_lift].
 * Requires S->K_lift % 128 == 0, and S->rows % 256 == 0 unless rows_d <= 64
 * (NM_ERR_UNSUPPORTED otherwise): decode-shaped products -- a few rows of D,
 * the tokens of a weight-sparse product -- run on single CTAs, 128 rows of S
 * per tile with split-K over the reduction, and take any row count; larger
 * ones run on SM pairs.  For NM_WEIGHT, S is a weight operand (see the
 * conventions at the top). */
int nm_sparse_gemm_fp8(const nm_sparse_operand *S, const float *S_scale, const void *D, const float *D_scale,
                       int64_t rows_d, nm_side side, void *Y, nm_dtype out_dt, void *stream);

/* ----------------------------------------------------------------- hybrid */

/* Dense column count for a dense share f: 4 * floor(f*K/4) (0 for f <= 0,
 * K for f >= 1). */
int64_t hybrid_dense_count(int64_t K, double dense_frac);

/* [SpenseGPT, technical summary §2.A (a dense region of K next to a 2:4
 *  region) and §2.B (the dense indices permuted into one contiguous block;
 *  the pages rank them by a calibration loss, replaced here by the weight's
 *  column energy).]
 * Offline: ranks the K columns of W [O x K] (bf16) by sum_r w[r][c]^2
 * (fp64, r ascending), keeps the top hybrid_dense_count(K, dense_frac)
 * columns dense (ties to the lower column), prunes the others 2:4 in
 * ascending column order, and fills `out` (buffers preallocated by the caller,
 * sizes in nm_hybrid_weight; out->O, out->K, out->K_dense must be set).
 * ws: hybrid_prepare_workspace_size(O, K) bytes. */
size_t hybrid_prepare_workspace_size(int64_t O, int64_t K);
int hybrid_prepare(const void *w, int64_t O, int64_t K, double dense_frac, nm_hybrid_weight *out,
                   void *ws, size_t ws_bytes, void *stream);

/* [SpenseGPT, technical summary §2.A (input-split: the sparse and the
 *  dense part of K accumulate into the same output).]
 * Y [B x O] = X[:, perm_s] . W_s^T + X[:, perm_d] . W_d^T (input-split, one
 * fp32 accumulator) for X bf16 [B x K] (row stride K).  With W->perm NULL,
 * X is taken as already permuted ([sparse columns | dense columns]) and no
 * gather runs.  ws: hybrid_gemm_workspace_size(W, B) bytes. */
size_t hybrid_gemm_workspace_size(const nm_hybrid_weight *W, int64_t B);
int hybrid_gemm(const void *X, int64_t B, const nm_hybrid_weight *W, void *Y, nm_dtype out_dt,
                void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------- hybrid GLU MLP */

/* The GLU mapping of the hybrid format.
 * [SpenseGPT, technical summary §2.A (output-split for W_up and W_gate,
 *  input-split for W_down) and §2.B (the intermediate indices can be
 *  permuted without changing the result; the dense ones are moved into one
 *  contiguous block).]
 * Dense count: D = 256 * floor(f * I / 256) (0 for f <= 0, I for f >= 1).
 * Selection: score[i] = (sum_k up[i][k]^2 + sum_k gate[i][k]^2) +
 * sum_o down[o][i]^2 in fp64 (each sum in ascending order); index i is dense
 * iff fewer than D indices beat it (higher score, or equal and lower index).
 * Requires d % 128 == 0 and I % 256 == 0. */
int64_t spense_dense_count(int64_t I, double dense_frac);
size_t spense_mlp_prepare_workspace_size(int64_t d, int64_t I);
int spense_mlp_prepare(const void *w_up, const void *w_gate, const void *w_down, double dense_frac,
                       nm_spense_mlp *out, void *ws, size_t ws_bytes, void *stream);

/* y [B x d] = the MLP of x [B x d] (bf16, row stride d): one output-split
 * GEMM for up and gate, silu(gate) * up in fp32, one input-split GEMM for
 * down; bf16 intermediates.  ws: spense_mlp_workspace_size(W, B) bytes. */
size_t spense_mlp_workspace_size(const nm_spense_mlp *W, int64_t B);
int spense_mlp(const void *X, int64_t B, const nm_spense_mlp *W, void *Y, void *ws, size_t ws_bytes,
               void *stream);

/* ------------------------------------------ per-token activation corrections */

/* Two corrections around the activation prune that need no calibration data.
 * [Motivating Next-Gen Accelerators with Flexible (N:M) Activation Sparsity,
 *  technical summary §2.B: D-PTS, a dynamic per-token shift that centres the
 *  activations on zero, and VAR, a per-token variance correction after
 *  pruning.  The page gives no formulas; these are the plainest readings.]
 *
 * NM_XF_SHIFT (D-PTS): mu[t] = fl32((sum_k x[t][k]) / K), the sum in fp64;
 *   the prune runs on xs[t][k] = bf16(fl32(x[t][k] - mu[t])) (nearest-even
 *   both times), and the product adds the shift back as mu[t] * s[o], with
 *   s[o] = fl32(sum_k W[o][k]) from nm_row_sums().
 * NM_XF_VAR: the kept entries of token t are rescaled by
 *   alpha[t] = sqrt(var(xs[t]) / var(kept xs[t])), var(u) = mean(u^2) -
 *   mean(u)^2 over all K entries (pruned ones as zeros), sums in fp64;
 *   alpha = 1 when the kept token has no variance.
 * The result is Y[t][o] = alpha[t] * (prune(xs[t]) . W[o]) + mu[t] * s[o],
 * with alpha = 1 without VAR and mu = 0 without the shift. */
#define NM_XF_SHIFT 1u
#define NM_XF_VAR 2u

/* nm_prune_compress() of the bf16 activation src [rows x K] (row stride ld)
 * with the corrections in `flags`: the compressed operand is that of xs (the
 * shifted token, or src itself without NM_XF_SHIFT), row_shift_out [rows]
 * receives mu (0 without the shift) and row_scale_out [rows] alpha (1 without
 * VAR), both fp32.  ws: nm_prune_compress_xf_workspace_size() bytes of scratch
 * when NM_XF_VAR is set (the per-chunk partial sums), else unused.  The
 * scales are 4-byte aligned; everything else as in nm_prune_compress(). */
size_t nm_prune_compress_xf_workspace_size(int64_t rows, int64_t K, int M);
int nm_prune_compress_xf(const void *src, int64_t rows, int64_t K, int64_t ld, int N, int M,
                         unsigned flags, uint32_t *mask_out, void *vals_out, void *meta_out,
                         float *row_scale_out, float *row_shift_out, void *ws, size_t ws_bytes,
                         void *stream);

/* Offline: sums_out[r] = fl32(sum_k w[r][k]) of a bf16 matrix [rows x K]
 * (row stride ld), the sum in fp64. */
int nm_row_sums(const void *w, int64_t rows, int64_t K, int64_t ld, float *sums_out, void *stream);

/* The activation-sparse product with the corrections applied in the GEMM
 * epilogue: Y[t][o] = (X_c[t] . W'[o]) * row_scale[t] + row_shift[t] *
 * w_row_sums[o], accumulated in fp32, stored as out_dt.  X is the operand
 * written by nm_prune_compress_xf(), W_lift the lifted weight [rows_w][K']
 * and w_row_sums [rows_w] the unlifted weight's row sums.  Other arguments
 * as in nm_sparse_gemm() with side NM_ACT. */
int nm_sparse_gemm_xf(const nm_sparse_operand *X, const void *W_lift, int64_t rows_w,
                      const float *row_scale, const float *row_shift, const float *w_row_sums,
                      void *Y, nm_dtype out_dt, void *stream);

/* Capacity, in bytes, of the library's built-in scratch array used by
 * hybrid_gemm_noalloc(): the gathered activations need B * K * 2 bytes. */
#define NM_NOALLOC_SCRATCH_BYTES (2u * 1024u * 1024u)

/* hybrid_gemm() for callers that cannot allocate device memory: no `ws`
 * argument, nothing is allocated.  (The pages have no counterpart to this
 * entry point; it exists for integration.)
 *
 * Who needs it: code whose device memory is owned and budgeted by a host
 * engine -- a plugin inside a serving framework that plans every byte ahead of
 * time, or a caller with no allocator of its own on the request path -- may not
 * call cudaMalloc or take memory from an allocator it does not control.
 *
 * Scratch: a fixed array of NM_NOALLOC_SCRATCH_BYTES (2 MiB) compiled into
 * the library.  Every GPU that loads the library keeps it until the process
 * exits.  Only a weight with a column permutation (W->perm not NULL) uses
 * it, for the gathered activations (B * K * 2 bytes); such calls with
 * B * K * 2 > NM_NOALLOC_SCRATCH_BYTES return NM_ERR_WORKSPACE and launch
 * nothing.  A malformed W (O or K not positive, K_dense outside [0, K])
 * returns NM_ERR_INVALID_ARG first.
 *
 * The first call on each device looks up the array's device address (with
 * that device current) and caches it; make that first call before any stream
 * capture.  The cached address does not survive cudaDeviceReset() (or any
 * other teardown of the device's primary context): after one, do not call
 * this entry point again in the same process.  All calls share the one
 * array: calls whose kernels overlap on the
 * GPU (different streams, no ordering between them) race on it.  Nothing in
 * the array has to start at zero -- each call writes every byte it reads.
 * Other arguments, layouts and errors are those of hybrid_gemm(). */
int hybrid_gemm_noalloc(const void *X, int64_t B, const nm_hybrid_weight *W, void *Y, nm_dtype out_dt,
                        void *stream);

/* ----------------------------------------------------- host-buffer pipeline */

/* The activation-sparse layer end to end from host memory:
 * y_host[T][O] = prune_{N:M}(x_host) . W^T, x_host bf16 [T][K] and y_host bf16
 * [T][O] in HOST memory (row-major, row strides K and O), w_lift the
 * device-resident lifted weight [O][K'] (nm_lift()).  The rows go through in
 * chunks of chunk_rows (a multiple of 128; 0 = 256 rows, or a multiple of 256
 * large enough that a chunk's product occupies at least half the SM pairs:
 * 512 for O = 4096 on 148 SMs; with this default a last chunk of F >= 256
 * rows goes as F - 128 and 128 rows, which shortens the work left after the
 * final copy in): each chunk is copied in
 * on one auxiliary stream, pruned and multiplied on `stream`, and copied out
 * on another, with two buffer slots, so that the copy in of the next chunk
 * and the copy out of the previous one overlap the math of the current one
 * (PCIe carries both directions at once).  The prune of a chunk is launched
 * without programmatic serialisation, so it starts only after its copy in.
 * The auxiliary streams and their events are created on the first call on a
 * device and kept; calls
 * are serialised on the host.  Host buffers should be page-locked
 * (cudaHostAlloc / cudaHostRegister), else the copies are not asynchronous.
 * Returns once everything is enqueued; y_host is complete when `stream`
 * reaches the point of the call, and both host buffers must stay allocated
 * until then.  Not for stream capture.
 * ws: nm_act_sparse_linear_host_workspace_size() bytes of device scratch (two
 * slots of: the chunk of X, its compressed values and metadata, the chunk of
 * Y), 16-byte aligned.  Results equal those of nm_prune_compress() +
 * nm_sparse_gemm() on each chunk. */
size_t nm_act_sparse_linear_host_workspace_size(int64_t T, int64_t K, int N, int M, int64_t O,
                                                int64_t chunk_rows);
/* Error after queuing: argument errors are found before anything is queued
 * (nothing runs, nothing is written).  A launch or copy that fails after
 * earlier chunks were queued returns its error with those chunks still
 * queued: their rows of y_host are written, the rest are not, and `stream`
 * is made to wait for the copies already queued, as on success. */
int nm_act_sparse_linear_host(const void *x_host, int64_t T, int64_t K, int N, int M, const void *w_lift,
                              int64_t O, void *y_host, int64_t chunk_rows, void *ws, size_t ws_bytes,
                              void *stream);

/* ------------------------------------------------------------- diagnostics */

const char *nm_status_string(int status);
/* The cudaError_t of the last NM_ERR_CUDA returned on this thread. */
int nm_last_cuda_error(void);
/* Name of the GEMM kernel instantiation that the most recent GEMM launch of
 * this library on the calling thread used, for example
 * "k_nm_gemm_2cta<256,1,1>" (tile width, accumulator buffers, 256-row
 * subtiles; ",fp8" for 8-bit operands, ",lift" for the in-GEMM lift,
 * "+splitS" when the last round's tiles were split into S parts along K) or
 * "k_nm_gemm<32>" (single-CTA kernel, tile width); "" before the first.  The string is owned by the
 * library and stays valid until the next GEMM launch on this thread. */
const char *nm_last_gemm_kernel(void);
/* Synchronises `stream`, then reads and clears the device status word that
 * kernels set when a bounded wait expires: NM_OK or NM_ERR_DEVICE_TIMEOUT
 * (or NM_ERR_CUDA if the synchronisation itself failed; NM_ERR_UNSUPPORTED
 * if a kernel found its launch shape beyond its shared-memory plan, which
 * the host-side checks rule out). */
int nm_get_device_error(void *stream);
/* Test hook for the launch-error path: the next kernel launch made by a call
 * of this library on the calling thread fails with cudaError_t `cuda_error`
 * (0 clears the hook) instead of launching, so that the call returns
 * NM_ERR_CUDA and nm_last_cuda_error() reports the code.  Nothing reaches
 * the GPU. */
int nm_debug_fail_next_launch(int cuda_error);
/* Test hook for the bounded-wait path: launches one CTA that waits on an
 * mbarrier no thread ever arrives on, giving up after timeout_us
 * microseconds and recording NM_ERR_DEVICE_TIMEOUT.  Faults nothing. */
int nm_debug_expire_wait(unsigned timeout_us, void *stream);
/* Tensor-core rate probe (diagnostic; grounds the roofline denominators):
 * every SM pair issues 4 * iters MMAs of 256 x 256 x K (cta_group::2) from
 * operands held in shared memory -- no loads, no epilogue -- so that
 * *flops_out / (the launch's duration) is the tensor pipe's own rate.
 * mode 0: bf16 dense (K = 16); 1: bf16 2:4 sparse (K = 32 logical);
 * 2: E4M3 2:4 sparse (K = 64 logical).  *flops_out counts 2 * M * N * K per
 * MMA (dense-equivalent), set on return; the caller times the launch (for
 * example with events around the call on `stream`). */
int nm_mma_rate_probe(int mode, int iters, double *flops_out, void *stream);
const char *nm_version(void);

#ifdef __cplusplus
}
#endif
#endif /* NMSPARSE_H */
