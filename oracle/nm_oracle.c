/*
 * nm_oracle.c -- CPU oracle for N:M semi-structured sparse linear layers.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this code.  It shares no code,
 * header, table or constant generator with the CUDA path, and the CUDA path
 * never calls it.
 *
 * What it computes, step by step, in plain loops (fp64 for every floating
 * point sum; bf16 and fp32 inputs are widened exactly to double):
 *
 *  1. prune     per aligned group of M along K keep the N entries of largest
 *               |value|, ties to the lower index.
 *               [Flexible (N:M) Activation Sparsity, technical summary
 *                §1 (N:M blocks, 6 configurations for 2:4, 12,870 for 8:16)
 *                and §2.A (ACT metric: absolute magnitude of the activation)]
 *  2. windows   a kept pattern of at most 2n-2 entries in a group of 2n is
 *               split over n-1 overlapping windows of width 4 and stride 2,
 *               each holding at most 2 entries; entries that do not fit in a
 *               window move on to the next one.
 *               [SlideSparse, technical summary §2.A, sliding-window
 *                decomposition; expansion factor gamma = (2N-2)/N]
 *  3. nibbles   every window stores two values and a 4-bit index pair.
 *  4. hw meta   the nibbles of a 128-row x 128-lifted-K block are permuted
 *               into the tensor-memory image that the sparse MMA reads.
 *  5. lift      the dense operand is widened so that lifted column
 *               g*4(n-1) + 4w + j holds source column g*2n + 2w + j.
 *               [SlideSparse, technical summary §2.B, activation lifting]
 *  6. linear    Y[t][o] = sum_k A[t][k] * B[o][k], k ascending, in fp64.
 *  7. hybrid    column energy sum_r w[r][c]^2 in fp64, the top share of K
 *               columns stays dense, the rest (ascending) is pruned 2:4;
 *               the input-split product accumulates both parts.
 *               [SpenseGPT, technical summary §2.A (dense region + 2:4 region,
 *                input-split with accumulation) and §2.B (permutation of the
 *                intermediate indices into one contiguous dense block)]
 *  7'. glu mlp  the GLU mapping of the hybrid format: one set of intermediate
 *               indices stays dense in all three projections, chosen by
 *               the summed fp64 energies of the up and gate rows and the down
 *               column; the indices are permuted into [sparse | dense]; up
 *               and gate are split by output (their sparse rows pruned 2:4
 *               along the model dimension), down by input (its sparse
 *               columns pruned 2:4 in the permuted order); h = silu(gate) * up.
 *               [SpenseGPT, technical summary §2.A (output-split for W_up
 *                and W_gate, input-split for W_down in GLU MLPs) and §2.B
 *                (intermediate indices can be permuted without changing the
 *                result; the dense ones are moved into one contiguous block)]
 *  8. fp8       8-bit (E4M3) variant: the dense operand is quantised per row
 *               (token) and lifted, the sparse operand's kept values are
 *               quantised per row (output channel), the sparse metadata takes
 *               the 8-bit image, and the product is rescaled by both scales.
 *               [SlideSparse, technical summary §2.B (lifting fused into the
 *                per-token quantisation of INT8/FP8 inference) and §2.C
 *                (offline packer, online quantisation-slide kernel)]
 *  9. shift/var two per-token corrections around the activation prune: the
 *               token is centred on its mean before pruning and the mean is
 *               added back through the weight's row sums (D-PTS, dynamic
 *               shift); the survivors are rescaled so that the pruned token
 *               keeps the variance of the token it came from (VAR).
 *               [Flexible (N:M) Activation Sparsity, technical summary §2.B
 *                (error mitigation: D-PTS, a dynamic per-token shift that
 *                centres the activations on zero; VAR, a per-token variance
 *                correction after pruning)]
 *
 * Where the pages are silent the plainest reading is taken and stated beside
 * the function that takes it.
 *
 * Parity pins: every function here is pinned by tests under tests/ against
 * invariants, brute force, closed forms or exact integer arithmetic.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_BF16 0
#define OR_FP32 1

/* ---------------------------------------------------------------- scalars */

static double bf16_bits_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double f32_bits_to_double(uint32_t u) {
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Magnitude key: the sign bit cleared, compared as an unsigned integer.  For
 * finite values this orders by |v|; +0 and -0 get the same key. */
static uint32_t key_at(const void *src, int dt, int64_t idx) {
    if (dt == OR_BF16) return ((const uint16_t *)src)[idx] & 0x7FFFu;
    return ((const uint32_t *)src)[idx] & 0x7FFFFFFFu;
}

static double value_at(const void *src, int dt, int64_t idx) {
    if (dt == OR_BF16) return bf16_bits_to_double(((const uint16_t *)src)[idx]);
    return f32_bits_to_double(((const uint32_t *)src)[idx]);
}

/* Round an fp32 bit pattern to bf16, nearest-even (used only where an fp32
 * input has to be stored as a bf16 value of the compressed operand). */
static uint16_t f32_bits_to_bf16_rne(uint32_t u) {
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0;
    uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7FFFu + lsb) >> 16);
}

static uint16_t bf16_at(const void *src, int dt, int64_t idx) {
    if (dt == OR_BF16) return ((const uint16_t *)src)[idx];
    return f32_bits_to_bf16_rne(((const uint32_t *)src)[idx]);
}

int or_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ prune */

/* Step 1.  Entry i of a group is kept iff fewer than N entries of the group
 * beat it, where j beats i when key_j > key_i, or key_j == key_i and j < i.
 * This is a stable sort by |value| descending followed by taking the first N.
 * keep[r*K + k] is set to 1 or 0.  Returns 0, or -1 on bad arguments. */
int or_prune(const void *src, int dt, int64_t rows, int64_t K, int N, int M,
             uint8_t *keep) {
    if (M <= 0 || N < 0 || N > M || K % M != 0 || rows < 0) return -1;
    const int64_t groups = K / M;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < groups; ++g) {
            const int64_t base = r * K + g * M;
            for (int i = 0; i < M; ++i) {
                uint32_t ki = key_at(src, dt, base + i);
                int beaten_by = 0;
                for (int j = 0; j < M; ++j) {
                    uint32_t kj = key_at(src, dt, base + j);
                    if (kj > ki || (kj == ki && j < i)) ++beaten_by;
                }
                keep[base + i] = (uint8_t)(beaten_by < N ? 1 : 0);
            }
        }
    }
    return 0;
}

/* Canonical bit mask: bit (k % 32) of word k / 32 of row r is keep[r][k]. */
void or_mask_pack(const uint8_t *keep, int64_t rows, int64_t K, uint32_t *mask) {
    const int64_t words = (K + 31) / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t w = 0; w < words; ++w) {
            uint32_t v = 0;
            for (int b = 0; b < 32; ++b) {
                int64_t k = w * 32 + b;
                if (k < K && keep[r * K + k]) v |= 1u << b;
            }
            mask[r * words + w] = v;
        }
}

/* ---------------------------------------------------------------- windows */

/* Step 2, one group of M = 2n positions.  Window w (0 <= w < n-1) spans the
 * positions 2w .. 2w+3, i.e. pairs w and w+1.  Window w first takes the kept
 * positions of pair w that no earlier window took, ascending, then kept
 * positions of pair w+1, ascending, until it holds two.
 * win[i] receives the window of kept position i (-1 if not kept), slot[i]
 * its slot 0/1 in that window.  For M == 4 the single window is the group.
 * Returns 0 on success, -1 if some kept position found no window (more than
 * 2n-2 kept), -2 on bad M. */
int or_window_assign(const uint8_t *keep_group, int M, int8_t *win, int8_t *slot) {
    if (M < 4 || M % 2 != 0 || M > 64) return -2;
    const int n = M / 2;
    for (int i = 0; i < M; ++i) { win[i] = -1; slot[i] = -1; }
    for (int w = 0; w < n - 1; ++w) {
        int held = 0;
        for (int p = w; p <= w + 1; ++p)
            for (int i = 2 * p; i <= 2 * p + 1; ++i)
                if (keep_group[i] && win[i] < 0 && held < 2) {
                    win[i] = (int8_t)w;
                    slot[i] = (int8_t)held;
                    ++held;
                }
    }
    for (int i = 0; i < M; ++i)
        if (keep_group[i] && win[i] < 0) return -1;
    return 0;
}

/* Batch form for exhaustive tests: masks[b] holds the kept bits of one group
 * (bit i = position i).  win_out[b*M + i] as in or_window_assign.  status[b]
 * receives the return value. */
void or_window_assign_batch(const uint64_t *masks, int64_t count, int M,
                            int8_t *win_out, int8_t *slot_out, int8_t *status) {
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < count; ++b) {
        uint8_t kg[64];
        for (int i = 0; i < M; ++i) kg[i] = (uint8_t)((masks[b] >> i) & 1u);
        status[b] = (int8_t)or_window_assign(kg, M, win_out + b * M, slot_out + b * M);
    }
}

/* Lifted width: K' = K * (2n-2) / n for M = 2n (4 windows-positions per
 * window, n-1 windows per group of 2n); K' = K for 2:4. */
int64_t or_lifted_k(int64_t K, int M) {
    if (M < 4 || M % 2 != 0 || K % M != 0) return -1;
    const int64_t n = M / 2;
    return K / M * 4 * (n - 1);
}

/* Steps 3 and 5 of one row set.  For each group g and window w the lifted
 * positions are g*4(n-1) + 4w + {0,1,2,3}; the two held entries are written
 * as values vals[r][g*2(n-1) + 2w + {0,1}] and their local indices (position
 * minus 2w) form the nibble i0 | i1 << 2 with i0 < i1.  A window holding one
 * entry at local index a is padded with the lowest local index other than a;
 * an empty window uses (0, 1).  Padded slots hold +0.0.
 * vals: bf16 bits [rows][K'/2]; nib: [rows][K'/4], one nibble per byte.
 * Returns 0, or -1 if a group's pattern does not fit the windows. */
int or_compress(const void *src, int dt, int64_t rows, int64_t K, int M,
                const uint8_t *keep, uint16_t *vals, uint8_t *nib) {
    const int64_t Kl = or_lifted_k(K, M);
    if (Kl < 0) return -2;
    const int n = M / 2, nw = n - 1;
    const int64_t groups = K / M;
    int failed = 0;
#pragma omp parallel for schedule(static) reduction(|: failed)
    for (int64_t r = 0; r < rows; ++r) {
        int8_t win[64], slot[64];
        for (int64_t g = 0; g < groups; ++g) {
            const int64_t base = r * K + g * M;
            if (or_window_assign(keep + base, M, win, slot) != 0) { failed = 1; continue; }
            for (int w = 0; w < nw; ++w) {
                int idx[2] = {-1, -1};
                uint16_t v[2] = {0, 0};
                for (int i = 0; i < M; ++i)
                    if (win[i] == w) {
                        idx[slot[i]] = i - 2 * w;
                        v[slot[i]] = bf16_at(src, dt, base + i);
                    }
                int i0, i1;
                uint16_t v0, v1;
                if (idx[0] < 0) {                 /* empty window */
                    i0 = 0; i1 = 1; v0 = 0; v1 = 0;
                } else if (idx[1] < 0) {          /* one entry, pad */
                    int a = idx[0], pad = (a == 0) ? 1 : 0;
                    if (pad < a) { i0 = pad; v0 = 0; i1 = a; v1 = v[0]; }
                    else         { i0 = a; v0 = v[0]; i1 = pad; v1 = 0; }
                } else {                          /* two entries, ascending */
                    i0 = idx[0]; v0 = v[0]; i1 = idx[1]; v1 = v[1];
                }
                const int64_t j = g * nw + w;     /* window index in the row */
                vals[r * (Kl / 2) + 2 * j + 0] = v0;
                vals[r * (Kl / 2) + 2 * j + 1] = v1;
                nib[r * (Kl / 4) + j] = (uint8_t)(i0 | (i1 << 2));
            }
        }
    }
    return failed ? -1 : 0;
}

/* Inverse of or_compress in the lifted coordinates: dense_lifted[r][k'] gets
 * the value of slot s at lifted position 4j + i_s, zero elsewhere (fp64). */
void or_expand_lifted(const uint16_t *vals, const uint8_t *nib, int64_t rows,
                      int64_t Kl, double *dense_lifted) {
    const int64_t nwin = Kl / 4;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < Kl; ++k) dense_lifted[r * Kl + k] = 0.0;
        for (int64_t j = 0; j < nwin; ++j) {
            uint8_t q = nib[r * nwin + j];
            int i0 = q & 3, i1 = (q >> 2) & 3;
            dense_lifted[r * Kl + 4 * j + i0] += bf16_bits_to_double(vals[r * (Kl / 2) + 2 * j]);
            dense_lifted[r * Kl + 4 * j + i1] += bf16_bits_to_double(vals[r * (Kl / 2) + 2 * j + 1]);
        }
    }
}

/* Maps the compressed row back to the original K coordinates: each value goes
 * to source column g*2n + 2w + i (the inverse of the lift map).  out[r][k] is
 * the bf16 bit pattern (0 where nothing was stored). */
void or_decompress(const uint16_t *vals, const uint8_t *nib, int64_t rows,
                   int64_t K, int M, uint16_t *out) {
    const int64_t Kl = or_lifted_k(K, M);
    const int n = M / 2, nw = n - 1;
    const int64_t groups = K / M;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < K; ++k) out[r * K + k] = 0;
        for (int64_t g = 0; g < groups; ++g)
            for (int w = 0; w < nw; ++w) {
                const int64_t j = g * nw + w;
                uint8_t q = nib[r * (Kl / 4) + j];
                int ii[2] = {q & 3, (q >> 2) & 3};
                for (int s = 0; s < 2; ++s) {
                    uint16_t v = vals[r * (Kl / 2) + 2 * j + s];
                    /* +0.0 is what padded slots hold; skipping it never loses
                     * a kept value (the output starts at +0.0), and a padded
                     * index may point at a position another window owns. */
                    if (v == 0) continue;
                    out[r * K + g * M + 2 * w + ii[s]] = v;
                }
            }
    }
}

/* ------------------------------------------------------ hardware metadata */

/* Step 4.  Sparse-MMA metadata image for 16-bit operands.  The nibble stream
 * of each row is cut into blocks of 128 rows x 32 windows (= 128 lifted K
 * positions, four MMAs of K = 32).  A block is 128 lanes x 16 bytes, one
 * 32-bit word per MMA.  Row m of the block and window j of the block
 * (c = j / 8, q = j % 8) land in
 *     lane   = (m % 8) + 8 * (q / 4) + 16 * (m / 16)
 *     word   = c            (byte offset lane*16 + 4*c)
 *     nibble = (q % 4) + 4 * ((m / 8) % 2)   (bits 4*nibble .. 4*nibble+3)
 * Blocks are stored row-block major: block (rb, kb) at byte
 * (rb * KB + kb) * 2048 with KB = ceil(K'/128).  Rows past `rows` and windows
 * past K'/4 are padded with the nibble 0x4 (indices 0 and 1). */
int64_t or_meta_hw_bytes(int64_t rows, int64_t Kl) {
    const int64_t RB = (rows + 127) / 128, KB = (Kl + 127) / 128;
    return RB * KB * 2048;
}

void or_meta_hw(const uint8_t *nib, int64_t rows, int64_t Kl, uint8_t *meta) {
    const int64_t RB = (rows + 127) / 128, KB = (Kl + 127) / 128;
    const int64_t nwin = Kl / 4;
    memset(meta, 0, (size_t)(RB * KB * 2048));
    for (int64_t rb = 0; rb < RB; ++rb)
        for (int64_t kb = 0; kb < KB; ++kb)
            for (int m = 0; m < 128; ++m)
                for (int jj = 0; jj < 32; ++jj) {
                    const int64_t r = rb * 128 + m, j = kb * 32 + jj;
                    uint8_t q = 0x4;
                    if (r < rows && j < nwin) q = nib[r * nwin + j];
                    const int c = jj / 8, g = jj % 8;
                    const int lane = (m % 8) + 8 * (g / 4) + 16 * (m / 16);
                    const int nb = (g % 4) + 4 * ((m / 8) % 2);
                    const int64_t byte = (rb * KB + kb) * 2048 + lane * 16 + c * 4 + nb / 2;
                    meta[byte] |= (uint8_t)((q & 0xF) << (4 * (nb % 2)));
                }
}

/* ------------------------------------------------------------------- lift */

/* Step 5.  dst[r][g*4(n-1) + 4w + j] = src[r][g*2n + 2w + j] (bf16 bits; an
 * fp32 source is rounded to bf16 nearest-even).  For M == 4 it is a copy. */
int or_lift(const void *src, int dt, int64_t rows, int64_t K, int M, uint16_t *dst) {
    const int64_t Kl = or_lifted_k(K, M);
    if (Kl < 0) return -1;
    const int n = M / 2, nw = n - 1;
    const int64_t groups = K / M;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t g = 0; g < groups; ++g)
            for (int w = 0; w < nw; ++w)
                for (int j = 0; j < 4; ++j)
                    dst[r * Kl + g * 4 * nw + 4 * w + j] =
                        bf16_at(src, dt, r * K + g * M + 2 * w + j);
    return 0;
}

/* ----------------------------------------------------------------- linear */

/* Widen a bf16 / fp32 matrix to fp64, optionally multiplying by a keep mask. */
void or_to_f64(const void *src, int dt, int64_t count, const uint8_t *keep, double *dst) {
    for (int64_t i = 0; i < count; ++i)
        dst[i] = (keep && !keep[i]) ? 0.0 : value_at(src, dt, i);
}

/* Step 6.  Y[t][o] = sum_{k ascending} A[t][k] * B[o][k] in fp64.  When
 * rows_sel is not NULL only the listed rows t are computed, and they are
 * written densely: Y[i][o] for t = rows_sel[i]. */
void or_linear_f64(const double *A, const double *B, int64_t T, int64_t O, int64_t K,
                   const int64_t *rows_sel, int64_t nsel, double *Y) {
    const int64_t nrow = rows_sel ? nsel : T;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nrow; ++i) {
        const int64_t t = rows_sel ? rows_sel[i] : i;
        const double *a = A + t * K;
        for (int64_t o = 0; o < O; ++o) {
            const double *b = B + o * K;
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k) s += a[k] * b[k];
            Y[i * O + o] = s;
        }
    }
}

/* ----------------------------------------------------------------- hybrid */

/* Step 7a.  colnorm[c] = sum_{r ascending} w[r][c]^2 in fp64. */
void or_colnorm_f64(const void *w, int dt, int64_t O, int64_t K, double *colnorm) {
    for (int64_t c = 0; c < K; ++c) colnorm[c] = 0.0;
    for (int64_t r = 0; r < O; ++r)
        for (int64_t c = 0; c < K; ++c) {
            double v = value_at(w, dt, r * K + c);
            colnorm[c] += v * v;
        }
}

/* Step 7'a.  rownorm[r] = sum_{k ascending} w[r][k]^2 in fp64. */
void or_rownorm_f64(const void *w, int dt, int64_t O, int64_t K, double *rownorm) {
    for (int64_t r = 0; r < O; ++r) {
        double s = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const double v = value_at(w, dt, r * K + k);
            s += v * v;
        }
        rownorm[r] = s;
    }
}

/* Step 7'b.  silu(z) = z / (1 + e^-z), elementwise in fp64. */
void or_silu_f64(const double *z, int64_t n, double *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = z[i] / (1.0 + exp(-z[i]));
}

/* Number of dense columns for a dense share f of K: 4 * floor(f * K / 4), so
 * that the sparse remainder is a whole number of 2:4 groups. */
int64_t or_hybrid_dense_count(int64_t K, double dense_frac) {
    if (dense_frac <= 0.0) return 0;
    if (dense_frac >= 1.0) return K;
    return 4 * (int64_t)((dense_frac * (double)K) / 4.0);
}

/* Step 7b.  Column c is dense iff fewer than D columns beat it, where c'
 * beats c when colnorm[c'] > colnorm[c], or equal and c' < c.
 * perm = [sparse columns ascending | dense columns ascending]. */
void or_hybrid_perm(const double *colnorm, int64_t K, int64_t D, int32_t *perm,
                    uint8_t *is_dense) {
    for (int64_t c = 0; c < K; ++c) {
        int64_t beaten_by = 0;
        for (int64_t c2 = 0; c2 < K; ++c2)
            if (colnorm[c2] > colnorm[c] || (colnorm[c2] == colnorm[c] && c2 < c)) ++beaten_by;
        is_dense[c] = (uint8_t)(beaten_by < D ? 1 : 0);
    }
    int64_t s = 0, d = K - D;
    for (int64_t c = 0; c < K; ++c) {
        if (is_dense[c]) perm[d++] = (int32_t)c;
        else perm[s++] = (int32_t)c;
    }
}

/* Step 7c.  Gathers W by perm: wperm[r][i] = w[r][perm[i]] (bf16 bits). */
void or_gather_cols_bf16(const uint16_t *w, int64_t rows, int64_t K, const int32_t *perm,
                         uint16_t *wperm) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t i = 0; i < K; ++i) wperm[r * K + i] = w[r * K + perm[i]];
}

/* --------------------------------------------------------- fp8 (E4M3) */

/* Step 8.  E4M3 as the OCP 8-bit format defines it: 1 sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits; exponent field 0 holds the subnormals
 * (m/8) * 2^-6; the code S.1111.111 is NaN and there is no infinity, so the
 * largest finite magnitude is 1.75 * 2^8 = 448. */
double or_e4m3_to_f64(uint8_t c) {
    const int e = (c >> 3) & 0xF, m = c & 7;
    if (e == 0xF && m == 7) return NAN;
    const double v = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return (c & 0x80) ? -v : v;
}

/* The e4m3 code nearest to the fp32 value x, ties to the even code (the
 * code's last bit is the mantissa's last bit); magnitudes of 448 and above,
 * infinity included, saturate to 448; NaN gives 0x7F.  The positive codes
 * 0x00..0x7E increase with their value, so the two neighbours of |x| are
 * found by bisection.  The sign is kept, also for results that are zero. */
uint8_t or_e4m3_from_f32(float x) {
    if (isnan(x)) return 0x7F;
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    const double a = fabs((double)x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    int lo = 0, hi = 0x7E;                       /* value(lo) <= a < value(hi) */
    while (hi - lo > 1) {
        const int mid = (lo + hi) / 2;
        if (or_e4m3_to_f64((uint8_t)mid) <= a) lo = mid;
        else hi = mid;
    }
    const double dlo = a - or_e4m3_to_f64((uint8_t)lo), dhi = or_e4m3_to_f64((uint8_t)hi) - a;
    const int c = dlo < dhi ? lo : (dhi < dlo ? hi : (lo % 2 == 0 ? lo : hi));
    return (uint8_t)(sign | c);
}

static float value_f32_at(const void *src, int dt, int64_t idx) {
    return (float)value_at(src, dt, idx);         /* exact: bf16 and fp32 are fp32 values */
}

/* Step 8a.  Per-row (per-token) quantisation.  amax = max_k |x[r][k]|,
 * scale = amax / 448 rounded to fp32 (1 for an all-zero row), inv = 1 / scale
 * rounded to fp32, and code = e4m3(x * inv) with the product rounded to fp32:
 * the quantised code is decided from the same fp32 product the kernel forms.
 * The pages say only that activations are quantised per token; a symmetric
 * scale that maps the row maximum to the largest code, applied through its
 * reciprocal, is the plainest reading. */
void or_quant_rows_e4m3(const void *src, int dt, int64_t rows, int64_t K, uint8_t *codes, float *scale) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            const float v = fabsf(value_f32_at(src, dt, r * K + k));
            if (v > amax) amax = v;
        }
        const float s = amax > 0.0f ? amax / 448.0f : 1.0f;
        const float inv = 1.0f / s;
        scale[r] = s;
        for (int64_t k = 0; k < K; ++k) codes[r * K + k] = or_e4m3_from_f32(value_f32_at(src, dt, r * K + k) * inv);
    }
}

/* Step 8b.  Codes of a row's compressed values (bf16 bits) with that row's
 * scale: code = e4m3(v * (1 / scale[r])), reciprocal and product rounded to
 * fp32 as in step 8a.  Padded slots (+0.0) give the code 0x00. */
void or_quant_vals_e4m3(const uint16_t *vals, int64_t rows, int64_t nv, const float *scale, uint8_t *codes) {
    for (int64_t r = 0; r < rows; ++r) {
        const float inv = 1.0f / scale[r];
        for (int64_t i = 0; i < nv; ++i)
            codes[r * nv + i] = or_e4m3_from_f32((float)bf16_bits_to_double(vals[r * nv + i]) * inv);
    }
}

/* Step 5 on bytes: dst[r][g*4(n-1) + 4w + j] = src[r][g*2n + 2w + j]. */
int or_lift_u8(const uint8_t *src, int64_t rows, int64_t K, int M, uint8_t *dst) {
    const int64_t Kl = or_lifted_k(K, M);
    if (Kl < 0) return -1;
    const int n = M / 2, nw = n - 1;
    const int64_t groups = K / M;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t g = 0; g < groups; ++g)
            for (int w = 0; w < nw; ++w)
                for (int j = 0; j < 4; ++j)
                    dst[r * Kl + g * 4 * nw + 4 * w + j] = src[r * K + g * M + 2 * w + j];
    return 0;
}

/* Step 8c.  The 8-bit sparse MMA reads its metadata as one 16-byte row per
 * operand row and 128 lifted K: in the block of rows 128 rb .. 128 rb + 127
 * and windows 32 kb .. 32 kb + 31, row m and window j of the block land in
 * byte m * 16 + j / 2, low nibble for even j.  Blocks are placed as in step 4
 * (block (rb, kb) at byte (rb * KB + kb) * 2048) and padded the same way. */
void or_meta8(const uint8_t *nib, int64_t rows, int64_t Kl, uint8_t *meta) {
    const int64_t RB = (rows + 127) / 128, KB = (Kl + 127) / 128;
    const int64_t nwin = Kl / 4;
    memset(meta, 0, (size_t)(RB * KB * 2048));
    for (int64_t rb = 0; rb < RB; ++rb)
        for (int64_t kb = 0; kb < KB; ++kb)
            for (int m = 0; m < 128; ++m)
                for (int jj = 0; jj < 32; ++jj) {
                    const int64_t r = rb * 128 + m, j = kb * 32 + jj;
                    uint8_t q = 0x4;
                    if (r < rows && j < nwin) q = nib[r * nwin + j];
                    meta[(rb * KB + kb) * 2048 + m * 16 + jj / 2] |= (uint8_t)((q & 0xF) << (4 * (jj % 2)));
                }
}

/* ------------------------------------------------- shift and variance */

/* Step 9a (D-PTS).  The page names a dynamic per-token shift that centres the
 * activations on zero and gives no formula; the plainest reading is the
 * token's mean: mu[r] = (sum_{k ascending} x[r][k]) / K in fp64, and the
 * shift the kernels apply is that mean rounded to fp32.  For bf16 inputs whose
 * magnitudes span fewer than 53 - 8 - log2(K) binades every partial sum is
 * exact, so the mean does not depend on the order of summation. */
void or_row_mean(const void *src, int dt, int64_t rows, int64_t K, double *mu64, float *mu32) {
    for (int64_t r = 0; r < rows; ++r) {
        double s = 0.0;
        for (int64_t k = 0; k < K; ++k) s += value_at(src, dt, r * K + k);
        mu64[r] = s / (double)K;
        mu32[r] = (float)mu64[r];
    }
}

/* Step 9b.  The shifted token, stored in the compute format:
 * xs[r][k] = bf16(fl32(x[r][k] - mu32[r])), the difference rounded to fp32,
 * then to bf16 (nearest-even both times).  The prune of step 1 runs on xs. */
void or_shift_bf16(const void *src, int dt, int64_t rows, int64_t K, const float *mu32, uint16_t *xs) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k) {
            const float d = value_f32_at(src, dt, r * K + k) - mu32[r];
            uint32_t u;
            memcpy(&u, &d, 4);
            xs[r * K + k] = f32_bits_to_bf16_rne(u);
        }
}

/* Step 9c (VAR).  The page names a per-token variance correction after
 * pruning and gives no formula; the plainest reading that keeps the pattern
 * sparse is one factor per token on the survivors, chosen so that the pruned
 * token gets back the variance of the dense token:
 * alpha[r] = sqrt(var(x[r]) / var(v[r] * keep[r])), where x is the token as
 * it came in, v the token the prune ran on (x itself, or the shifted token of
 * step 9b -- the variance does not change under a shift),
 * var(u) = (1/K) sum u^2 - ((1/K) sum u)^2 over all K entries (pruned ones as
 * zeros), sums in fp64, k ascending; alpha = 1 when the pruned token has no
 * variance. */
void or_var_scale(const void *x_in, int dt, const uint16_t *v, const uint8_t *keep, int64_t rows, int64_t K,
                  double *alpha) {
    for (int64_t r = 0; r < rows; ++r) {
        double s = 0.0, q = 0.0, sp = 0.0, qp = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const double x = value_at(x_in, dt, r * K + k);
            s += x;
            q += x * x;
            if (keep[r * K + k]) {
                const double y = bf16_bits_to_double(v[r * K + k]);
                sp += y;
                qp += y * y;
            }
        }
        const double mi = s / (double)K, mp = sp / (double)K;
        const double var_in = q / (double)K - mi * mi;
        const double var_p = qp / (double)K - mp * mp;
        alpha[r] = var_p > 0.0 ? sqrt(var_in / var_p) : 1.0;
    }
}

/* Step 9d.  Row sums of the weight, s[o] = sum_{k ascending} w[o][k] in fp64:
 * the shift mu enters the product as mu * s[o]. */
void or_rowsum_f64(const void *w, int dt, int64_t O, int64_t K, double *s) {
    for (int64_t o = 0; o < O; ++o) {
        double a = 0.0;
        for (int64_t k = 0; k < K; ++k) a += value_at(w, dt, o * K + k);
        s[o] = a;
    }
}

/* ---------------------------------------------------------------- version */

int or_abi_version(void) { return 1; }
