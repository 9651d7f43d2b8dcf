/*
 * hq_oracle.h -- plain fp64 CPU restatement of the HadaNorm Hadamard-domain
 * quantized linear layer.  TEST INFRASTRUCTURE ONLY: the tests, the smoke
 * check and the CPU-baseline leg of the benchmark may call it; the product
 * library never does.  It shares no source with the CUDA path.
 *
 * Sources (page title, section / equation):
 *   - "HadaNorm: Diffusion Transformer Quantization through Mean-Centered
 *     Transformations" (pith.science review), "What carries the argument":
 *     Eq. (1) XW+b = X~W~+b~ with X~ = X diag(sigma^-1) H - mu,
 *     W~ = H^T diag(sigma) W, b~ = b + mu W~, and Eq. (3)
 *     sigma_i = max|X_i|^alpha / max|W_i|^(1-alpha).
 *   - "Hadamard-Domain Model Quantization for Learned Image Coding" (HaTQ),
 *     Sec. III-A Eq. (3) (symmetric quantizer), Sec. III-C Eq. (7)-(8)
 *     (normalized Hadamard), Sec. IV-B Eq. (13)-(14), (18) (double-Hadamard
 *     product, accumulator scale), Supplement VII-A Eq. (34) (Sylvester).
 *   - "Data-free 4-bit quantization for diffusion transformers",
 *     "Hadamard rotation: the int4 improvement", step 7 (block-diagonal H).
 *
 * Conventions: bf16 values are passed as their 16-bit patterns (uint16_t).
 * Matrices are row-major.  X is [T,K] (tokens x channels), W is [N,K]
 * (output channels x input channels, so the math-convention weight of the
 * pages is W^T).  Every function returns 0 on success, -1 on a bad argument.
 */
#ifndef HQ_ORACLE_H
#define HQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Unnormalized Sylvester-order Hadamard entry (-1)^popcount(j & k). */
int hqo_hadamard_entry(int64_t j, int64_t k);

/* Builds the unnormalized Sylvester matrix of order n (a power of two) by the
 * doubling recursion H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]] into
 * out[n*n] (row-major, entries +-1). */
int hqo_sylvester(int64_t n, int8_t* out);

/* Exact bf16 -> double, and double -> bf16 with round-half-to-even. */
double hqo_bf16_to_f64(uint16_t b);
uint16_t hqo_f64_to_bf16(double x);

/* Round half to even on doubles. */
double hqo_rne(double x);

/* out[c] = max_r |M[r,c]| for a bf16 matrix M[R,C]. */
int hqo_col_absmax(const uint16_t* M, int64_t R, int64_t C, double* out);

/* out[c] = (1/R) sum_r M[r,c] for a bf16 matrix M[R,C] (R > 0): the
 * per-channel mean over tokens of the appended-token centring. */
int hqo_channel_mean(const uint16_t* M, int64_t R, int64_t C, double* out);

/* sigma_k = amax_x[k]^alpha / amax_w[k]^(1-alpha); sigma_k = 1 when either
 * maximum is zero. */
int hqo_sigma(int64_t K, const double* amax_x, const double* amax_w,
              double alpha, double* sigma);

/* Activation side of the layer for the rows listed in `rows` (all T rows when
 * rows == NULL, then nrows must equal T):
 *   Y = X diag(sigma^-1)
 *   centering 0: V = Y H                       (dense block-diagonal H of order n)
 *   centering 1: Z = Y H, m_t = mean_k Z[t,k], V = Z - m      (HadaNorm's mu
 *                after the rotation; reported mean m_t)
 *   centering 2: mu_t = mean_k Y[t,k], V = (Y - mu_t) H       (the mean removed
 *                before the rotation; reported mean mu_t)
 *   shift (any centering; NULL = none): a per-channel vector removed from Y
 *                before everything above, Y[t,k] -= shift[k] (the per-channel
 *                mean over tokens, in Y's units: the appended-token reading
 *                of the HadaNorm review's mu in R^d; its product with the
 *                weights goes into the bias, see hqo_prepare_weights)
 *   per token  (gran 0): s_t = max_k |V[t,k]| / q
 *   per tensor (gran 1): s   = max_{t,k} |V[t,k]| / q   over ALL T rows
 *   static     (gran 2): s   = static_scale
 *   code = clamp(rne(V / s), -q, q), q = 2^(bits-1) - 1; s = 0 gives code 0.
 * Outputs per listed row i: codes[i*K+k], scale[i], mean[i]; optional
 * tie[i*K+k] = | |V/s| - floor(|V/s|) - 1/2 | (distance of the scaled value
 * from a rounding tie, in code units; 0.5 when s = 0) and Z[i*K+k]. */
int hqo_quantize_act(int64_t K, int64_t n, int bits, int gran, int centering,
                     const uint16_t* X, int64_t T, const double* sigma,
                     const double* shift, double static_scale, const int64_t* rows, int64_t nrows,
                     int8_t* codes, double* scale, double* mean, double* tie,
                     double* Z, int nthreads);

/* Weight side:  W~[n,k] = sum_j H[j,k] sigma_j W[n,j]  (W~ = H^T diag(sigma) W
 * in the pages' orientation), colsum[n] = sum_k W~[n,k] (the correction of
 * centering 1), corr_pre[n] = sum_k sigma_k W[n,k] (the correction of
 * centering 2; optional output),
 * w_scale[n] = max_k |W~[n,k]| / q, w_codes = clamp(rne(W~ / w_scale), -q, q),
 * bias_out[n] = b[n] (0 when bias == NULL) + sum_k shift_k sigma_k W[n,k]
 * (the appended token's contribution, shift == NULL: none).  sigma == NULL
 * means sigma = 1.
 * Optional outputs: tie[N*K] and Wt[N*K] (the unquantized W~). */
int hqo_prepare_weights(int64_t K, int64_t N, int64_t n, int bits,
                        const uint16_t* W, const uint16_t* bias,
                        const double* sigma, const double* shift, int8_t* w_codes, double* w_scale,
                        double* colsum, double* corr_pre, double* bias_out,
                        double* tie, double* Wt, int nthreads);

/* acc[i*N+c] = sum_k A[rows[i],k] * B[c,k] in 64-bit integers, for int8
 * matrices A[M,K] and B[N,K] (rows == NULL: all M rows, nrows == M). */
int hqo_gemm_acc(const int8_t* A, const int8_t* B, int64_t M, int64_t N,
                 int64_t K, const int64_t* rows, int64_t nrows, int64_t* acc,
                 int nthreads);

/* y[i*N+c] = sx[i] * sw[c] * acc[i*N+c] + b[c] + m[i] * colsum[c]  (fp64), and
 * y_bf16 its bf16 rounding (either output may be NULL).  sx and m are per
 * listed row; m == NULL means m = 0; b == NULL means b = 0. */
int hqo_epilogue(const int64_t* acc, int64_t nrows, int64_t N,
                 const double* sx, const double* m, const double* sw,
                 const double* b, const double* colsum, double* y,
                 uint16_t* y_bf16);

/* Unquantized reference y[i*N+c] = sum_k X[rows[i],k] W[c,k] + b[c] (fp64). */
int hqo_exact_linear(const uint16_t* X, const uint16_t* W, const uint16_t* bias,
                     int64_t T, int64_t K, int64_t N, const int64_t* rows,
                     int64_t nrows, double* y, int nthreads);

/* Weight-only Hadamard (WH) form, HaTQ Sec. IV-B Eq. (15)-(17) and
 * supplement Eq. (40)-(41): the weights are rotated along the output
 * channels instead of the input channels.  H_out is block diagonal with
 * normalized Sylvester blocks of order n_out along N.
 *   Wbar[c,k] = sum_j H_out[c,j] sigma_k W[j,k]   (Wbar = H_out W diag(sigma))
 *   b_bar     = b H_out
 *   w_scale[c] = max_k |Wbar[c,k]| / q,  w_codes = clamp(rne(Wbar / w_scale), +-q)
 * sigma == NULL means sigma = 1; bias == NULL means b = 0.  tie (distance of
 * each |Wbar / w_scale| from a rounding tie) and Wbar may be NULL. */
int hqo_prepare_weights_wh(int64_t K, int64_t N, int64_t n_out, int bits,
                           const uint16_t* W, const uint16_t* bias,
                           const double* sigma, int8_t* w_codes, double* w_scale,
                           double* b_bar, double* tie, double* Wbar, int nthreads);

/* The WH output side (Eq. (41)): A[i,j] = sx[i] * sw[j] * acc[i*N+j] + b_bar[j],
 * then y[i,c] = sum_j A[i,j] H_out[j,c] (back to the original output basis),
 * and y_bf16 its bf16 rounding (either output may be NULL; b_bar may be NULL). */
int hqo_epilogue_wh(const int64_t* acc, int64_t nrows, int64_t N, int64_t n_out,
                    const double* sx, const double* sw, const double* b_bar,
                    double* y, uint16_t* y_bf16);

/* out[i,c] = sum_j M[i,j] H_out[j,c] for an fp64 matrix M [rows, N]: the WH
 * output-basis restoration alone. */
int hqo_output_rotation(const double* M, int64_t rows, int64_t N, int64_t n_out,
                        double* out);

/* Group-wise form with a low-rank branch ("Data-free 4-bit quantization for
 * diffusion transformers", "Hadamard rotation: the int4 improvement", steps
 * 1-7), in the [N,K] orientation (y[t,n] = sum_k W[n,k] X[t,k] + b[n]):
 *   smoothing   x^ = X diag(sigma^-1),  W^ = W diag(sigma)          (step 2)
 *   low rank    W^ = L2 L1 + R; the factors are kept in 16 bits: l2 =
 *               bf16(L2), and the down factor with the smoothing folded in,
 *               l1 = bf16(L1 diag(sigma^-1)), so that L1 x^ is computed as
 *               l1 X; R is what the 16-bit branch leaves,
 *               R = W^ - l2 l1 diag(sigma)                           (step 3)
 *   rotation    H = diag(H_g, ..., H_g) (normalized Sylvester, one block per
 *               quantization group of g channels): R H and x^ H       (5-7)
 *   quantizers  per output channel and group of R H, per token and group of
 *               x^ H: s = max |.| / q over the group's g values, codes =
 *               clamp(rne(. / s), +-q)                                (4, 6)
 *   output      y = sum_groups s_x s_w (codes . codes) + l2 bf16(l1 X) + b
 * The caller supplies the rank-r factors L1 [rank,K] and L2 [N,rank] (fp64),
 * e.g. from a singular value decomposition of W^; the method fixes only
 * their product. */
int hqo_gw_prepare_weights(int64_t K, int64_t N, int64_t g, int bits, int64_t rank,
                           const uint16_t* W, const uint16_t* bias, const double* sigma,
                           const double* L1, const double* L2, uint16_t* l1s, uint16_t* l2b,
                           int8_t* w_codes, double* w_gscale, double* bias_out, double* tie,
                           double* Rh, int nthreads);
/* Activations for the listed rows: codes [nrows,K], gscale [nrows,K/g]
 * (per token and group), u [nrows,rank] = bf16(l1 X) (the 16-bit branch's
 * down projection, fp64 sums); optional tie and Z (x^ H) [nrows,K]. */
int hqo_gw_quantize_act(int64_t K, int64_t g, int bits, int64_t rank, const uint16_t* X,
                        int64_t T, const double* sigma, const uint16_t* l1s, const int64_t* rows,
                        int64_t nrows, int8_t* codes, double* gscale, uint16_t* u, double* tie,
                        double* Z, int nthreads);
/* y[i,n] = sum_j ascale[i,j] wscale[n,j] sum_{k in group j} A[i,k] B[n,k]
 *          + sum_r u[i,r] l2b[n,r] + b[n]   (fp64; the integer sums exact),
 * and its bf16 rounding (either output may be NULL; b may be NULL). */
int hqo_gw_epilogue(const int8_t* A, const int8_t* B, int64_t nrows, int64_t N, int64_t K,
                    int64_t g, const double* ascale, const double* wscale, const uint16_t* u,
                    const uint16_t* l2b, int64_t rank, const double* b, double* y,
                    uint16_t* y_bf16, int nthreads);

/* Packed storage of 3- and 4-bit codes, two per byte.  The blog "Data-free
 * 4-bit quantization for diffusion transformers" ("Hadamard rotation: the int4
 * improvement") runs a W4A4 GEMM on 4-bit operands but fixes no storage
 * layout; the reading taken here: element 2j of a row in the
 * low nibble of byte j, element 2j+1 in the high nibble, each as a 4-bit
 * two's-complement value.  count is the number of codes (even); every code
 * must lie in [-8, 7] (hqo_pack_i4 returns -1 otherwise). */
int hqo_pack_i4(const int8_t* codes, int64_t count, uint8_t* out);
/* The inverse: count codes from count / 2 bytes, nibble v read as v - 16 when
 * v >= 8. */
int hqo_unpack_i4(const uint8_t* packed, int64_t count, int8_t* codes);

#ifdef __cplusplus
}
#endif

#endif /* HQ_ORACLE_H */
