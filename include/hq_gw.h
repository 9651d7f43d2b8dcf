/* hq_gw.h -- C ABI of the group-wise 4-bit linear layer with a 16-bit
 * low-rank branch.
 *
 * Source: the blog "Data-free 4-bit quantization for diffusion transformers",
 * section "Hadamard rotation: the int4 improvement", math steps 1-7.  In the
 * [N,K] orientation used throughout this library (y[t,n] = sum_k W[n,k]
 * X[t,k] + b[n]) the layer computes
 *
 *   smoothing   x^ = X diag(sigma^-1),  W^ = W diag(sigma)            (step 2)
 *   low rank    W^ = L2 L1 + R: the rank-r factors are kept in 16 bits,
 *               l2 = bf16(L2) [N,r] and l1 = bf16(L1 diag(sigma^-1)) [r,K]
 *               (the smoothing folded in, so L1 x^ is computed as l1 X), and
 *               R = (W - l2 l1) diag(sigma) is what they leave        (step 3)
 *   rotation    one normalized Sylvester block H_64 per group of 64 input
 *               channels: R H and x^ H                                (5-7)
 *   quantizers  one scale per output channel and group of R H, and per
 *               token and group of x^ H: s = max|.| / q, codes =
 *               clamp(rne(. / s), +-q), q = 2^(bits-1) - 1             (4, 6)
 *   output      Y[t,n] = bf16( sum_j s_x[t,j] s_w[n,j] sum_{k in group j}
 *                                 A[t,k] B[n,k]
 *                              + sum_r u[t,r] l2[n,r] + b[n] ),
 *               u = bf16(l1 X)  (the 16-bit branch's down projection).
 *
 * The method fixes only the product L2 L1 (the pages take it from a singular
 * value decomposition of W^); the caller computes the factors and passes
 * them in, with sigma_inv from hq_gw_sigma_inv.
 *
 * Storage.  Codes are bytes in the fp8 e4m3 encoding, which holds every
 * integer code of magnitude <= 7 exactly; the tensor cores multiply them
 * (tcgen05 kind::f8f6f4) into fp32 accumulators, one accumulator per group,
 * and every group's integer sum (at most 64 * 7 * 7 in magnitude) is exact.
 * Activation scales are laid out group-major: a_scale[j * ld + t] with
 * ld = hq_gw_scale_ld(T); weight scales w_scale[j * N + n].
 *
 * Shapes supported: group 64; K a multiple of 64, at most 16384; N a multiple
 * of 16; rank 0 (no branch) or 32; a_bits and w_bits in 2..4.  Every device
 * pointer is 16-byte aligned (bias: 4-byte).  All pointers are caller-owned
 * device memory; T = 0 is a no-op (the pointers are still checked).  Errors:
 * HQ_ERR_INVALID_ARGUMENT for a null pointer, a negative size or alpha
 * outside [0, 1], HQ_ERR_MISALIGNED for a misaligned pointer,
 * HQ_ERR_UNSUPPORTED for a shape outside the list above, HQ_ERR_CUDA for a
 * failed launch; a kernel that gave up waiting records HQ_ERR_TIMEOUT for
 * hq_check_device_error.  Argument checks precede any launch. */
#ifndef HQ_GW_H_
#define HQ_GW_H_

#include <stddef.h>
#include <stdint.h>

#include "hq.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct hq_gw_desc {
  int32_t K;      /* input channels */
  int32_t N;      /* output channels */
  int32_t group;  /* channels per quantization group = order of the H block (64) */
  int32_t rank;   /* rank of the 16-bit branch (0 or 32) */
  int32_t a_bits; /* activation code width */
  int32_t w_bits; /* weight code width */
} hq_gw_desc;

/* Leading dimension (elements) of an activation scale array for T tokens:
 * T rounded up to a multiple of 4, so every group's row starts on a 16-byte
 * boundary.  a_scale holds (K / 64) * hq_gw_scale_ld(T) floats. */
int64_t hq_gw_scale_ld(int64_t T);

/* hq_gw_sigma_inv -- the smoothing factors (HadaNorm review Eq. (3), as in
 * hq_prepare_weights): sigma_k = act_absmax[k]^alpha / max_n|W[n,k]|^(1-alpha),
 * 1 when act_absmax is NULL or either maximum is 0; sigma_inv = 1 / sigma.
 * W bf16 [N,K]; act_absmax fp32 [K] or NULL; sigma_inv fp32 [K] (output, also
 * scratch during the call).  alpha in [0, 1]. */
hq_status hq_gw_sigma_inv(const hq_gw_desc* desc, const uint16_t* W, const float* act_absmax,
                          float alpha, float* sigma_inv, hq_stream_t stream);

/* hq_gw_prepare_weights -- offline weight side (steps 2-5):
 * Inputs:  W bf16 [N,K]; bias bf16 [N] or NULL; sigma_inv fp32 [K] or NULL
 *          (sigma = 1); L1 fp32 [rank,K] and L2 fp32 [N,rank], the factors of
 *          W diag(sigma) (ignored when rank = 0).
 * Outputs: w_codes e4m3 bytes [N,K]; w_scale fp32 [K/64][N];
 *          l1s bf16 [rank,K] = bf16(L1 diag(sigma_inv)) (fp64 product, one
 *          rounding); l2b bf16 [N,rank] = bf16(L2); bias_f32 fp32 [N]
 *          (0 without a bias).  l1s / l2b may be NULL when rank = 0.
 * R = (W - l2b l1s) / sigma_inv is formed in fp32 and transformed with the
 * unnormalized 64-point fast Walsh-Hadamard transform (1/8 folded into the
 * scale). */
hq_status hq_gw_prepare_weights(const hq_gw_desc* desc, const uint16_t* W, const uint16_t* bias,
                                const float* sigma_inv, const float* L1, const float* L2,
                                uint8_t* w_codes, float* w_scale, uint16_t* l1s, uint16_t* l2b,
                                float* bias_f32, hq_stream_t stream);

/* Bytes of device workspace that let hq_gw_quantize_act split a block of
 * 128 tokens over two CTAs when the blocks fill less than half the GPU
 * (0 when rank = 0, which needs none). */
size_t hq_gw_quantize_act_workspace_bytes(const hq_gw_desc* desc, int64_t T);

/* hq_gw_quantize_act -- runtime activation side, one pass over X (steps 2, 3,
 * 6, 7): per token t and group j, V = (X[t, group j] * sigma_inv) H~_64 and
 * a_scale[j * ld + t] = max|V| / (8 q), codes = rne(V q / max|V|); and, from
 * the same tiles of X on the tensor cores, u[t,:] = bf16(X[t,:] l1s^T) with
 * fp32 sums.
 * Inputs:  X bf16 [T,K]; sigma_inv fp32 [K] or NULL; l1s bf16 [rank,K]
 *          (from hq_gw_prepare_weights; NULL when rank = 0).
 * Outputs: a_codes e4m3 bytes [T,K]; a_scale fp32 [K/64][ld]; u bf16
 *          [T,rank] (NULL when rank = 0).  A group whose max is 0 gets scale
 *          0 and zero codes.
 * workspace: device, 16-byte aligned, >= hq_gw_quantize_act_workspace_bytes
 *   bytes, or NULL; contents need not be initialised.  When the blocks of 128
 *   tokens fill less than half the GPU, a workspace lets each block's groups
 *   be split over two CTAs, whose fp32 parts of u the one finishing last adds
 *   in a fixed order (deterministic; codes and scales are the same either
 *   way, u's fp32 sum is taken in two parts).  Without one, blocks stay
 *   whole. */
hq_status hq_gw_quantize_act(const hq_gw_desc* desc, const uint16_t* X, int64_t T,
                             const float* sigma_inv, const uint16_t* l1s, uint8_t* a_codes,
                             float* a_scale, uint16_t* u, void* workspace,
                             size_t workspace_bytes, hq_stream_t stream);

/* hq_gw_linear -- the output (step 4): the group-wise GEMM with the 16-bit
 * branch and the bias fused into its epilogue (the formula at the top).
 * Inputs:  a_codes, a_scale, u from hq_gw_quantize_act for T tokens;
 *          w_codes, w_scale, l2b, bias_f32 from hq_gw_prepare_weights
 *          (bias_f32 may be NULL: no bias).
 * Output:  Y bf16 [T,N], round to nearest even. */
hq_status hq_gw_linear(const hq_gw_desc* desc, int64_t T, const uint8_t* a_codes,
                       const float* a_scale, const uint16_t* u, const uint8_t* w_codes,
                       const float* w_scale, const uint16_t* l2b, const float* bias_f32,
                       uint16_t* Y, hq_stream_t stream);

/* hq_gw_debug_linear_f32 -- hq_gw_linear with the fp32 sums written to
 * Y32 fp32 [T,N] before any bf16 rounding (for exactness checks). */
hq_status hq_gw_debug_linear_f32(const hq_gw_desc* desc, int64_t T, const uint8_t* a_codes,
                                 const float* a_scale, const uint16_t* u, const uint8_t* w_codes,
                                 const float* w_scale, const uint16_t* l2b, const float* bias_f32,
                                 float* Y32, hq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HQ_GW_H_ */
