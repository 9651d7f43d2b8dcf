/*
 * hq.h -- C ABI of the B200 (sm_100a) Hadamard-domain quantized linear layer.
 *
 * The layer is the HadaNorm identity (HadaNorm review, "What carries the
 * argument", Eq. (1)):
 *
 *     X W + b = X~ W~ + b~,   X~ = X diag(sigma^-1) H - mu,
 *                             W~ = H^T diag(sigma) W,  b~ = b + mu W~,
 *
 * with sigma_i = max|X_i|^alpha / max|W_i|^(1-alpha) (same page, Eq. (3)),
 * mu the per-token mean of the scaled and rotated activations, and H a
 * block-diagonal Sylvester Hadamard matrix with blocks of order had_order
 * ("Data-free 4-bit quantization for diffusion transformers", "Hadamard
 * rotation", step 7; HaTQ supplement Eq. (34)).  X~ is quantized per token
 * (or per tensor) and W~ per output channel with the symmetric quantizer of
 * HaTQ Sec. III-A Eq. (3), round half to even, and the product runs as an
 * int8 x int8 -> int32 tensor-core GEMM whose accumulator has scale
 * s_x * s_w (HaTQ Sec. IV-B Eq. (18)).  HaTQ's weight-only Hadamard form
 * (Sec. IV-B Eq. (15)-(17)) is the same pipeline with X unrotated and W
 * rotated along the output channels (hq_layer_desc.out_order).
 *
 * Memory conventions (all entry points):
 *   - Every tensor pointer is a DEVICE pointer owned by the caller, except
 *     the host buffers of hq_forward_host.  The library never allocates,
 *     frees or retains device memory; it keeps one 4-byte device error word
 *     per device (see hq_check_device_error), and hq_forward_host creates two
 *     copy streams per device on its first call.
 *   - Matrices are row-major.  X is [T,K] (tokens x input channels; NHWC
 *     pixels for a 1x1 convolution), W is [N,K] (output x input channels, the
 *     nn.Linear orientation, i.e. the transpose of the pages' W), Y is [T,N].
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - Pointers to tensors read or written by the tensor-memory engine or by
 *     16-byte vector accesses must be 16-byte aligned (HQ_ERR_MISALIGNED).
 *   - All calls are asynchronous on `stream` (NULL = legacy default stream)
 *     and never synchronize, except hq_check_device_error; hq_forward_host
 *     forks onto its copy streams and joins back into `stream`.
 *   - Errors are returned, never raised: the library does not abort, exit or
 *     trap.  Argument checks happen before any launch; a rejected call
 *     launches nothing.
 *
 * Shapes supported:  had_order a power of two in [16, 1024], or 1 (no
 * rotation along K); K a multiple of had_order and of 16, K <= 15360 with a
 * rotation and K <= 10240 without one (K a multiple of 32 for packed
 * codes); N a multiple of 16 (and of out_order in the weight-only form,
 * out_order in {16, 32, 64}); T >= 0 (T = 0 is a no-op); a_bits in {3, 4, 8}, w_bits in
 * {4, 8} (codes in an int8 container, one code per byte; 3- and 4-bit
 * activation codes optionally two per byte, hq_layer_desc.code_format).
 */
#ifndef HQ_H
#define HQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Compatible with cudaStream_t (struct CUstream_st*). */
typedef struct CUstream_st* hq_stream_t;

typedef enum hq_status {
  HQ_OK = 0,
  HQ_ERR_INVALID_ARGUMENT = 1, /* null pointer, negative size, bad enum */
  HQ_ERR_UNSUPPORTED = 2,      /* shape / bit-width outside the list above */
  HQ_ERR_MISALIGNED = 3,       /* a tensor pointer is not 16-byte aligned */
  HQ_ERR_CUDA = 4,             /* a CUDA runtime call or launch failed */
  HQ_ERR_TIMEOUT = 5,          /* a bounded device-side wait gave up */
  HQ_ERR_DEVICE = 6            /* the device lacks sm_100a / tensor maps */
} hq_status;

enum { HQ_PER_TOKEN = 0, HQ_PER_TENSOR_DYNAMIC = 1, HQ_PER_TENSOR_STATIC = 2 };
enum { HQ_CENTER_NONE = 0, HQ_CENTER_TOKEN_MEAN = 1, HQ_CENTER_TOKEN_MEAN_PRE = 2 };
enum { HQ_CODES_I8 = 0, HQ_CODES_I4_PACKED = 1 };

/* Layer description, host memory, passed by const pointer.
 *   K, N        input / output channels.
 *   had_order   Hadamard block order n along K (H = diag(H_n, ..., H_n), K/n
 *               blocks): 16 .. 1024, or 1 for no input-side rotation (then
 *               centering must be HQ_CENTER_NONE).
 *   a_bits      activation code width: 4 (int4, [-7,7]), 3 (int3, [-3,3]) or
 *               8 (int8, [-127,127]); q_a = 2^(a_bits-1) - 1.
 *   w_bits      weight code width: 4 or 8; q_w = 2^(w_bits-1) - 1.
 *   act_gran    HQ_PER_TOKEN: one dynamic scale per token.
 *               HQ_PER_TENSOR_DYNAMIC: one scale from the whole tensor's
 *               max |X~| (two passes over X).
 *               HQ_PER_TENSOR_STATIC: one scale given by the caller.
 *   centering   HQ_CENTER_TOKEN_MEAN: mu_t = mean over all K channels of the
 *               scaled and rotated token, removed after the rotation
 *               (HadaNorm review, "What carries the argument", Eq. (1)).
 *               HQ_CENTER_TOKEN_MEAN_PRE: mu_t = mean over all K channels of
 *               the scaled token Y = X diag(sigma^-1), removed before the
 *               rotation: V = (Y - mu_t) H, i.e. Eq. (1)'s mu read as the
 *               vector mu_t 1^T H.  Only each block's first rotated channel
 *               changes (by -sqrt(n) mu_t); the layer's correction becomes
 *               mu_t * sum_k sigma_k W[n,k].
 *               HQ_CENTER_NONE: mu = 0.
 *   code_format HQ_CODES_I8: one signed activation code per byte, a_codes
 *               [T,K] int8.
 *               HQ_CODES_I4_PACKED (a_bits 3 or 4): two activation codes per
 *               byte, a_codes [T,K/2] bytes: element 2j of a row in the low
 *               nibble of byte j, element 2j+1 in the high nibble, each a
 *               4-bit two's-complement value.  hq_quantize_act writes this
 *               form and hq_linear reads it (the GEMM widens each tile to
 *               int8 in tensor memory, where the MMA takes its A operand).
 *               Weight codes stay one per byte.
 *   out_order   0 or 1: the double-Hadamard form above (no output-side
 *               transform).  16, 32 or 64: the weight-only Hadamard form
 *               (HaTQ Sec. IV-B, Eq. (15)-(17)): the weights are rotated
 *               along the output channels by H_out = diag(H_m, ..., H_m),
 *               m = out_order, and the output basis is restored after the
 *               integer GEMM; requires had_order == 1, centering
 *               HQ_CENTER_NONE and N % out_order == 0. */
typedef struct hq_layer_desc {
  int32_t K, N, had_order;
  int32_t a_bits, w_bits;
  int32_t act_gran;
  int32_t centering;
  int32_t code_format;
  int32_t out_order;
} hq_layer_desc;

/* Human-readable name of a status code (static string, never NULL). */
const char* hq_status_string(hq_status s);

/* Library version as 10000*major + 100*minor + patch. */
int hq_version(void);

/* hq_calib_act_absmax -- calibration reduction feeding sigma
 * (HadaNorm review Eq. (3), the max|X_i| term).
 *   X       bf16 [T,K] device, 16-byte aligned.
 *   absmax  fp32 [K] device: on return absmax[k] = max(absmax[k], max_t |X[t,k]|),
 *           so several batches can be accumulated; zero it before the first.
 * Only desc->K is used (any K that is a multiple of 8).  T = 0 is a no-op. */
hq_status hq_calib_act_absmax(const hq_layer_desc* desc, const uint16_t* X,
                              int64_t T, float* absmax, hq_stream_t stream);

/* hq_prepare_weights -- offline weight side of Eq. (1) (HadaNorm review):
 *   sigma_k   = act_absmax[k]^alpha / max_n|W[n,k]|^(1-alpha)   (Eq. (3));
 *               sigma_k = 1 when act_absmax == NULL or either max is zero
 *   sigma_inv = 1 / sigma  (fp32 [K]; feeds hq_quantize_act)
 *   W~[n,:]   = (W[n,:] * sigma) H    (W~ = H^T diag(sigma) W in the pages'
 *               orientation), computed with a fast Walsh-Hadamard transform
 *   colsum[n] = sum_k W~[n,k]          (the mu W~ term of b~), or, for
 *               HQ_CENTER_TOKEN_MEAN_PRE, sum_k sigma_k W[n,k]
 *   w_scale[n]= max_k |W~[n,k]| / q_w,  w_codes = clamp(rne(W~ / w_scale), +-q_w)
 *   bias_f32  = float(bias), or 0 when bias == NULL.
 * Inputs:  W bf16 [N,K], bias bf16 [N] or NULL, act_absmax fp32 [K] or NULL.
 * Weight-only Hadamard form (desc->out_order > 1; had_order is 1, so no
 * rotation along K):
 *   Wbar[n,:] = sum_j H_out[n,j] sigma W[j,:]   (Wbar = H_out W diag(sigma),
 *               HaTQ Eq. (15)-(17); j over n's block of out_order rows)
 *   w_scale[n]= max_k |Wbar[n,k]| / q_w,  w_codes = clamp(rne(Wbar / w_scale), +-q_w)
 *   colsum    = 0;  bias_f32 = float(bias) (added after the output basis is
 *               restored, which equals supplement Eq. (41)'s b_bar = b H_out
 *               added before it).
 * Outputs: w_codes int8 [N,K], w_scale fp32 [N], colsum fp32 [N],
 *          sigma_inv fp32 [K], bias_f32 fp32 [N] (all device, caller-owned).
 * sigma_inv is also used as scratch during the call.  alpha in [0, 1]. */
hq_status hq_prepare_weights(const hq_layer_desc* desc, const uint16_t* W,
                             const uint16_t* bias, const float* act_absmax,
                             float alpha, int8_t* w_codes, float* w_scale,
                             float* colsum, float* sigma_inv, float* bias_f32,
                             hq_stream_t stream);

/* Bytes of device workspace hq_quantize_act needs for this description
 * (16 for HQ_PER_TENSOR_DYNAMIC, 0 otherwise). */
size_t hq_quantize_act_workspace_bytes(const hq_layer_desc* desc, int64_t T);

/* hq_quantize_act -- runtime activation side of Eq. (1), fused in one pass
 * over X (two for HQ_PER_TENSOR_DYNAMIC):
 *   Y = X diag(sigma^-1); Z = Y H (block fast Walsh-Hadamard transform);
 *   HQ_CENTER_TOKEN_MEAN:     m_t = mean_k Z[t,k], V = Z - m;
 *   HQ_CENTER_TOKEN_MEAN_PRE: m_t = mean_k Y[t,k], V = (Y - m_t) H;
 *   HQ_CENTER_NONE:           m_t = 0, V = Z;
 *   s = max|V| / q_a per token (or per tensor);  codes = clamp(rne(V/s), +-q_a).
 * Inputs:  X bf16 [T,K]; sigma_inv fp32 [K] or NULL (sigma = 1).
 * Outputs: a_codes int8 [T,K], or [T,K/2] bytes of two codes each for
 *            HQ_CODES_I4_PACKED;
 *          a_scale fp32 [T] (HQ_PER_TOKEN) or [1] (per tensor; for
 *            HQ_PER_TENSOR_STATIC it is an INPUT holding s);
 *          a_mean fp32 [T] or NULL: m_t, in the units hq_linear multiplies
 *            by colsum (zeros when centering is off).
 * workspace: device, >= hq_quantize_act_workspace_bytes(), 16-byte aligned,
 *   contents need not be initialised (the call clears what it uses).
 * With had_order == 1 (no input-side rotation, as in the weight-only
 * Hadamard form) H is the identity and Z = Y.
 * A token whose max|V| is 0 gets scale 0 and all-zero codes. */
hq_status hq_quantize_act(const hq_layer_desc* desc, const uint16_t* X,
                          int64_t T, const float* sigma_inv, int8_t* a_codes,
                          float* a_scale, float* a_mean, void* workspace,
                          size_t workspace_bytes, hq_stream_t stream);

/* hq_linear -- integer GEMM and epilogue (HaTQ Eq. (18); HadaNorm Eq. (1)):
 *   acc[t,n] = sum_k a_codes[t,k] * w_codes[n,k]            (int32, exact)
 *   Y[t,n]   = bf16_rne( s_x[t] * w_scale[n] * acc[t,n]
 *                        + bias_f32[n] + a_mean[t] * colsum[n] )
 * on 5th-generation tensor cores (tcgen05 kind::i8, accumulator in TMEM).
 * Inputs:  a_codes int8 [T,K] (or [T,K/2] packed bytes, HQ_CODES_I4_PACKED:
 *          K a multiple of 32, a_bits <= 4; such A tiles enter the tensor
 *          cores as 16 * code and the accumulator is scaled back by 1/16,
 *          exactly), a_scale fp32 [T] or [1] (per tensor, selected
 *          by desc->act_gran), a_mean fp32 [T] or NULL (then mu = 0),
 *          w_codes int8 [N,K], w_scale fp32 [N], colsum fp32 [N] (may be NULL
 *          when a_mean is NULL), bias_f32 fp32 [N] or NULL (b = 0).
 * Outputs: Y bf16 [T,N]; acc_debug int32 [T,N] or NULL (the accumulators
 *          sum_k a_codes * w_codes, for bit-exact checks; costs an extra 4
 *          bytes per output).
 * Weight-only Hadamard form (desc->out_order = m > 1; a_mean and colsum
 * must be NULL): the accumulator is in the output Hadamard basis and the
 * epilogue restores the original basis (HaTQ Eq. (17), supplement Eq. (41)):
 *   Z[t,n]   = s_x[t] * w_scale[n] * acc[t,n]
 *   Y[t,:]   = bf16_rne( Z[t,:] H_out + bias_f32 ),  H_out = diag(H_m, ...)
 * with H_m the normalized Sylvester block, applied as an fp32 fast
 * Walsh-Hadamard transform over each group of m output columns.
 * acc_debug then holds the accumulators in the Hadamard basis.
 * Codes must lie within the declared widths: |a_codes| <= 2^(a_bits-1) and
 * |w_codes| <= 2^(w_bits-1) (a_bits, w_bits in [2, 8]; 8 admits every int8
 * value).  The epilogue converts accumulators exactly either way. */
hq_status hq_linear(const hq_layer_desc* desc, int64_t T, const int8_t* a_codes,
                    const float* a_scale, const float* a_mean,
                    const int8_t* w_codes, const float* w_scale,
                    const float* colsum, const float* bias_f32, uint16_t* Y,
                    int32_t* acc_debug, hq_stream_t stream);

/* hq_forward_host -- the layer end to end on host buffers:
 *   upload X_host -> X_dev, hq_quantize_act, hq_linear -> Y_dev, download
 *   Y_dev -> Y_host,
 * split into up to `chunks` row chunks (multiples of 128 rows) whose uploads,
 * kernels and downloads overlap: the uploads run back to back on a
 * library-owned upload stream, each chunk's two kernels run on `stream` as
 * soon as its upload has landed, and its download runs on a library-owned
 * download stream once its output is ready, so that both directions of the
 * host link are busy at once.  Results equal the four steps made one after
 * the other.  HQ_PER_TENSOR_DYNAMIC uses one chunk (its scale needs every
 * row).  Fork and join use events, so the call is ordered on `stream` and
 * may be captured in a CUDA graph; the first call on a device creates the two
 * streams, which live until the process exits (make it before any stream
 * capture).  X_host and Y_host should be page-locked (cudaHostAlloc or
 * pinned) for the copies to be asynchronous.
 * Arguments: X_host bf16 [T,K] and Y_host bf16 [T,N] (host); X_dev bf16 [T,K]
 * and Y_dev bf16 [T,N] (device staging, caller-owned); chunks in [1, 64];
 * the others as in hq_quantize_act and hq_linear (a_mean is passed on to the
 * GEMM only when desc->centering is not HQ_CENTER_NONE). */
hq_status hq_forward_host(const hq_layer_desc* desc, const uint16_t* X_host, int64_t T,
                          uint16_t* X_dev, const float* sigma_inv, int8_t* a_codes,
                          float* a_scale, float* a_mean, void* workspace,
                          size_t workspace_bytes, const int8_t* w_codes,
                          const float* w_scale, const float* colsum, const float* bias_f32,
                          uint16_t* Y_dev, uint16_t* Y_host, int chunks, hq_stream_t stream);

/* hq_quantize_act_noalloc -- hq_quantize_act without a caller workspace.
 * (The paper has no counterpart: this is a deployment convenience.)
 * For callers that cannot allocate device memory when they quantize -- a
 * runtime whose device memory is fixed at load time, a plugin or host
 * callback without an allocator, code where an allocation would be forbidden
 * or would synchronize.  Same arguments and results as hq_quantize_act, but
 * the per-tensor dynamic scale's workspace comes from a fixed device array of
 * 256 bytes that the library holds on every device that loads it, until the
 * process exits; the call itself allocates nothing.
 *   - Returns HQ_ERR_UNSUPPORTED if the description needs more workspace than
 *     the 256-byte array (hq_quantize_act_workspace_bytes > 256).
 *   - The first call made with a given device current looks up the array's
 *     device address; make that first call before any stream capture.
 *   - All calls share the array and it keeps the last call's contents; each
 *     call clears the bytes it uses before using them.  Calls whose kernels
 *     overlap on the GPU (unordered streams) race on the array. */
hq_status hq_quantize_act_noalloc(const hq_layer_desc* desc, const uint16_t* X,
                                  int64_t T, const float* sigma_inv, int8_t* a_codes,
                                  float* a_scale, float* a_mean, hq_stream_t stream);

/* hq_check_device_error -- synchronizes `stream`, then reads and clears the
 * current device's error word, which kernels set instead of trapping when a
 * bounded wait gives up (HQ_ERR_TIMEOUT).  Returns HQ_ERR_CUDA if the stream
 * itself reports an error. */
hq_status hq_check_device_error(hq_stream_t stream);

/* Test hook: sets the time in nanoseconds after which every bounded device
 * wait gives up (0 restores the default of 2 s).  Host state, applies to
 * launches issued after the call. */
hq_status hq_debug_set_wait_limit(uint64_t nanoseconds);

/* Test hook: which GEMM kernel hq_linear launches.  Host state, applies to
 * calls issued after it.
 *   HQ_GEMM_AUTO (0)        chosen per shape (default);
 *   HQ_GEMM_SINGLE_CTA (1)  one CTA per 128 x BN output tile (BN 64..256);
 *   HQ_GEMM_CTA_PAIR (2)    clusters of two CTAs per 256 x 256 output tile
 *                           (tcgen05 CTA-pair MMA); hq_linear returns
 *                           HQ_ERR_UNSUPPORTED if the device cannot hold
 *                           one such cluster.
 * Results are identical either way: the integer accumulators are exact and
 * the epilogue is the same code.  Returns HQ_ERR_INVALID_ARGUMENT for any
 * other value. */
enum { HQ_GEMM_AUTO = 0, HQ_GEMM_SINGLE_CTA = 1, HQ_GEMM_CTA_PAIR = 2 };
hq_status hq_debug_set_gemm_variant(int variant);

/* Test hook for the bounded-wait error path, without faulting the GPU:
 *   HQ_FAULT_NONE (0)                    normal operation;
 *   HQ_FAULT_QUANT_WITHHOLD_ROW (1)      in each CTA of the next activation
 *       quantize launches, one wait never completes: with a rotation along K
 *       (had_order >= 16, K <= 8192) the copy of the CTA's first tile of
 *       rows into shared memory is never issued, so its consumers' bounded
 *       wait for it expires; otherwise the statistics of the first row of
 *       the first tile are never released.  The kernel records
 *       HQ_ERR_TIMEOUT, waits for the copies it did issue and exits.
 * Host state, applies to launches issued after the call. */
enum { HQ_FAULT_NONE = 0, HQ_FAULT_QUANT_WITHHOLD_ROW = 1 };
hq_status hq_debug_inject_fault(int kind);

/* Test hook, host only (no device call, usable without a GPU): the launch
 * shapes hq_quantize_act and hq_linear choose for `desc` and T tokens on a
 * device with `sms` SMs that holds `pair_clusters` co-resident CTA-pair
 * clusters (0: none), under the automatic GEMM choice.
 *   quant_rows, quant_threads  rows per quantizer tile, threads per CTA;
 *   gemm_pair                  1: the CTA-pair kernel, 0: one CTA per tile;
 *   gemm_bn                    the tile width (256 for the pair).
 * Output pointers are host pointers and may be NULL.  Returns the
 * description's validation status, or HQ_ERR_INVALID_ARGUMENT for T < 1,
 * sms < 1 or pair_clusters < 0. */
hq_status hq_debug_plan(const hq_layer_desc* desc, int64_t T, int sms, int pair_clusters,
                        int32_t* quant_rows, int32_t* quant_threads, int32_t* gemm_pair,
                        int32_t* gemm_bn);

/* Test hook, host only: how many tensor maps hq_linear and hq_quantize_act
 * took from the library's cache and how many they encoded.  A tensor map
 * depends only on its buffer's address, extents and box, so the library keeps
 * the last 64 it encoded and reuses them for later calls on the same buffers
 * and shapes (no per-call encoding on the host).  Outputs are host pointers
 * and may be NULL; counts are cumulative for the process. */
hq_status hq_debug_tmap_cache(uint64_t* hits, uint64_t* misses);

/* Diagnostic hook, host only: the code behind the last HQ_ERR_CUDA any call
 * returned (a cudaError_t value, or 100000 + a CUresult from encoding a
 * tensor map), 0 if none; reading it clears it. */
int hq_debug_last_cuda_error(void);

/* Measurement hook (no counterpart on the pages): the int8 tensor-core
 * ceiling of this device, the denominator the GEMM's throughput is reported
 * against beside the nominal figure.  Launches the GEMM's main loop with
 * nothing but the MMAs: every CTA (one per SM, resident at once) zeroes four
 * operand stages laid out like the GEMM's and one thread issues k_blocks x 4
 * tcgen05.mma kind::i8 of 128 x 256 x 32 into tensor memory (pair = 1:
 * clusters of two CTAs issuing cta_group::2 MMAs of 256 x 256 x 32, the
 * CTA-pair GEMM's shape), then waits for them.  No loads, no epilogue.
 *   pair      0 or 1;  k_blocks  1 .. 2^24 (four MMAs each);
 *   ctas      (host) receives the number of CTAs launched, so that one launch
 *             performs ctas * k_blocks * 4 * 2 * 128 * 256 * 32 integer ops.
 * Time the launch on `stream` with events.  Returns HQ_ERR_UNSUPPORTED for
 * pair = 1 on a device that cannot hold a cluster of two such CTAs. */
hq_status hq_debug_mma_ceiling(int pair, int64_t k_blocks, int32_t* ctas, hq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HQ_H */
